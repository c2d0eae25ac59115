// kq_api.cu — the libkq C ABI: argument validation, schedule planning and
// launch of the fused K-quant GEMV kernels (see include/kq.h).
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/kq.h"
#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {

static thread_local char g_last_error[512] = "";

static int fail(int status, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return status;
}

int set_last_error(int status, const char* msg) { return fail(status, "%s", msg); }

static int cuda_fail(cudaError_t err, const char* what) {
    return fail(KQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

// Per-device properties, read once.
struct DevInfo {
    int sm_count = 0;
    int smem_optin = 0;
    int smem_per_sm = 0;
};
static std::mutex g_dev_mu;
static DevInfo g_dev[64];

static cudaError_t dev_info(DevInfo& out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_dev[dev].sm_count == 0) {
        int sms = 0, smem = 0;
        err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        err = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (err != cudaSuccess) return err;
        int smem_sm = 0;
        err = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        if (err != cudaSuccess) return err;
        g_dev[dev].sm_count = sms;
        g_dev[dev].smem_optin = smem;
        g_dev[dev].smem_per_sm = smem_sm;
    }
    out = g_dev[dev];
    return cudaSuccess;
}

cudaError_t ensure_smem_attr(const void* func, size_t bytes) {
    // cudaFuncSetAttribute is cheap but not free; remember the largest value
    // set per (device, kernel).
    struct Entry {
        int dev;
        const void* func;
        size_t bytes;
    };
    static std::mutex mu;
    static Entry cache[256];
    static int n = 0;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    {
        std::lock_guard<std::mutex> lk(mu);
        for (int i = 0; i < n; ++i)
            if (cache[i].dev == dev && cache[i].func == func && cache[i].bytes >= bytes) return cudaSuccess;
    }
    err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < n; ++i)
        if (cache[i].dev == dev && cache[i].func == func) {
            if (cache[i].bytes < bytes) cache[i].bytes = bytes;
            return cudaSuccess;
        }
    if (n < 256) cache[n++] = Entry{dev, func, bytes};
    return cudaSuccess;
}

static int next_pow2(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

static size_t round_up(size_t v, size_t m) { return (v + m - 1) / m * m; }


int plan_gemv(int fmt, int ncol, GemvArgs& a, LaunchPlan& p) {
    DevInfo di;
    cudaError_t err = dev_info(di);
    if (err != cudaSuccess) return cuda_fail(err, "device query");
    const int nb = a.nbs;  // blocks per K range (all of K unless split)
    if (fmt != KQ_FMT_Q4_K && fmt != KQ_FMT_Q6_K && ncol > 1)
        return fail(KQ_ERR_UNSUPPORTED, "format %d with %d columns: not in this kernel", fmt, ncol);
    // Rows (and split-K ranges) off the 16-byte grid: whole stages are copied
    // from the boundary below their start, but per-row copies (split K) need
    // 16-byte rows, and the several-column Q6_K layout 16-byte blocks groups.
    const bool rows16 = a.row_bytes % 16 == 0;
    if (a.ksplit > 1 && (!rows16 || (static_cast<int64_t>(nb) * kq_block_bytes(fmt)) % 16 != 0))
        return fail(KQ_ERR_UNSUPPORTED, "split K needs 16-byte aligned rows and ranges, K=%lld", (long long)a.K);
    if (fmt == KQ_FMT_Q6_K && ncol > 1 && nb % 8 != 0)
        return fail(KQ_ERR_UNSUPPORTED, "Q6_K with %d columns needs K %% 2048 == 0, K=%lld", ncol, (long long)a.K);
    a.par = 0;
    if (fmt == KQ_FMT_Q6_K && ncol == 1 && nb >= 24 && nb % 2 == 0 && a.row_bytes % 4 == 0) {
        // block-parity lane order: each parity's nb half-block units on whole
        // warps of their own, so that a warp's blocks share their alignment
        const int lr = 2 * static_cast<int>(round_up(nb, 32));
        if (lr > kConsumers) return fail(KQ_ERR_UNSUPPORTED, "K=%lld > 32768", (long long)a.K);
        a.par = nb;
        a.lanes_per_rp = lr;
        a.ps = kConsumers / lr;
        a.parts = lr / 32;
    } else if (fmt != KQ_FMT_Q6_K || ncol == 1) {  // lanes take (row pair, block, half)
        const int ur = 2 * nb;  // half-block units per row pair
        const int lr = ur <= 32 ? next_pow2(ur) : static_cast<int>(round_up(ur, 32));
        if (lr > kConsumers) return fail(KQ_ERR_UNSUPPORTED, "K=%lld > 32768", (long long)a.K);
        a.lanes_per_rp = lr;
        a.ps = kConsumers / lr;
        a.parts = lr > 32 ? lr / 32 : 1;
    } else {
        const int urw = 2 * (nb / 8);  // units per row pair in each of the 8 warps
        if (urw > 32) return fail(KQ_ERR_UNSUPPORTED, "Q6_K with K=%lld > 32768", (long long)a.K);
        const int lrw = next_pow2(urw);
        a.lanes_per_rp = lrw;
        a.ps = 32 / lrw;
        a.parts = kConsumerWarps;
    }
    const size_t srow = a.ksplit > 1 ? static_cast<size_t>(a.nbs) * kq_block_bytes(fmt)
                                     : static_cast<size_t>(a.row_bytes);
    const size_t stage = round_up(static_cast<size_t>(a.ps) * 2 * srow + 32, 128);
    // Two consumer groups (16 compute warps) for the single-column kernels:
    // measured to hide shared-memory latency better than one group; the
    // multi-column kernels need more registers per thread and keep one.
    const int ng = ncol == 1 ? 2 : 1;
    const bool shared_x = a.x_seg_stride == 0;
    // partial sums: the general kernel's group buffers, or (one column) the
    // larger of those and the single-matrix kernel's per-slot buffers
    size_t wp_bytes = round_up(sizeof(float) * ng * 2 * a.ps * a.parts * 2 * ncol, 128);
    if (ncol == 1) {
        const size_t lean = round_up(static_cast<size_t>(kMaxStages) * a.ps * (8 * a.parts + 8), 128);
        if (lean > wp_bytes) wp_bytes = lean;
    }
    // one column: integer activation regions (2 x 336 bytes per
    // super-block); otherwise fp32 regions
    const size_t xcopy = ncol == 1 ? static_cast<size_t>(672) * nb
                                                          : sizeof(float) * ncol * 2 * nb * kRegion;
    const size_t xs_bytes = round_up((shared_x ? 1 : ng) * xcopy, 128);
    const size_t head = kHeadBytes;
    const size_t fixed = head + wp_bytes + xs_bytes;
    const size_t extra = a.pro == KQ_PRO_RMSNORM ? kProBytes : 0;  // RMSNorm scratch after the ring
    const size_t limit = static_cast<size_t>(di.smem_optin) - extra;
    if (fixed + 2 * stage > limit)
        return fail(KQ_ERR_UNSUPPORTED, "K=%lld with %d columns needs %zu bytes of shared memory (limit %zu)",
                    (long long)a.K, ncol, fixed + 2 * stage, limit);
    size_t ns = (limit - fixed) / stage;
    if (ns > kMaxStages) ns = kMaxStages;
    // no more stages than the busiest CTA will ever use
    const int64_t rps = (a.N + 1) / 2;
    const int64_t P = static_cast<int64_t>(a.n_seg) * rps;
    const int64_t ranges = di.sm_count / a.ksplit;        // row-pair ranges per K range
    const int64_t grid = (P < ranges ? P : ranges) * a.ksplit;
    const int64_t per_cta = (P + grid / a.ksplit - 1) / (grid / a.ksplit);
    const int64_t need = (per_cta + a.ps - 1) / a.ps + (a.n_seg > 1 ? 1 : 0);
    if (static_cast<int64_t>(ns) > need) ns = need < 2 ? 2 : static_cast<size_t>(need);
    a.nstage = static_cast<int>(ns);
    a.stage_bytes = static_cast<int>(stage);
    a.wp_offset = static_cast<int>(head);
    a.xs_offset = static_cast<int>(head + wp_bytes);
    a.sbuf_offset = static_cast<int>(fixed);
    p.grid = static_cast<int>(grid);
    p.cluster = 1;
    p.ng = ng;
    a.pro_offset = static_cast<int>(fixed + ns * stage);
    p.smem_bytes = fixed + ns * stage + extra;
    p.pdl = true;
    return KQ_OK;
}

// Shared-memory layout of the tensor-core kernel for K ranges of `nbs`
// blocks split over `S` CTAs of a cluster (S = 1: no cluster).
struct MmaLayout {
    size_t sp, stage, wp, bs, red, xb, fixed;
};
static MmaLayout mma_layout(int fmt, int nt, int nbs, int S, int ng) {
    MmaLayout L;
    // the staged row (which may start up to 14 bytes into the smem row) plus
    // 4 bytes (Q6_K word loads may read 2 bytes past a block), rounded up to
    // the residue mod 128 that spreads the 8 rows of a warp over distinct
    // banks
    const size_t srow = static_cast<size_t>(nbs) * kq_block_bytes(fmt) + 16 + 4;
    const size_t res = fmt == KQ_FMT_Q4_K || fmt == KQ_FMT_Q5_K ? 64 : 16;
    L.sp = srow <= res ? res : round_up(srow - res, 128) + res;
    L.stage = round_up(16 * L.sp, 128);
    const size_t nc = 8 * static_cast<size_t>(nt);  // columns of nt n-tiles
    L.wp = sizeof(float) * ng * 2 * kConsumerWarps * 16 * nc;
    L.bs = round_up(sizeof(float) * 2 * nc * nbs, 128);
    L.red = S > 1 ? sizeof(float) * 2 * (S - 1) * 16 * nc : 0;
    const size_t min_steps = fmt == KQ_FMT_Q6_K || fmt == KQ_FMT_Q8_0 ? 0
                           : fmt == KQ_FMT_Q2_K || fmt == KQ_FMT_Q3_K ? 2 * 256 : 2 * 128;
    L.xb = static_cast<size_t>(nbs) * nt * (16 * 256 + min_steps);
    L.fixed = kHeadBytes + L.wp + L.bs + L.red + L.xb;
    return L;
}

// Instantiation key of the tensor-core kernel per format (+ groups - 1).
static int mma_key(int fmt) {
    switch (fmt) {
        case KQ_FMT_Q4_K: return 0;
        case KQ_FMT_Q6_K: return 2;
        case KQ_FMT_Q5_K: return 4;
        case KQ_FMT_Q8_0: return 6;
        case KQ_FMT_Q2_K: return 8;
        default: return 10;  // Q3_K
    }
}

static cudaError_t active_clusters(int fmt, int nt, int ng, int S, size_t smem, bool pro, int* out) {
    struct Entry {
        int dev, fmt, nt, ng, S;
        size_t smem;
        bool pro;
        int n;
    };
    static std::mutex mu;
    static Entry cache[64];
    static int count = 0;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    {
        std::lock_guard<std::mutex> lk(mu);
        for (int i = 0; i < count; ++i)
            if (cache[i].dev == dev && cache[i].fmt == fmt && cache[i].nt == nt && cache[i].ng == ng &&
                cache[i].S == S && cache[i].smem == smem && cache[i].pro == pro) {
                *out = cache[i].n;
                return cudaSuccess;
            }
    }
    // (one n-tile of 8 columns serves every column count)
    const int key = mma_key(fmt) + (ng - 1);
    switch (key) {
        case 0: err = mma_active_clusters<1, 1, 1>(S, smem, pro, out); break;
        case 1: err = mma_active_clusters<1, 1, 2>(S, smem, pro, out); break;
        case 2: err = mma_active_clusters<2, 1, 1>(S, smem, pro, out); break;
        case 3: err = mma_active_clusters<2, 1, 2>(S, smem, pro, out); break;
        case 4: err = mma_active_clusters<3, 1, 1>(S, smem, pro, out); break;
        case 5: err = mma_active_clusters<3, 1, 2>(S, smem, pro, out); break;
        case 6: err = mma_active_clusters<6, 1, 1>(S, smem, pro, out); break;
        case 7: err = mma_active_clusters<6, 1, 2>(S, smem, pro, out); break;
        case 8: err = mma_active_clusters<4, 1, 1>(S, smem, pro, out); break;
        case 9: err = mma_active_clusters<4, 1, 2>(S, smem, pro, out); break;
        case 10: err = mma_active_clusters<5, 1, 1>(S, smem, pro, out); break;
        default: err = mma_active_clusters<5, 1, 2>(S, smem, pro, out); break;
    }
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lk(mu);
    if (count < 64) cache[count++] = Entry{dev, fmt, nt, ng, S, smem, pro, *out};
    return cudaSuccess;
}

// Schedule of the tensor-core kernel (2..8 columns): 16-row stages, rows
// `sp` bytes apart in smem, B fragments of the CTA's K range for NT
// n-tiles, two partial-sum buffers.  Unless the caller split K itself
// (a.ksplit > 1, partial sums in its workspace), K is split into S equal
// ranges over the CTAs of a cluster when the activations of 8 columns and
// two stages do not fit otherwise: the smallest S (<= 8, dividing the
// blocks) that fits and whose clusters still occupy 85% of the SMs, else
// the fitting S that occupies the most.  The split depends on (format, K)
// only, so every column count sums alike and a column's result does not
// depend on how many columns share the call.
int plan_mma(int fmt, int nt, GemvArgs& a, LaunchPlan& p) {
    DevInfo di;
    cudaError_t err = dev_info(di);
    if (err != cudaSuccess) return cuda_fail(err, "device query");
    if (fmt == KQ_FMT_Q6_K && a.nb % 8 != 0)
        return fail(KQ_ERR_UNSUPPORTED, "Q6_K rows must be 16-byte aligned (K %% 2048 == 0), K=%lld", (long long)a.K);
    // RMSNorm scratch after the ring: 8 columns' sums per super-block, 8 norms
    const size_t extra = a.pro == KQ_PRO_RMSNORM ? round_up(sizeof(float) * (8 * static_cast<size_t>(a.nb) + 8), 128) : 0;
    const size_t limit = static_cast<size_t>(di.smem_optin) - extra;
    int S = a.ksplit, nbs = a.nbs;
    bool cl = false;
    if (S == 1) {
        int best = 0, best_use = 0;
        for (int s = 1; s <= 8 && s <= a.nb; ++s) {
            if (a.nb % s != 0) continue;
            const MmaLayout L8 = mma_layout(fmt, 1, a.nb / s, s, 1);
            if (L8.fixed + 2 * L8.stage > limit) continue;
            int use = di.sm_count;
            if (s > 1) {
                const MmaLayout Ln = mma_layout(fmt, nt, a.nb / s, s, 1);
                size_t nsn = (limit - Ln.fixed) / Ln.stage;
                if (nsn > kMaxStages) nsn = kMaxStages;
                int fit = 0;
                err = active_clusters(fmt, nt, 1, s, Ln.fixed + nsn * Ln.stage + extra, a.pro != 0, &fit);
                if (err != cudaSuccess) return cuda_fail(err, "cluster occupancy query");
                use = fit * s;
            }
            if (use > best_use) {
                best = s;
                best_use = use;
            }
            if (20 * use >= 17 * di.sm_count) {
                best = s;
                break;
            }
        }
        if (best > 1) {
            S = best;
            nbs = a.nb / best;
            cl = true;
        }
    }
    // two consumer groups when they leave room for three stages
    int ng = 2;
    MmaLayout L = mma_layout(fmt, nt, nbs, S, 2);
    if (L.fixed + 3 * L.stage > limit) {
        ng = 1;
        L = mma_layout(fmt, nt, nbs, S, 1);
    }
    if (L.fixed + 2 * L.stage > limit)
        return fail(KQ_ERR_UNSUPPORTED, "K=%lld with %d columns needs %zu bytes of shared memory (limit %zu)",
                    (long long)a.K, 8 * nt, L.fixed + 2 * L.stage, limit);
    size_t ns = (limit - L.fixed) / L.stage;
    if (ns > kMaxStages) ns = kMaxStages;
    const int64_t rps = (a.N + 1) / 2;
    const int64_t tiles = (rps + 7) / 8;  // 16-row stages of the matrix
    int64_t ranges = di.sm_count / S;     // row ranges (clusters, or CTAs per K range)
    if (cl) {
        int fit = 0;
        err = active_clusters(fmt, nt, ng, S, L.fixed + ns * L.stage + extra, a.pro != 0, &fit);
        if (err != cudaSuccess) return cuda_fail(err, "cluster occupancy query");
        if (fit < 1) return fail(KQ_ERR_UNSUPPORTED, "no cluster of %d CTAs fits", S);
        ranges = fit;
    }
    const int64_t grid = (tiles < ranges ? tiles : ranges) * S;
    const int64_t per_cta = (rps + grid / S - 1) / (grid / S);
    const int64_t need = (per_cta + 7) / 8 + 1;
    if (static_cast<int64_t>(ns) > need) ns = need < 2 ? 2 : static_cast<size_t>(need);
    a.ksplit = S;
    a.nbs = nbs;
    a.cluster = cl ? 1 : 0;
    a.ps = 8;
    a.parts = 1;
    a.lanes_per_rp = 0;
    a.sp = static_cast<int>(L.sp);
    a.nstage = static_cast<int>(ns);
    a.stage_bytes = static_cast<int>(L.stage);
    a.wp_offset = kHeadBytes;
    a.xscale_offset = static_cast<int>(kHeadBytes + L.wp);
    a.red_offset = static_cast<int>(kHeadBytes + L.wp + L.bs);
    a.xs_offset = static_cast<int>(kHeadBytes + L.wp + L.bs + L.red);
    a.sbuf_offset = static_cast<int>(L.fixed);
    p.grid = static_cast<int>(grid);
    p.cluster = cl ? S : 1;
    p.ng = ng;
    a.pro_offset = static_cast<int>(L.fixed + ns * L.stage);
    p.smem_bytes = L.fixed + ns * L.stage + extra;
    p.pdl = true;
    return KQ_OK;
}

static bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

static bool known_format(int fmt) { return fmt >= KQ_FMT_Q4_K && fmt <= KQ_FMT_Q8_0; }

static int check_matrix(const void* W, int fmt, int64_t N, int64_t K) {
    if (!known_format(fmt))
        return fail(KQ_ERR_INVALID_ARG, "unknown format %d", fmt);
    if (N < 0 || K < 0) return fail(KQ_ERR_INVALID_ARG, "negative size N=%lld K=%lld", (long long)N, (long long)K);
    if (K % 256 != 0) return fail(KQ_ERR_INVALID_ARG, "K=%lld is not a multiple of 256", (long long)K);
    if (N > 0 && K > 0) {
        if (!W) return fail(KQ_ERR_INVALID_ARG, "W is NULL");
        if (!aligned(W, 16)) return fail(KQ_ERR_INVALID_ARG, "W is not 16-byte aligned");
    }
    if (N > (int64_t(1) << 31)) return fail(KQ_ERR_UNSUPPORTED, "N=%lld too large", (long long)N);
    return KQ_OK;
}

// Kernels exist for 1, 2, 4 and 8 columns; other counts run padded (the
// extra columns repeat the last real one and are not written back), which
// leaves every real column's arithmetic unchanged.
static int padded_cols(int k) { return k <= 1 ? 1 : k <= 2 ? 2 : k <= 4 ? 4 : 8; }

static cudaError_t dispatch(const GemvArgs& a, const LaunchPlan& p, int fmt, int ncol, cudaStream_t s) {
    if (fmt != KQ_FMT_Q4_K && fmt != KQ_FMT_Q6_K) {
        if (ncol != 1) return cudaErrorNotSupported;  // (plan_gemv refuses it first)
        if (fmt == KQ_FMT_Q5_K) return launch_one<3, 1, 2>(a, p, s);
        if (fmt == KQ_FMT_Q2_K) return launch_one<4, 1, 2>(a, p, s);
        if (fmt == KQ_FMT_Q3_K) return launch_one<5, 1, 2>(a, p, s);
        return launch_one<6, 1, 2>(a, p, s);
    }
    if (fmt == KQ_FMT_Q4_K) {
        switch (ncol) {
            case 1: return launch_one<1, 1, 2>(a, p, s);
            case 2: return launch_one<1, 2, 1>(a, p, s);
            case 4: return launch_one<1, 4, 1>(a, p, s);
            default: return launch_one<1, 8, 1>(a, p, s);
        }
    }
    switch (ncol) {
        case 1: return launch_one<2, 1, 2>(a, p, s);
        case 2: return launch_one<2, 2, 1>(a, p, s);
        case 4: return launch_one<2, 4, 1>(a, p, s);
        default: return launch_one<2, 8, 1>(a, p, s);
    }
}

// One column of one whole matrix: the lean single-matrix kernel.
static cudaError_t dispatch_gemv1(const GemvArgs& a, const LaunchPlan& p, int fmt, cudaStream_t s) {
    const bool pro = a.pro != 0;
    switch (fmt) {
        case KQ_FMT_Q4_K: return pro ? launch_gemv1<1, true>(a, p, s) : launch_gemv1<1, false>(a, p, s);
        case KQ_FMT_Q6_K: return pro ? launch_gemv1<2, true>(a, p, s) : launch_gemv1<2, false>(a, p, s);
        case KQ_FMT_Q5_K: return pro ? launch_gemv1<3, true>(a, p, s) : launch_gemv1<3, false>(a, p, s);
        case KQ_FMT_Q2_K: return pro ? launch_gemv1<4, true>(a, p, s) : launch_gemv1<4, false>(a, p, s);
        case KQ_FMT_Q3_K: return pro ? launch_gemv1<5, true>(a, p, s) : launch_gemv1<5, false>(a, p, s);
        default: return pro ? launch_gemv1<6, true>(a, p, s) : launch_gemv1<6, false>(a, p, s);
    }
}

static cudaError_t dispatch_mma(const GemvArgs& a, const LaunchPlan& p, int fmt, cudaStream_t s) {
    // one n-tile of 8 columns serves every column count
    const int key = mma_key(fmt) + (p.ng - 1);
    switch (key) {
        case 0: return launch_mma<1, 1, 1>(a, p, s);
        case 1: return launch_mma<1, 1, 2>(a, p, s);
        case 2: return launch_mma<2, 1, 1>(a, p, s);
        case 3: return launch_mma<2, 1, 2>(a, p, s);
        case 4: return launch_mma<3, 1, 1>(a, p, s);
        case 5: return launch_mma<3, 1, 2>(a, p, s);
        case 6: return launch_mma<6, 1, 1>(a, p, s);
        case 7: return launch_mma<6, 1, 2>(a, p, s);
        case 8: return launch_mma<4, 1, 1>(a, p, s);
        case 9: return launch_mma<4, 1, 2>(a, p, s);
        case 10: return launch_mma<5, 1, 1>(a, p, s);
        default: return launch_mma<5, 1, 2>(a, p, s);
    }
}

// Calls with 2 or more columns (speculative verify) run on the tensor-core
// kernel, every column group of the call included, so a column's arithmetic
// never depends on how the call was grouped.  Its per-row copies need
// 16-byte rows; other shapes run one single-column launch per column.
static bool use_mma(int fmt, int k, int64_t row_bytes) {
    (void)fmt;
    return k >= 2 && row_bytes % 16 == 0;
}

static int plan_for(int fmt, int k, bool mma, GemvArgs& a, LaunchPlan& p) {
    if (mma) return plan_mma(fmt, 1, a, p);
    return plan_gemv(fmt, padded_cols(k), a, p);
}

// kq_inject("hold@S"): the next single-column launch withholds stage S of
// CTA 0 and gives its bounded waits 1 ms (one-shot; 0 = none).
static std::atomic<int> g_inject_hold{0};
constexpr unsigned long long kInjectWaitNs = 1000000ull;

static int run(GemvArgs& a, int fmt, int k, bool mma, cudaStream_t stream) {
    a.ncol_real = k;
    if (!mma && g_inject_hold.load(std::memory_order_relaxed) != 0) {
        const int hold = g_inject_hold.exchange(0);
        if (hold) {
            a.test_hold = hold;
            a.wait_ns = kInjectWaitNs;
        }
    }
    cudaError_t err = fault_word(&a.fault);
    if (err != cudaSuccess) return cuda_fail(err, "fault word");
    LaunchPlan p;
    int st = plan_for(fmt, k, mma, a, p);
    if (st != KQ_OK) return st;
    if (mma) err = dispatch_mma(a, p, fmt, stream);
    else if (k == 1 && a.n_seg == 1 && !a.ids && a.ksplit == 1 && a.x_seg_stride == 0)
        err = dispatch_gemv1(a, p, fmt, stream);
    else err = dispatch(a, p, fmt, padded_cols(k), stream);
    if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
    if (a.ksplit > 1 && !a.cluster) {  // cluster splits add their partial sums in the kernel
        err = launch_splitk_combine(a.partial, a.ksplit, k, a.N, a.y, a.ldy, stream);
        if (err != cudaSuccess) return cuda_fail(err, "split-K combine launch");
    }
    return KQ_OK;
}

// Split over K across CTAs for matrices with fewer row pairs than SMs:
// S ranges of nbs super-blocks each (a multiple of 8 for Q3_K and Q6_K, of
// 4 for Q2_K, keeping every range 16-byte aligned).  A pure function of (fmt, N, K, SM count), so
// single- and multi-column calls split alike.
static void choose_split(int fmt, int64_t N, int nb, int sm_count, int* S, int* nbs) {
    *S = 1;
    *nbs = nb;
    const int64_t P = (N + 1) / 2;
    if (P * 2 > sm_count) return;                       // enough row pairs already
    if (static_cast<int64_t>(nb) * kq_block_bytes(fmt) % 16 != 0) return;  // rows off the 16-byte grid
    const int unit = fmt == KQ_FMT_Q6_K || fmt == KQ_FMT_Q3_K ? 8 : fmt == KQ_FMT_Q2_K ? 4 : 1;
    const int max_s = nb / unit;
    int want = static_cast<int>((sm_count + P - 1) / P);
    if (want > max_s) want = max_s;
    if (want <= 1) return;
    int per = (nb / unit + want - 1) / want * unit;      // blocks per range
    *nbs = per;
    *S = (nb + per - 1) / per;
    if (*S <= 1) *nbs = nb;
}

// Largest padded column count whose staged activations fit in shared
// memory next to a two-stage weight ring (0 if not even one column fits).
static int max_fitting_cols(const GemvArgs& proto, int fmt, bool mma) {
    for (int c = 8; c >= (mma ? 4 : 1); c >>= 1) {
        GemvArgs t = proto;
        LaunchPlan p;
        if (plan_for(fmt, c, mma, t, p) == KQ_OK) return c;
    }
    return 0;
}

// k columns in groups that fit; each group is one launch (the weights are
// read once per group).  Every column's arithmetic is the same whatever the
// grouping, so results do not depend on it.
static int run_grouped(GemvArgs& a, int fmt, int k, cudaStream_t stream) {
    // the tensor-core kernel when its activation fragments fit (for the
    // whole call), else the CUDA-core kernel
    bool mma = use_mma(fmt, k, a.row_bytes);
    int g = mma ? max_fitting_cols(a, fmt, true) : 0;
    if (g == 0) {
        mma = false;
        g = max_fitting_cols(a, fmt, false);
    }
    if (g == 0) {
        LaunchPlan p;
        return plan_for(fmt, 1, false, a, p);  // fails again, recording the reason
    }
    g_last_error[0] = 0;
    for (int c0 = 0; c0 < k; c0 += g) {
        GemvArgs t = a;
        t.x = a.x + static_cast<int64_t>(c0) * a.ldx;
        t.y = a.y + static_cast<int64_t>(c0) * a.ldy;  // partial sums restart at the workspace base
        const int kk = k - c0 < g ? k - c0 : g;
        int st = run(t, fmt, kk, mma, stream);
        if (st != KQ_OK) return st;
    }
    return KQ_OK;
}

// Outputs of an empty dot product (K == 0) are zero.
static int zero_outputs(float* y, int64_t ldy, int64_t rows, int cols, cudaStream_t stream) {
    for (int j = 0; j < cols; ++j) {
        cudaError_t err = cudaMemsetAsync(y + j * ldy, 0, sizeof(float) * rows, stream);
        if (err != cudaSuccess) return cuda_fail(err, "cudaMemsetAsync");
    }
    return KQ_OK;
}

}  // namespace kq

using namespace kq;

extern "C" {

int kq_version(void) { return 100; }

const char* kq_status_str(int status) {
    switch (status) {
        case KQ_OK: return "ok";
        case KQ_ERR_INVALID_ARG: return "invalid argument";
        case KQ_ERR_UNSUPPORTED: return "unsupported";
        case KQ_ERR_NOT_PINNED: return "host memory not pinned";
        case KQ_ERR_OOM: return "out of memory";
        case KQ_ERR_CUDA: return "CUDA error";
        case KQ_ERR_TIMEOUT: return "timeout";
        case KQ_ERR_DEVICE_CHECK: return "device-side check failed";
        case KQ_ERR_INJECTED: return "injected failure";
        default: return "unknown status";
    }
}

const char* kq_last_error(void) { return g_last_error; }

int kq_read_probe(const void* src, size_t bytes, int mode, uint32_t* out, kq_stream_t stream) {
    g_last_error[0] = 0;
    if (mode != 0 && mode != 1) return fail(KQ_ERR_INVALID_ARG, "unknown probe mode %d", mode);
    if (!src || !out || !aligned(src, 16) || !aligned(out, 4) || bytes % 16 != 0)
        return fail(KQ_ERR_INVALID_ARG, "src must be 16-byte aligned, bytes a multiple of 16, out non-NULL");
    if (bytes == 0) return KQ_OK;
    DevInfo di;
    cudaError_t err = dev_info(di);
    if (err != cudaSuccess) return cuda_fail(err, "device query");
    err = launch_probe(src, bytes, mode, out, di.sm_count, reinterpret_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_fail(err, "probe launch");
    return KQ_OK;
}

int kq_inject(const char* spec) {
    g_last_error[0] = 0;
    if (!spec || !spec[0]) {
        g_inject_hold.store(0);
        return KQ_OK;
    }
    if (strncmp(spec, "hold@", 5) == 0) {
        char* end = nullptr;
        const long v = strtol(spec + 5, &end, 10);
        if (end && *end == 0 && v >= 1 && v <= 1000000) {
            g_inject_hold.store(static_cast<int>(v));
            return KQ_OK;
        }
    }
    return fail(KQ_ERR_INVALID_ARG, "unknown injection '%s'", spec);
}

size_t kq_block_bytes(int fmt) {
    switch (fmt) {
        case KQ_FMT_Q4_K: return kQ4Bytes;
        case KQ_FMT_Q6_K: return kQ6Bytes;
        case KQ_FMT_Q5_K: return kQ5Bytes;
        case KQ_FMT_Q2_K: return kQ2Bytes;
        case KQ_FMT_Q3_K: return kQ3Bytes;
        case KQ_FMT_Q8_0: return kQ80Bytes;
        default: return 0;
    }
}

size_t kq_row_bytes(int fmt, int64_t K) {
    if (K < 0 || K % 256 != 0) return 0;
    return static_cast<size_t>(K / 256) * kq_block_bytes(fmt);
}

int kq_device_fault(int* out) {
    g_last_error[0] = 0;
    if (!out) return fail(KQ_ERR_INVALID_ARG, "out is NULL");
    cudaError_t err = read_and_clear_fault(out);
    if (err != cudaSuccess) return cuda_fail(err, "read fault word");
    return KQ_OK;
}

// kq_gemv_multi and kq_gemv_fused: one validation and launch path.
static int gemv_columns(const void* W, int fmt, int64_t N, int64_t K, const float* x, int64_t ldx, int k,
                        const kq_prologue* pro, float* y, int64_t ldy, kq_stream_t stream) {
    g_last_error[0] = 0;
    int st = check_matrix(W, fmt, N, K);
    if (st != KQ_OK) return st;
    if (k < 1 || k > 8) return fail(KQ_ERR_INVALID_ARG, "k=%d outside 1..8", k);
    const int kind = pro ? pro->kind : KQ_PRO_NONE;
    if (kind != KQ_PRO_NONE && kind != KQ_PRO_RMSNORM && kind != KQ_PRO_SWIGLU)
        return fail(KQ_ERR_INVALID_ARG, "unknown prologue kind %d", kind);
    if (kind == KQ_PRO_RMSNORM && (!pro->gamma || !aligned(pro->gamma, 4) || !(pro->eps > 0.f)))
        return fail(KQ_ERR_INVALID_ARG, "RMSNorm needs a 4-byte aligned gamma and eps > 0");
    const int64_t xlen = kind == KQ_PRO_SWIGLU ? 2 * K : K;  // floats per activation column
    if (N == 0) return KQ_OK;
    if (!y || !aligned(y, 4)) return fail(KQ_ERR_INVALID_ARG, "y is NULL or misaligned");
    if (k > 1 && ldy < N) return fail(KQ_ERR_INVALID_ARG, "ldy=%lld < N", (long long)ldy);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (K == 0) return zero_outputs(y, ldy, N, k, s);
    if (!x || !aligned(x, 4)) return fail(KQ_ERR_INVALID_ARG, "x is NULL or misaligned");
    if (k > 1 && ldx < xlen) return fail(KQ_ERR_INVALID_ARG, "ldx=%lld < %lld", (long long)ldx, (long long)xlen);
    GemvArgs a = {};
    a.W = static_cast<const uint8_t*>(W);
    a.N = N;
    a.K = K;
    a.row_bytes = static_cast<int64_t>(kq_row_bytes(fmt, K));
    a.nb = static_cast<int>(K / 256);
    a.n_seg = 1;
    a.ids = nullptr;
    a.E = 1;
    a.seg_stride = 0;
    a.x = x;
    a.ldx = k > 1 ? ldx : xlen;
    a.x_seg_stride = 0;
    a.y = y;
    a.ldy = k > 1 ? ldy : N;
    a.y_seg_stride = 0;
    a.status = nullptr;
    a.ksplit = 1;
    a.nbs = a.nb;
    a.partial = nullptr;
    a.pro = kind;
    a.gamma = kind == KQ_PRO_RMSNORM ? pro->gamma : nullptr;
    a.eps = kind == KQ_PRO_RMSNORM ? pro->eps : 0.f;
    return run_grouped(a, fmt, k, s);
}

int kq_gemv_multi(const void* W, int fmt, int64_t N, int64_t K, const float* x, int64_t ldx, int k, float* y,
                  int64_t ldy, kq_stream_t stream) {
    return gemv_columns(W, fmt, N, K, x, ldx, k, nullptr, y, ldy, stream);
}

int kq_gemv_fused(const void* W, int fmt, int64_t N, int64_t K, const float* x, int64_t ldx, int k,
                  const kq_prologue* pro, float* y, int64_t ldy, kq_stream_t stream) {
    return gemv_columns(W, fmt, N, K, x, ldx, k, pro, y, ldy, stream);
}

int kq_gemv_steps(const kq_step* steps, int n_steps, kq_stream_t stream) {
    g_last_error[0] = 0;
    if (n_steps < 0) return fail(KQ_ERR_INVALID_ARG, "n_steps=%d < 0", n_steps);
    if (n_steps == 0) return KQ_OK;
    if (!steps) return fail(KQ_ERR_INVALID_ARG, "steps is NULL");
    DevInfo di;
    cudaError_t err = dev_info(di);
    if (err != cudaSuccess) return cuda_fail(err, "device query");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // validate and plan every step (the single-column kernel's schedule)
    struct Planned {
        StepArgs a;
        size_t stage, wp, xs;
        bool zero;  // K = 0: y is all zeros
        bool skip;  // N = 0: nothing to do
    };
    std::vector<Planned> pl(static_cast<size_t>(n_steps));
    for (int i = 0; i < n_steps; ++i) {
        const kq_step& q = steps[i];
        Planned& P = pl[static_cast<size_t>(i)];
        P.zero = P.skip = false;
        int st = check_matrix(q.W, q.fmt, q.N, q.K);
        const int kind = q.pro.kind;
        if (st == KQ_OK && kind != KQ_PRO_NONE && kind != KQ_PRO_RMSNORM && kind != KQ_PRO_SWIGLU)
            st = fail(KQ_ERR_INVALID_ARG, "unknown prologue kind %d", kind);
        if (st == KQ_OK && kind == KQ_PRO_RMSNORM && (!q.pro.gamma || !aligned(q.pro.gamma, 4) || !(q.pro.eps > 0.f)))
            st = fail(KQ_ERR_INVALID_ARG, "RMSNorm needs a 4-byte aligned gamma and eps > 0");
        if (st == KQ_OK && q.N > 0 && (!q.y || !aligned(q.y, 4))) st = fail(KQ_ERR_INVALID_ARG, "y is NULL or misaligned");
        if (st == KQ_OK && q.N > 0 && q.K > 0 && (!q.x || !aligned(q.x, 4)))
            st = fail(KQ_ERR_INVALID_ARG, "x is NULL or misaligned");
        if (st == KQ_OK && q.N > 0 && q.K > 0) {
            GemvArgs a = {};
            a.W = static_cast<const uint8_t*>(q.W);
            a.N = q.N;
            a.K = q.K;
            a.row_bytes = static_cast<int64_t>(kq_row_bytes(q.fmt, q.K));
            a.nb = static_cast<int>(q.K / 256);
            a.n_seg = 1;
            a.E = 1;
            a.ksplit = 1;
            a.nbs = a.nb;
            a.ncol_real = 1;
            a.pro = kind;
            LaunchPlan lp;
            st = plan_gemv(q.fmt, 1, a, lp);
            if (st == KQ_OK) {
                StepArgs& sa = P.a;
                sa = StepArgs{};
                sa.W = a.W;
                sa.x = q.x;
                sa.y = q.y;
                sa.gamma = kind == KQ_PRO_RMSNORM ? q.pro.gamma : nullptr;
                sa.N = q.N;
                sa.row_bytes = a.row_bytes;
                sa.K = static_cast<int>(q.K);
                sa.nb = a.nb;
                sa.fmt = q.fmt;
                sa.pro = kind;
                sa.eps = kind == KQ_PRO_RMSNORM ? q.pro.eps : 0.f;
                sa.after = q.after != 0;
                sa.ps = a.ps;
                sa.lanes_per_rp = a.lanes_per_rp;
                sa.par = a.par;
                sa.parts = a.parts;
                P.stage = static_cast<size_t>(a.stage_bytes);
                P.wp = static_cast<size_t>(a.xs_offset - a.wp_offset);
                P.xs = static_cast<size_t>(a.sbuf_offset - a.xs_offset);
            }
        }
        if (st != KQ_OK) {
            char msg[512];
            snprintf(msg, sizeof(msg), "%s", g_last_error);
            return fail(st, "step %d: %s", i, msg);
        }
        P.skip = q.N == 0;
        P.zero = !P.skip && q.K == 0;
    }
    // launches: runs of at most kMaxSteps steps, ended also by a K = 0 step
    // (its zeros are written in stream order between launches)
    struct Op {
        bool zero;
        float* y;
        int64_t N;
        StepsArgs args;
        size_t smem;
    };
    std::vector<Op> ops;
    std::vector<int> run;
    auto close_run = [&]() -> int {
        if (run.empty()) return KQ_OK;
        Op op = {};
        op.zero = false;
        size_t slot = 0, wp = 0, xs = 0;
        bool rms = false;
        for (size_t j = 0; j < run.size(); ++j) {
            const Planned& P = pl[static_cast<size_t>(run[j])];
            op.args.st[j] = P.a;
            slot = P.stage > slot ? P.stage : slot;
            wp = P.wp > wp ? P.wp : wp;
            xs = P.xs > xs ? P.xs : xs;
            rms = rms || P.a.pro == KQ_PRO_RMSNORM;
        }
        op.args.n = static_cast<int>(run.size());
        const size_t pro = rms ? kProBytes : 0;
        const size_t fixed = round_up(kHeadBytes + wp + xs + pro, 128);
        const size_t limit = static_cast<size_t>(di.smem_optin);
        size_t ns = fixed + 2 * slot <= limit ? (limit - fixed) / slot : 0;
        if (ns < 2)
            return fail(KQ_ERR_UNSUPPORTED, "steps %d..%d need %zu bytes of shared memory together (limit %zu)",
                        run.front(), run.back(), fixed + 2 * slot, limit);
        if (ns > kMaxStages) ns = kMaxStages;
        op.args.ns = static_cast<int>(ns);
        op.args.slot_bytes = static_cast<int>(slot);
        op.args.wp_offset = kHeadBytes;
        op.args.xs_offset = static_cast<int>(kHeadBytes + wp);
        op.args.pro_offset = static_cast<int>(kHeadBytes + wp + xs);
        op.args.sbuf_offset = static_cast<int>(fixed);
        op.smem = fixed + ns * slot;
        ops.push_back(op);
        run.clear();
        return KQ_OK;
    };
    for (int i = 0; i < n_steps; ++i) {
        const Planned& P = pl[static_cast<size_t>(i)];
        if (P.skip) continue;
        if (P.zero) {
            int st = close_run();
            if (st != KQ_OK) return st;
            Op op = {};
            op.zero = true;
            op.y = steps[i].y;
            op.N = steps[i].N;
            ops.push_back(op);
            continue;
        }
        run.push_back(i);
        if (static_cast<int>(run.size()) == kMaxSteps) {
            int st = close_run();
            if (st != KQ_OK) return st;
        }
    }
    int st = close_run();
    if (st != KQ_OK) return st;
    int* fault = nullptr;
    err = fault_word(&fault);
    if (err != cudaSuccess) return cuda_fail(err, "fault word");
    for (Op& op : ops) {
        if (op.zero) {
            st = zero_outputs(op.y, op.N, op.N, 1, s);
            if (st != KQ_OK) return st;
            continue;
        }
        op.args.fault = fault;
        err = steps_sync_pair(&op.args.sync);
        if (err != cudaSuccess) return cuda_fail(err, "step counters");
        err = launch_steps<2>(op.args, di.sm_count, op.smem, true, s);
        if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
    }
    return KQ_OK;
}

int kq_gemv(const void* W, int fmt, int64_t N, int64_t K, const float* x, float* y, kq_stream_t stream) {
    return kq_gemv_multi(W, fmt, N, K, x, K, 1, y, N, stream);
}

int kq_moe_gemv(const void* W_experts, int fmt, int E, int64_t N, int64_t K, size_t expert_stride_bytes,
                const int32_t* ids, int n_ids, const float* x, int64_t x_stride, float* y, int32_t* status,
                kq_stream_t stream) {
    g_last_error[0] = 0;
    int st = check_matrix(W_experts, fmt, N, K);
    if (st != KQ_OK) return st;
    if (E < 1) return fail(KQ_ERR_INVALID_ARG, "E=%d < 1", E);
    if (n_ids < 0) return fail(KQ_ERR_INVALID_ARG, "n_ids=%d < 0", n_ids);
    if (n_ids == 0 || N == 0) return KQ_OK;
    if (!ids || !aligned(ids, 4)) return fail(KQ_ERR_INVALID_ARG, "ids is NULL or misaligned");
    if (!y || !aligned(y, 4)) return fail(KQ_ERR_INVALID_ARG, "y is NULL or misaligned");
    if (status && !aligned(status, 4)) return fail(KQ_ERR_INVALID_ARG, "status misaligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (K == 0) return zero_outputs(y, N, N, n_ids, s);
    const size_t rb = kq_row_bytes(fmt, K);
    if (expert_stride_bytes < static_cast<size_t>(N) * rb || expert_stride_bytes % 16 != 0)
        return fail(KQ_ERR_INVALID_ARG, "expert stride %zu must be >= N*row_bytes and a multiple of 16",
                    expert_stride_bytes);
    if (!x || !aligned(x, 4)) return fail(KQ_ERR_INVALID_ARG, "x is NULL or misaligned");
    if (x_stride != 0 && x_stride < K) return fail(KQ_ERR_INVALID_ARG, "x_stride=%lld < K", (long long)x_stride);
    GemvArgs a = {};
    a.W = static_cast<const uint8_t*>(W_experts);
    a.N = N;
    a.K = K;
    a.row_bytes = static_cast<int64_t>(rb);
    a.nb = static_cast<int>(K / 256);
    a.n_seg = n_ids;
    a.ids = ids;
    a.E = E;
    a.seg_stride = static_cast<int64_t>(expert_stride_bytes);
    a.x = x;
    a.ldx = K;
    a.x_seg_stride = x_stride;
    a.y = y;
    a.ldy = 0;
    a.y_seg_stride = N;
    a.status = status;
    a.ksplit = 1;
    a.nbs = a.nb;
    a.partial = nullptr;
    return run(a, fmt, 1, false, s);
}

static int split_for(int fmt, int64_t N, int64_t K, int* S, int* nbs) {
    DevInfo di;
    cudaError_t err = dev_info(di);
    if (err != cudaSuccess) return cuda_fail(err, "device query");
    choose_split(fmt, N, static_cast<int>(K / 256), di.sm_count, S, nbs);
    return KQ_OK;
}

size_t kq_splitk_workspace_bytes(int fmt, int64_t N, int64_t K, int k) {
    if (!known_format(fmt) || N < 1 || K < 256 || K % 256 != 0 || k < 1 ||
        k > 8)
        return 0;
    int S = 1, nbs = 0;
    if (split_for(fmt, N, K, &S, &nbs) != KQ_OK || S <= 1) return 0;
    return sizeof(float) * static_cast<size_t>(S) * k * static_cast<size_t>(N);
}

int kq_gemv_splitk(const void* W, int fmt, int64_t N, int64_t K, const float* x, int64_t ldx, int k, float* y,
                   int64_t ldy, void* workspace, size_t workspace_bytes, kq_stream_t stream) {
    g_last_error[0] = 0;
    int st = check_matrix(W, fmt, N, K);
    if (st != KQ_OK) return st;
    if (k < 1 || k > 8) return fail(KQ_ERR_INVALID_ARG, "k=%d outside 1..8", k);
    if (N == 0 || K == 0) return kq_gemv_multi(W, fmt, N, K, x, ldx, k, y, ldy, stream);
    int S = 1, nbs = 0;
    st = split_for(fmt, N, K, &S, &nbs);
    if (st != KQ_OK) return st;
    if (S <= 1) return kq_gemv_multi(W, fmt, N, K, x, ldx, k, y, ldy, stream);
    const size_t need = sizeof(float) * static_cast<size_t>(S) * k * static_cast<size_t>(N);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 4))
        return fail(KQ_ERR_INVALID_ARG, "workspace of %zu bytes needed (got %zu)", need, workspace_bytes);
    if (!y || !aligned(y, 4) || !x || !aligned(x, 4)) return fail(KQ_ERR_INVALID_ARG, "x or y NULL or misaligned");
    if (k > 1 && (ldx < K || ldy < N)) return fail(KQ_ERR_INVALID_ARG, "ldx < K or ldy < N");
    GemvArgs a = {};
    a.W = static_cast<const uint8_t*>(W);
    a.N = N;
    a.K = K;
    a.row_bytes = static_cast<int64_t>(kq_row_bytes(fmt, K));
    a.nb = static_cast<int>(K / 256);
    a.n_seg = 1;
    a.E = 1;
    a.x = x;
    a.ldx = k > 1 ? ldx : K;
    a.y = y;
    a.ldy = k > 1 ? ldy : N;
    a.ksplit = S;
    a.nbs = nbs;
    a.partial = static_cast<float*>(workspace);
    return run_grouped(a, fmt, k, reinterpret_cast<cudaStream_t>(stream));
}

int kq_unpack(const void* W, int fmt, int64_t n_blocks, int8_t* q, uint8_t* sc_or_s, uint8_t* m, float* d,
              float* dmin, kq_stream_t stream) {
    g_last_error[0] = 0;
    if (!known_format(fmt)) return fail(KQ_ERR_INVALID_ARG, "unknown format %d", fmt);
    if (n_blocks < 0) return fail(KQ_ERR_INVALID_ARG, "n_blocks < 0");
    if (n_blocks == 0) return KQ_OK;
    if (!W || !q || !sc_or_s || !d) return fail(KQ_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(W, 16) || !aligned(d, 4) || !aligned(dmin, 4)) return fail(KQ_ERR_INVALID_ARG, "misaligned pointer");
    cudaError_t err = launch_unpack(static_cast<const uint8_t*>(W), fmt, n_blocks, reinterpret_cast<uint8_t*>(q),
                                    sc_or_s, m, d, dmin, true, reinterpret_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_fail(err, "unpack launch");
    return KQ_OK;
}

int kq_unpack_fields(const void* W, int fmt, int64_t n_blocks, uint8_t* q, uint8_t* sc, float* d,
                     kq_stream_t stream) {
    g_last_error[0] = 0;
    if (!known_format(fmt)) return fail(KQ_ERR_INVALID_ARG, "unknown format %d", fmt);
    if (n_blocks < 0) return fail(KQ_ERR_INVALID_ARG, "n_blocks < 0");
    if (n_blocks == 0) return KQ_OK;
    if (!W || !q || !sc || !d) return fail(KQ_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(W, 16) || !aligned(d, 4)) return fail(KQ_ERR_INVALID_ARG, "misaligned pointer");
    cudaError_t err = launch_unpack(static_cast<const uint8_t*>(W), fmt, n_blocks, q, sc, nullptr, d, nullptr, false,
                                    reinterpret_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_fail(err, "unpack launch");
    return KQ_OK;
}

}  // extern "C"
