// kq_steps.cuh — several single-column GEMVs in one persistent launch.
//
// A decode step is a chain of matrix-vector products, each a launch of its
// own in the single-column kernel, and every launch pays its start: the
// producer of launch n+1 can only begin fetching weights once the CTA of
// launch n on that SM has exited (one CTA fills an SM), so HBM idles while
// the new CTAs fetch their first stages and stage their activations.  Here
// one grid of one CTA per SM runs a list of GEMVs ("steps"): the producer
// warp streams the weights of step after step without a break (weights
// never depend on an earlier step), while the consumers take the steps in
// order.  A step marked `after` reads activations that an earlier step of
// the same launch writes; its consumers start only once every CTA has
// finished the steps before it (a grid-wide counter, waited on with a
// bound).  Each step is computed exactly as the single-column kernel
// computes it (same units, lane layout, staging and summation order), so
// its outputs equal that kernel's bit for bit.
//
// The method and its sources are those of the single-column kernel: the
// fused dequant-matmul of "Kortex: Streaming 70B Models on Consumer GPUs"
// (Key components 3) and of "Out-of-core LLM inference engine written from
// scratch in Rust" (Approach), over whole decode chains.
#pragma once

#include "kq_gemv.cuh"

namespace kq {

// The CTA's row pairs of a step: [P*b/G, P*(b+1)/G) of its P row pairs.
__device__ __forceinline__ void step_range(const StepArgs& s, int b, int G, int& rp0, int& rp1) {
    const int64_t P = (s.N + 1) / 2;
    rp0 = static_cast<int>(P * b / G);
    rp1 = static_cast<int>(P * (b + 1) / G);
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// A GemvArgs view of one step for the staging passes (single column,
// shared activations, K unsplit).
__device__ __forceinline__ GemvArgs step_view(const StepArgs& s) {
    GemvArgs a = {};
    a.W = s.W;
    a.N = s.N;
    a.K = s.K;
    a.row_bytes = s.row_bytes;
    a.nb = s.nb;
    a.nbs = s.nb;
    a.n_seg = 1;
    a.E = 1;
    a.x = s.x;
    a.ldx = s.pro == 2 ? 2 * static_cast<int64_t>(s.K) : s.K;
    a.y = s.y;
    a.ldy = s.N;
    a.ncol_real = 1;
    a.ksplit = 1;
    a.ps = s.ps;
    a.lanes_per_rp = s.lanes_per_rp;
    a.par = s.par;
    a.parts = s.parts;
    a.pro = s.pro;
    a.gamma = s.gamma;
    a.eps = s.eps;
    return a;
}

template <int NG>
__global__ void __launch_bounds__(32 + NG * kConsumers, 1) steps_kernel(const __grid_constant__ StepsArgs A) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 2 * kMaxStages * 8);
    uint8_t* sbuf = smem + A.sbuf_offset;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ns = A.ns;
    const int b = static_cast<int>(blockIdx.x), G = static_cast<int>(gridDim.x);

    if (tid == 0) {
        for (int s = 0; s < ns; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // fault reports go through a GemvArgs view (raise_fault's interface)
    GemvArgs fa = {};
    fa.fault = A.fault;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();
            int slot = -1, count = 0;
            uint32_t phase = 0;
            bool ok = true;
            RingTrack ring;
            for (int si = 0; si < A.n && ok; ++si) {
                const StepArgs& s = A.st[si];
                int rp0, rp1;
                step_range(s, b, G, rp0, rp1);
                for (int off = rp0; off < rp1; off += s.ps) {
                    const int nrp = rp1 - off < s.ps ? rp1 - off : s.ps;
                    const int64_t row0 = 2 * static_cast<int64_t>(off);
                    const int64_t rows = s.N - row0 < 2 * nrp ? s.N - row0 : 2 * nrp;
                    if (++slot == ns) {
                        slot = 0;
                        phase ^= 1u;
                    }
                    ++count;
                    if (count > ns && !mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag)) {
                        raise_fault(fa, abort_flag, 6);
                        ok = false;
                        break;
                    }
                    if (*abort_flag) {  // nothing more is issued once the CTA has aborted
                        ok = false;
                        break;
                    }
                    // from the 16-byte boundary at or below the stage's
                    // first byte (rows need not be 16-byte aligned)
                    const uintptr_t s0 = reinterpret_cast<uintptr_t>(s.W + row0 * s.row_bytes);
                    const uintptr_t b0 = s0 & ~uintptr_t(15);
                    const uintptr_t e0 = (s0 + static_cast<uintptr_t>(rows * s.row_bytes) + 15) & ~uintptr_t(15);
                    const uint32_t bytes = static_cast<uint32_t>(e0 - b0);
                    mbar_arrive_expect_tx(&full[slot], bytes);
                    bulk_g2s(sbuf + static_cast<size_t>(slot) * A.slot_bytes, reinterpret_cast<const void*>(b0), bytes,
                             &full[slot], pol);
                    ring.issue(slot, phase);
                }
            }
            // let every copy issued land before the CTA can exit, abort or
            // not (bounded)
            ring.drain(full, ns);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int ct_all = tid - 32;               // 0 .. NG*256-1
    const int g = NG == 2 ? (ct_all >> 8) : 0;
    const int ct = ct_all & (kConsumers - 1);  // thread within the group
    const int gbar = 1 + g;                    // the group's named barrier
    const int nthr = NG * kConsumers;          // all consumer threads (named barrier 3)
    const uint32_t xs_s = smem_u32(smem + A.xs_offset);
    const uint32_t sbuf_s = smem_u32(sbuf);
    const uint32_t pro_r = smem_u32(smem + A.pro_offset);
    pdl_wait();  // the first step's activations may come from the previous grid
    pdl_launch_dependents();

    int k = -1;  // the CTA's stage sequence number (the producer's order)
    int own = 0;  // stages this group has reduced (partial-sum buffer parity)
    for (int si = 0; si < A.n; ++si) {
        const StepArgs& s = A.st[si];
        if (si > 0) {
            // every consumer is done with the previous step's activations and
            // has written its outputs; publish this CTA's completion of it
            named_bar_sync(3, nthr);
            if (ct_all == 0) {
                __threadfence();
                atomicAdd(A.sync, 1);
            }
        }
        if (s.after && si > 0) {
            // wait until every CTA has finished steps 0 .. si-1
            if (ct_all == 0 && !*abort_flag) {
                const int target = si * G;
                const unsigned long long t0 = globaltimer_ns();
                while (ld_acquire_gpu(A.sync) < target) {
                    if (globaltimer_ns() - t0 > kWaitNs) {
                        raise_fault(fa, abort_flag, 6);
                        break;
                    }
                    __nanosleep(64);
                }
                __threadfence();
            }
            named_bar_sync(3, nthr);
        }
        // this step's activations, staged by all consumer threads
        const GemvArgs a = step_view(s);
        float rinv = 1.f;
        if (s.fmt == 2 || s.fmt == 4 || s.fmt == 5) {  // Q2_K, Q3_K, Q6_K: integer regions with 16-sums
            if (s.pro) stage_all<2, 1, true, true>(a, 0, xs_s, ct_all, nthr, 3, 0, s.nb, pro_r);
            else stage_all<2, 1, true, false>(a, 0, xs_s, ct_all, nthr, 3, 0, s.nb, pro_r);
        } else {  // Q4_K, Q5_K, Q8_0: integer regions
            if (s.pro) stage_all<1, 1, true, true>(a, 0, xs_s, ct_all, nthr, 3, 0, s.nb, pro_r);
            else stage_all<1, 1, true, false>(a, 0, xs_s, ct_all, nthr, 3, 0, s.nb, pro_r);
        }
        if (s.pro == 1) rinv = ld_s32f(pro_inv_addr(pro_r));

        // this lane's unit within a stage (as in the single-column kernel)
        const int nb = s.nb;
        const int LR = s.lanes_per_rp;
        const LaneUnit L = lane_unit(ct, LR, nb, s.par);
        const int u_rp = L.rp, u_b = L.b, u_H = L.H;
        const bool u_active = L.active;
        const int group = LR < 32 ? LR : 32;
        const int part = LR > 32 ? ((ct - u_rp * LR) >> 5) : 0;
        const int parts = s.parts;
        const bool direct = parts == 1;
        const uint32_t xri = xs_s + kXRegionBytes * L.pos;
        const uint32_t wp_s = smem_u32(smem + A.wp_offset) + 4 * g * (2 * s.ps * parts * 2);
        const int srow = static_cast<int>(s.row_bytes);

        int rp0, rp1;
        step_range(s, b, G, rp0, rp1);
        for (int off = rp0; off < rp1; off += s.ps) {
            ++k;
            if (NG == 2 && (k & 1) != g) continue;
            const int slot = k % ns;
            const uint32_t phase = static_cast<uint32_t>((k / ns) & 1);
            const int nrp = rp1 - off < s.ps ? rp1 - off : s.ps;
            const int64_t row0 = 2 * static_cast<int64_t>(off);
            const int nrows = static_cast<int>(s.N - row0 < 2 * nrp ? s.N - row0 : 2 * nrp);
            // with an odd ring depth, first the other group's release of the
            // slot's previous stage (see gemv_kernel)
            if (NG == 2 && (ns & 1) && k >= ns && !mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag))
                raise_fault(fa, abort_flag, 6);
            if (!mbar_wait_bounded(&full[slot], phase, abort_flag)) raise_fault(fa, abort_flag, 6);
            float out[2][1] = {{0.f}, {0.f}};
            const bool work = u_active && u_rp < nrp && !*abort_flag;
            if (work) {
                const uint32_t rw = sbuf_s + slot * A.slot_bytes + 2 * u_rp * srow +
                                    static_cast<uint32_t>(reinterpret_cast<uintptr_t>(s.W + row0 * s.row_bytes) & 15u);
                if (s.fmt == 1) q4k_unit_int(rw, srow, u_b, u_H, xri, out);
                else if (s.fmt == 3) q5k_unit_int(rw, srow, u_b, u_H, xri, out);
                else if (s.fmt == 4) q2k_unit_int(rw, srow, u_b, u_H, xri, out);
                else if (s.fmt == 5) q3k_unit_int(rw, srow, u_b, u_H, xri, out);
                else if (s.fmt == 6) q80_unit_int(rw, srow, u_b, u_H, xri, out);
                else if (s.par == 0) q6k_unit_int<2>(rw, srow, u_b, u_H, xri, out);
                else if (u_b & 1) q6k_unit_int<1>(rw, srow, u_b, u_H, xri, out);
                else q6k_unit_int<0>(rw, srow, u_b, u_H, xri, out);
            }
            // butterfly over the lanes of this row pair (fixed order)
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                if (o < group) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) out[r][0] += __shfl_xor_sync(0xffffffffu, out[r][0], o);
                }
            }
            if (direct) {
                // the warp holds whole row pairs: its lead lanes write y
                if (lane == 0) mbar_arrive(&empty[slot]);
                if ((lane & (group - 1)) == 0 && u_rp < nrp) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int row = 2 * u_rp + r;
                        if (row < nrows) s.y[row0 + row] = out[r][0] * rinv;
                    }
                }
                continue;
            }
            // partial sums of the parts, fixed-order sum, then store
            const uint32_t wb = wp_s + 4 * ((own & 1) * (s.ps * parts * 2));
            ++own;
            if ((lane & (group - 1)) == 0 && u_rp < s.ps) {
#pragma unroll
                for (int r = 0; r < 2; ++r) st_s32f(wb + 4 * ((u_rp * parts + part) * 2 + r), out[r][0]);
            }
            named_bar_sync(gbar, kConsumers);
            if (lane == 0) mbar_arrive(&empty[slot]);
            for (int t = ct; t < nrows; t += kConsumers) {
                const int rp = t >> 1, r = t & 1;
                float v = 0.f;
                for (int p = 0; p < parts; ++p) v += ld_s32f(wb + 4 * ((rp * parts + p) * 2 + r));
                s.y[row0 + t] = v * rinv;
            }
        }
    }
    // the last CTA to finish resets the pair for the next launch that gets it
    named_bar_sync(3, nthr);
    if (ct_all == 0) {
        __threadfence();
        if (atomicAdd(A.sync + 1, 1) == G - 1) {
            atomicExch(A.sync, 0);
            atomicExch(A.sync + 1, 0);
            __threadfence();
        }
    }
}

template <int NG>
cudaError_t launch_steps(const StepsArgs& a, int grid, size_t smem_bytes, bool pdl, cudaStream_t stream) {
    auto kern = steps_kernel<NG>;
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem_bytes);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(32 + NG * kConsumers);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace kq
