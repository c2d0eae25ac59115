// kq_internal.h — host/device shared definitions of libkq (not installed).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace kq {

// Kernel arguments of one fused GEMV launch.  A launch covers n_seg
// "segments" of N rows each: one matrix (n_seg = 1), or the routed experts
// of a MoE layer (segment i = expert ids[i]).
struct GemvArgs {
    const uint8_t* W;        // matrix, or expert 0 of the expert stack
    int64_t N, K;
    int64_t row_bytes;
    int nb;                  // super-blocks per row (K / 256)
    int n_seg;
    const int32_t* ids;      // routed expert ids (device) or nullptr
    int E;                   // valid segment ids are [0, E)
    int64_t seg_stride;      // bytes between experts
    const float* x;
    int64_t ldx;             // floats between activation columns
    int64_t x_seg_stride;    // floats between segments' activations (0 = shared)
    float* y;
    int64_t ldy;             // floats between output columns
    int64_t y_seg_stride;    // floats between segments' outputs
    int32_t* status;         // optional device status word
    int* fault;              // device fault word (timeouts)
    int ncol_real;           // columns written (the kernel may pad to 2/4/8)
    // split-K across CTAs (ksplit == 1: every CTA covers all of K)
    int ksplit;              // number of K ranges
    int nbs;                 // super-blocks per K range (the last may be shorter)
    float* partial;          // ksplit x ncol_real x N partial sums (ksplit > 1)
    // schedule (from plan_gemv)
    int ps;                  // row pairs per stage
    int lanes_per_rp;        // lanes per row pair (several-column Q6_K: per row pair and warp)
    int par;                 // single-column Q6_K: block-parity lane order over par blocks (0: off)
    int parts;               // partial sums per row pair
    int nstage;
    int stage_bytes;
    int wp_offset, xs_offset, sbuf_offset;
    // tensor-core (multi-column) kernel only
    int sp;                  // smem bytes between staged rows (padded)
    int xscale_offset;       // power-of-two scales per super-block and column
    int cluster;             // 1: the ksplit K ranges are the CTAs of a cluster, reduced in shared memory
    int red_offset;          // cluster reduction buffers (rank 0)
    // activation prologue (kq_prologue): applied while staging
    int pro;                 // 0 none, 1 RMSNorm, 2 SwiGLU ([g; u] columns of 2K floats)
    const float* gamma;      // RMSNorm weights (K)
    float eps;
    int pro_offset;          // RMSNorm scratch (kProBytes) after the stage ring
    // test hooks (kq_inject): CTA 0's producer never copies its stage number
    // test_hold (1-based; 0 = none), and CTA 0's bounded waits give up after
    // wait_ns (0 = the default limit)
    int test_hold;
    unsigned long long wait_ns;
};

// ---------------------------------------------------- multi-step launch

constexpr int kMaxSteps = 16;  // steps per launch (the host splits longer lists)

// One step of a multi-step launch as the kernel sees it (planned on the host).
struct StepArgs {
    const uint8_t* W;
    const float* x;
    float* y;
    const float* gamma;  // RMSNorm weights (pro == 1)
    int64_t N;
    int64_t row_bytes;
    int K, nb, fmt, pro;
    float eps;
    int after;           // wait for every CTA to finish the steps before this one
    int ps;              // row pairs per stage
    int lanes_per_rp;    // as in GemvArgs
    int par;             // as in GemvArgs
    int parts;
};

struct StepsArgs {
    StepArgs st[kMaxSteps];
    int n;
    int ns;              // ring slots
    int slot_bytes;      // bytes between ring slots (the largest stage)
    int wp_offset, xs_offset, pro_offset, sbuf_offset;
    int* sync;           // (step completions, CTAs finished) pair, zero between launches
    int* fault;
};

// Launch of the multi-step kernel (NG consumer groups), one CTA per SM.
template <int NG>
cudaError_t launch_steps(const StepsArgs& a, int grid, size_t smem_bytes, bool pdl, cudaStream_t stream);
// The next counter pair of this device's pool for a multi-step launch.
cudaError_t steps_sync_pair(int** out);
constexpr int kSyncPairs = 4096;

// Shared-memory scratch of RMSNorm in the single-column kernel: per consumer
// group, partial sums of squares (16 warps x 8 columns) and the columns'
// 1/rms.  Reserved only by launches that normalise.  (The tensor-core
// kernel sizes its own: 8 columns x the row's super-blocks, and 8 floats.)
constexpr int kProBytes = 2 * 4 * (8 * 16 + 8);
constexpr int kHeadBytes = 256;  // barriers and flags

struct LaunchPlan {
    int grid;
    int cluster;     // CTAs per cluster (1: no cluster launch)
    int ng;          // consumer groups of 8 warps (1 or 2)
    size_t smem_bytes;
    bool pdl;
};

// Fills the schedule fields of `a` and the launch plan; returns a kq_status.
int plan_gemv(int fmt, int ncol, GemvArgs& a, LaunchPlan& p);

template <int FMT, int NCOL, int NG>
cudaError_t launch_one(const GemvArgs& a, const LaunchPlan& p, cudaStream_t stream);
// The single-column GEMV of one whole matrix (one segment, K unsplit).
template <int FMT, bool PRO>
cudaError_t launch_gemv1(const GemvArgs& a, const LaunchPlan& p, cudaStream_t stream);
// Tensor-core kernel for 2..8 columns: NT n-tiles of 8 columns (NT = 1).
int plan_mma(int fmt, int nt, GemvArgs& a, LaunchPlan& p);
template <int FMT, int NT, int NG>
cudaError_t launch_mma(const GemvArgs& a, const LaunchPlan& p, cudaStream_t stream);
template <int FMT, int NT, int NG>
cudaError_t mma_active_clusters(int cluster, size_t smem_bytes, bool pro, int* out);
cudaError_t fault_word(int** out);
cudaError_t launch_splitk_combine(const float* partial, int S, int ncol, int64_t N, float* y, int64_t ldy,
                                  cudaStream_t stream);
cudaError_t launch_unpack(const uint8_t* W, int fmt, int64_t nblocks, uint8_t* q, uint8_t* sc, uint8_t* m, float* d,
                          float* dmin, bool split, cudaStream_t stream);
cudaError_t ensure_smem_attr(const void* func, size_t bytes);
// Read-only bandwidth probes (kq_read_probe): mode 0 loads, mode 1 bulk-copy ring.
cudaError_t launch_probe(const void* src, size_t bytes, int mode, uint32_t* out, int sm_count, cudaStream_t s);
cudaError_t read_and_clear_fault(int* out);
// Records `msg` as the calling thread's kq_last_error() text; returns status.
int set_last_error(int status, const char* msg);

}  // namespace kq
