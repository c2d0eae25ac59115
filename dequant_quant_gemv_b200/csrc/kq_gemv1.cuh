// kq_gemv1.cuh — the single-column GEMV of one matrix (kq_gemv, the layer
// chain): gemv_kernel's producer, staging and units with a stage loop that
// carries no more control than this case needs.
//
// Decode multiplies one activation vector by each weight matrix ("Kortex:
// Streaming 70B Models on Consumer GPUs", the paragraph before the first
// table: bound by the weight bytes), so the consumers must turn weight bytes
// into products faster than HBM delivers them.  In the general kernel
// (several columns, routed experts, split K) the per-stage bookkeeping took
// about as many instructions as the dequantisation itself; here a lane's
// stages are an arithmetic sequence (this group's stages s = g, g+2, ... of
// the CTA's row-pair range), the matrix is a single segment, K is whole,
// and the lane layout is fixed for the launch.
//
// DIRECT: a warp holds all units of its row pairs (a butterfly gives the
// row sums and the lead lanes store y).  Otherwise a row pair spans
// `parts` warps: each warp's lead lane writes its partial sums into the
// stage slot's partial buffer and arrives on the row pair's mbarrier; the
// row pair's first warp waits for the others (bounded), adds the parts in
// a fixed order and stores y.  No barrier couples the warps of different
// row pairs.  The slot is released to the producer by every warp after its
// unit, the first warp after the sum, so a partial buffer (one per slot) is
// never rewritten before it has been read.
#pragma once

#include "kq_gemv.cuh"

namespace kq {

// Shared-memory bytes of the partial buffers and their barriers: per slot
// and row pair of a stage, `parts` float pairs and one mbarrier.
__host__ __device__ constexpr int lean_red_bytes(int ps, int parts) {
    return kMaxStages * ps * (8 * parts + 8);
}

// Weight stages copied before the producer waits for the activation
// staging (measured on the 8B-shaped chain: 2 beat 1 and a full ring).
constexpr int kLeadStages = 2;

// FULL: a row pair spans at least a whole warp (lanes_per_rp >= 32), so the
// butterfly runs all five levels unconditionally.  PAR: the block-parity
// lane order (single-column Q6_K).
template <int FMT, bool PRO, bool DIRECT, bool FULL, bool PAR>
__global__ void __launch_bounds__(32 + 2 * kConsumers, 1) gemv1_kernel(const __grid_constant__ GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 2 * kMaxStages * 8);
    volatile int* staged = abort_flag + 1;  // set once the activations are staged
    uint8_t* sbuf = smem + a.sbuf_offset;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ns = a.nstage, ps = a.ps, parts = a.parts;
    // partial buffers: red barriers [slot][rp] then floats [slot][rp][part][2]
    uint64_t* red = reinterpret_cast<uint64_t*>(smem + a.wp_offset);
    const uint32_t pbuf = smem_u32(smem + a.wp_offset) + 8u * kMaxStages * ps;

    if (tid == 0) {
        for (int s = 0; s < ns; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        if (!DIRECT)
            for (int i = 0; i < ns * ps; ++i) mbar_init(&red[i], parts);
        *abort_flag = 0;
        *staged = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int64_t rps = (a.N + 1) / 2;
    const int64_t rp_begin = rps * blockIdx.x / gridDim.x;
    const int64_t rp_end = rps * (blockIdx.x + 1) / gridDim.x;
    constexpr int BS = block_bytes_of<FMT>();
    const int nb = a.nb;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_activations(a, 0, nb);
            produce_stages<BS>(a, full, empty, abort_flag, sbuf, rp_begin, rp_end, rps, ns, 0, nb,
                               static_cast<int>(a.row_bytes), true, staged, kLeadStages);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int ct_all = tid - 32;
    const int g = ct_all >> 8;                 // consumer group: stages s = g, g + 2, ...
    const int ct = ct_all & (kConsumers - 1);
    const int LR = a.lanes_per_rp;
    const LaneUnit L = lane_unit(ct, LR, nb, PAR ? a.par : 0);
    const int part = DIRECT ? 0 : ((ct - L.rp * LR) >> 5);
    const uint32_t xs_s = smem_u32(smem + a.xs_offset);
    const uint32_t xri = xs_s + kXRegionBytes * L.pos;
    const uint32_t pro_r = smem_u32(smem + a.pro_offset);
    const int srow = static_cast<int>(a.row_bytes);
    const uint32_t sbuf_s = smem_u32(sbuf) + 2u * static_cast<uint32_t>(L.rp) * static_cast<uint32_t>(srow);
    const uint32_t stage_bytes = static_cast<uint32_t>(a.stage_bytes);
    const unsigned long long wait_lim = a.wait_ns && blockIdx.x == 0 ? a.wait_ns : kWaitNs;
    const int64_t N = a.N;
    float* const y = a.y;
    pdl_wait();                      // activations may come from the previous grid
    pdl_launch_dependents();
    stage_all<FMT, 1, true, PRO, PAR>(a, 0, xs_s, ct_all, 2 * kConsumers, 3, 0, nb, pro_r);
    float rinv = 1.f;
    if (PRO && a.pro == 1) rinv = ld_s32f(pro_inv_addr(pro_r));
    if (ct_all == 0) *staged = 1;

    const int64_t nrp_all = rp_end - rp_begin;
    const int nst = static_cast<int>((nrp_all + ps - 1) / ps);
    int slot = g;       // stage s = g: slot s % ns (ns >= 2), phase 0
    uint32_t phase = 0;
    bool dead = false;  // a wait of this lane ran out
    const bool lead = DIRECT ? (lane & ((LR < 32 ? LR : 32) - 1)) == 0 : lane == 0;
    // When LR does not divide the group's 256 lanes (LR = 96, 160, 192 or
    // 224), the warps past its ps row pairs hold no unit: they only keep the
    // ring's protocol (wait for each stage, release it) and never touch the
    // stage's bytes or a row pair's partial buffer.
    const bool in_stage = L.rp < ps;
    for (int s = g; s < nst; s += 2) {
        const int64_t rp0 = rp_begin + static_cast<int64_t>(s) * ps;
        const bool mine = in_stage && L.active && rp0 + L.rp < rp_end;
        // with an odd ring depth a slot alternates between the groups: first
        // the other group's release of the slot's previous stage
        if ((ns & 1) && s >= ns && !mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag, wait_lim)) {
            raise_fault(a, abort_flag, 6);
            dead = true;
        }
        if (!mbar_wait_bounded(&full[slot], phase, abort_flag, wait_lim)) {
            raise_fault(a, abort_flag, 6);
            dead = true;
        }
        float out[2][1] = {{0.f}, {0.f}};
        if (mine && !dead) {
            // the stage starts (its first byte's address % 16) into its slot
            const uint32_t row0 = sbuf_s + static_cast<uint32_t>(slot) * stage_bytes +
                                  static_cast<uint32_t>(reinterpret_cast<uintptr_t>(a.W + 2 * rp0 * a.row_bytes) & 15u);
            if constexpr (FMT == 1) q4k_unit_int(row0, srow, L.b, L.H, xri, out);
            else if constexpr (FMT == 3) q5k_unit_int(row0, srow, L.b, L.H, xri, out);
            else if constexpr (FMT == 4) q2k_unit_int(row0, srow, L.b, L.H, xri, out);
            else if constexpr (FMT == 5) q3k_unit_int(row0, srow, L.b, L.H, xri, out);
            else if constexpr (FMT == 6) q80_unit_int(row0, srow, L.b, L.H, xri, out);
            else if constexpr (!PAR) q6k_unit_int<2>(row0, srow, L.b, L.H, xri, out);
            else if (L.b & 1) q6k_unit_int<1>(row0, srow, L.b, L.H, xri, out);
            else q6k_unit_int<0>(row0, srow, L.b, L.H, xri, out);
        }
        // butterfly over the lanes of this row pair (fixed order)
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            if (FULL || off < LR) {
                out[0][0] += __shfl_xor_sync(0xffffffffu, out[0][0], off);
                out[1][0] += __shfl_xor_sync(0xffffffffu, out[1][0], off);
            }
        }
        if constexpr (DIRECT) {
            if (lane == 0) mbar_arrive(&empty[slot]);
            if (lead && in_stage && rp0 + L.rp < rp_end) {
                const int64_t row = 2 * (rp0 + L.rp);
                y[row] = out[0][0] * rinv;
                if (row + 1 < N) y[row + 1] = out[1][0] * rinv;
            }
        } else if (!in_stage) {
            if (lane == 0) mbar_arrive(&empty[slot]);
        } else {
            const int k = slot * ps + L.rp;  // this row pair's partial buffer and barrier
            if (lane == 0) {
                st_s64u(pbuf + 8u * static_cast<uint32_t>(k * parts + part), __float_as_uint(out[0][0]),
                        __float_as_uint(out[1][0]));
                mbar_arrive(&red[k]);  // release: the partials above
                if (part != 0) mbar_arrive(&empty[slot]);
            }
            if (part == 0) {
                if (lane == 0) {
                    if (!mbar_wait_bounded(&red[k], phase, abort_flag, wait_lim)) {
                        raise_fault(a, abort_flag, 6);
                        dead = true;
                    }
                    if (rp0 + L.rp < rp_end) {
                        float v0 = 0.f, v1 = 0.f;
                        for (int p = 0; p < parts; ++p) {
                            const float2 f = ld_s64f(pbuf + 8u * static_cast<uint32_t>(k * parts + p));
                            v0 += f.x;
                            v1 += f.y;
                        }
                        const int64_t row = 2 * (rp0 + L.rp);
                        y[row] = v0 * rinv;
                        if (row + 1 < N) y[row + 1] = v1 * rinv;
                    }
                    mbar_arrive(&empty[slot]);
                }
                __syncwarp();
            }
        }
        slot += 2;
        if (slot >= ns) {
            slot -= ns;
            phase ^= 1u;
        }
    }
}

template <int FMT, bool PRO>
cudaError_t launch_gemv1(const GemvArgs& a, const LaunchPlan& p, cudaStream_t stream) {
    // the layouts that occur: a row pair on part of a warp, on one whole
    // warp, or on several (with the parity order only for Q6_K)
    auto kern = a.lanes_per_rp < 32 ? gemv1_kernel<FMT, PRO, true, false, false>
              : a.parts == 1        ? gemv1_kernel<FMT, PRO, true, true, false>
              : (FMT == 2 && a.par) ? gemv1_kernel<FMT, PRO, false, true, FMT == 2>
                                    : gemv1_kernel<FMT, PRO, false, true, false>;
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void*>(kern), p.smem_bytes);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(32 + 2 * kConsumers);
    cfg.dynamicSmemBytes = p.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = p.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace kq
