// kq_probe.cu — read-only bandwidth probes: the HBM read roofline that the
// weight stream of the GEMV kernels is measured against.
//
// Decode is bound by weight bytes ("Kortex: Streaming 70B Models on Consumer
// GPUs", the paragraph before the first table), and a GEMV only READS its
// weights, so the ceiling for it is the device's read bandwidth, not the
// copy (read + write) rate.  Two probes read a buffer once:
//  mode 0: every thread streams 16-byte loads (L1 bypassed) over the buffer;
//  mode 1: the GEMV kernels' own weight path -- one persistent CTA per SM
//          whose producer thread bulk-copies (TMA, no multicast) stages of a
//          contiguous range into a shared-memory ring, and a consumer warp
//          that reads each stage from shared memory and releases it: the
//          rate this design streams at when the dequantisation costs
//          nothing.
// Both XOR what they read into *out so that no load can be dropped.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/kq.h"
#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {

__device__ __forceinline__ uint4 ld_nc_v4(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__global__ void __launch_bounds__(512) probe_loads_kernel(const uint4* __restrict__ src, int64_t n16, uint32_t* out) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    uint32_t acc = 0;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = ld_nc_v4(src + i), b = ld_nc_v4(src + i + stride);
        const uint4 c = ld_nc_v4(src + i + 2 * stride), d = ld_nc_v4(src + i + 3 * stride);
        acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
    }
    for (; i < n16; i += stride) {
        const uint4 a = ld_nc_v4(src + i);
        acc ^= a.x ^ a.y ^ a.z ^ a.w;
    }
    for (int off = 16; off >= 1; off >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, off);
    if ((threadIdx.x & 31) == 0 && acc) atomicXor(out, acc);
}

constexpr int kProbeSlots = 4;
constexpr uint32_t kProbeStage = 48 * 1024;

__global__ void __launch_bounds__(64, 1) probe_ring_kernel(const uint8_t* __restrict__ src, int64_t bytes,
                                                            uint32_t* out, int* fault) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kProbeSlots;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 2 * kProbeSlots * 8);
    uint8_t* ring = smem + 128;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kProbeSlots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // this CTA's contiguous range, in 16-byte units
    const int64_t units = bytes / 16;
    const int64_t u0 = units * blockIdx.x / gridDim.x, u1 = units * (blockIdx.x + 1) / gridDim.x;
    const int64_t b0 = 16 * u0, b1 = 16 * u1;
    const int64_t nst = (b1 - b0 + kProbeStage - 1) / kProbeStage;
    if (threadIdx.x == 0) {  // producer
        const uint64_t pol = l2_evict_first();
        RingTrack track;
        for (int64_t i = 0; i < nst; ++i) {
            const int slot = static_cast<int>(i % kProbeSlots);
            const uint32_t ph = static_cast<uint32_t>((i / kProbeSlots) & 1);
            if (i >= kProbeSlots && !mbar_wait_bounded(&empty[slot], ph ^ 1u, abort_flag)) {
                *abort_flag = 1;
                atomicExch(fault, KQ_ERR_TIMEOUT);
                break;
            }
            if (*abort_flag) break;
            const int64_t o = b0 + i * kProbeStage;
            const uint32_t n = static_cast<uint32_t>(b1 - o < kProbeStage ? b1 - o : kProbeStage);
            mbar_arrive_expect_tx(&full[slot], n);
            bulk_g2s(ring + static_cast<size_t>(slot) * kProbeStage, src + o, n, &full[slot], pol);
            track.issue(slot, ph);
        }
        track.drain(full, kProbeSlots);
    } else if (threadIdx.x >= 32) {  // consumer warp: read each stage from shared memory, release it
        const int lane = threadIdx.x - 32;
        uint32_t acc = 0;
        for (int64_t i = 0; i < nst; ++i) {
            const int slot = static_cast<int>(i % kProbeSlots);
            const uint32_t ph = static_cast<uint32_t>((i / kProbeSlots) & 1);
            // every lane waits (and so sees the copy's data); the warp leaves
            // the loop as one if any lane gave up
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full[slot], ph, abort_flag));
            if (!ok) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicExch(fault, KQ_ERR_TIMEOUT);
                }
                break;
            }
            const int64_t o = b0 + i * kProbeStage;
            const int n16 = static_cast<int>((b1 - o < kProbeStage ? b1 - o : kProbeStage) / 16);
            const uint4* st = reinterpret_cast<const uint4*>(ring + static_cast<size_t>(slot) * kProbeStage);
            for (int j = lane; j < n16; j += 32) {
                const uint4 v = st[j];
                acc ^= v.x ^ v.y ^ v.z ^ v.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        for (int off = 16; off >= 1; off >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0 && acc) atomicXor(out, acc);
    }
}

cudaError_t launch_probe(const void* src, size_t bytes, int mode, uint32_t* out, int sm_count, cudaStream_t s) {
    if (mode == 0) {
        probe_loads_kernel<<<sm_count * 4, 512, 0, s>>>(static_cast<const uint4*>(src),
                                                        static_cast<int64_t>(bytes / 16), out);
        return cudaGetLastError();
    }
    int* fault = nullptr;
    cudaError_t err = fault_word(&fault);
    if (err != cudaSuccess) return err;
    const size_t smem = 128 + static_cast<size_t>(kProbeSlots) * kProbeStage;
    err = ensure_smem_attr(reinterpret_cast<const void*>(probe_ring_kernel), smem);
    if (err != cudaSuccess) return err;
    probe_ring_kernel<<<sm_count, 64, smem, s>>>(static_cast<const uint8_t*>(src), static_cast<int64_t>(bytes), out,
                                                 fault);
    return cudaGetLastError();
}

}  // namespace kq
