// kq_misc.cu — the debug unpack kernel and the device fault word.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {

// Set by a kernel whose bounded wait ran out (launches without a caller
// status pointer); read and cleared by kq_device_fault().
__device__ int g_kq_fault = 0;

// ------------------------------------------------------- debug unpack

// One thread per super-block: the integer fields, decoded with the same
// helpers the GEMV kernels use.
__global__ void unpack_kernel(const uint8_t* W, int fmt, int64_t nblocks, uint8_t* q, uint8_t* sc, float* d) {
    const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (b >= nblocks) return;
    if (fmt == 1 || fmt == 3) {
        // Q4_K, Q5_K: the same header; Q5_K quants sit after its 32 qh bytes
        const uint8_t* blk = W + b * (fmt == 1 ? kQ4Bytes : kQ5Bytes);
        const uint8_t* qs = blk + (fmt == 1 ? 16 : 48);
        const uint4 hd = *reinterpret_cast<const uint4*>(blk);
        for (int H = 0; H < 2; ++H) {
            uint32_t sc4, m4;
            q4k_half_scales(hd.y, hd.z, hd.w, H, sc4, m4);
            for (int k = 0; k < 4; ++k) {
                sc[16 * b + 4 * H + k] = static_cast<uint8_t>(sc4 >> (8 * k));
                sc[16 * b + 8 + 4 * H + k] = static_cast<uint8_t>(m4 >> (8 * k));
            }
        }
        d[2 * b] = __half2float(__ushort_as_half(static_cast<unsigned short>(hd.x & 0xFFFFu)));
        d[2 * b + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(hd.x >> 16)));
        for (int w = 0; w < 32; ++w) {
            const uint32_t v = *reinterpret_cast<const uint32_t*>(qs + 4 * w);
            const int c = w >> 3, l0 = (w & 7) * 4;
            // Q5_K: 5th bits of chunk c at bits 2c, 2c+1 of qh[l]
            const uint32_t e = fmt == 3 ? *reinterpret_cast<const uint32_t*>(blk + 16 + l0) : 0u;
            for (int k = 0; k < 4; ++k) {
                const uint32_t eb = e >> (8 * k);
                q[256 * b + 64 * c + l0 + k] =
                    static_cast<uint8_t>(((v >> (8 * k)) & 15u) | (((eb >> (2 * c)) & 1u) << 4));
                q[256 * b + 64 * c + 32 + l0 + k] =
                    static_cast<uint8_t>(((v >> (8 * k + 4)) & 15u) | (((eb >> (2 * c + 1)) & 1u) << 4));
            }
        }
    } else if (fmt == 4) {
        // Q2_K: 4-byte aligned blocks
        const uint8_t* blk = W + b * kQ2Bytes;
        for (int g = 0; g < 16; ++g) sc[16 * b + g] = blk[g];
        for (int i = 0; i < 64; ++i) {
            const uint32_t v = blk[16 + i];
            const int n = i >> 5, l = i & 31;
            for (int j = 0; j < 4; ++j) q[256 * b + 128 * n + 32 * j + l] = static_cast<uint8_t>((v >> (2 * j)) & 3u);
        }
        const uint32_t dw = *reinterpret_cast<const uint32_t*>(blk + 80);
        d[2 * b] = __half2float(__ushort_as_half(static_cast<unsigned short>(dw & 0xFFFFu)));
        d[2 * b + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(dw >> 16)));
    } else if (fmt == 6) {
        // Q8_0: a unit of eight 34-byte blocks, read by bytes
        const uint8_t* u = W + b * kQ80Bytes;
        for (int j = 0; j < 8; ++j) {
            sc[16 * b + 2 * j] = u[34 * j];
            sc[16 * b + 2 * j + 1] = u[34 * j + 1];
            for (int i = 0; i < 32; ++i) q[256 * b + 32 * j + i] = u[34 * j + 2 + i];
        }
        d[2 * b] = 0.0f;
        d[2 * b + 1] = 0.0f;
    } else if (fmt == 5) {
        // Q3_K: 2-byte aligned blocks, read by bytes
        const uint8_t* blk = W + b * kQ3Bytes;
        for (int i = 0; i < 64; ++i) {
            const uint32_t v = blk[32 + i];
            const int n = i >> 5, l = i & 31;
            for (int j = 0; j < 4; ++j) {
                const uint32_t third = (blk[l] >> (4 * n + j)) & 1u;
                q[256 * b + 128 * n + 32 * j + l] = static_cast<uint8_t>(((v >> (2 * j)) & 3u) + 4 * third - 4);
            }
        }
        for (int g = 0; g < 16; ++g) {
            const uint32_t lo = g < 8 ? (blk[96 + g] & 15u) : (blk[96 + g - 8] >> 4);
            const uint32_t hi = (blk[104 + (g & 3)] >> (2 * (g >> 2))) & 3u;
            sc[16 * b + g] = static_cast<uint8_t>(lo | (hi << 4));
        }
        const unsigned short dh = static_cast<unsigned short>(blk[108] | (blk[109] << 8));
        d[2 * b] = __half2float(__ushort_as_half(dh));
        d[2 * b + 1] = 0.0f;
    } else {
        const uint8_t* blk = W + b * kQ6Bytes;  // 2-byte aligned only
        auto word = [&](int off) -> uint32_t {
            return static_cast<uint32_t>(blk[off]) | (static_cast<uint32_t>(blk[off + 1]) << 8) |
                   (static_cast<uint32_t>(blk[off + 2]) << 16) | (static_cast<uint32_t>(blk[off + 3]) << 24);
        };
        for (int H = 0; H < 2; ++H)
            for (int s = 0; s < 8; ++s) {
                uint32_t qv[4];
                q6k_build(word(64 * H + 4 * s), word(64 * H + 32 + 4 * s), word(128 + 32 * H + 4 * s), qv[0], qv[1],
                          qv[2], qv[3]);
                for (int t = 0; t < 4; ++t)
                    for (int k = 0; k < 4; ++k)
                        q[256 * b + 128 * H + 32 * t + 4 * s + k] = static_cast<uint8_t>(qv[t] >> (8 * k));
            }
        for (int g = 0; g < 16; ++g) sc[16 * b + g] = blk[192 + g];
        const unsigned short dh = static_cast<unsigned short>(blk[208] | (blk[209] << 8));
        d[2 * b] = __half2float(__ushort_as_half(dh));
        d[2 * b + 1] = 0.0f;
    }
}

cudaError_t launch_unpack(const uint8_t* W, int fmt, int64_t nblocks, uint8_t* q, uint8_t* sc, float* d,
                          cudaStream_t stream) {
    const int threads = 128;
    const int64_t grid = (nblocks + threads - 1) / threads;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    unpack_kernel<<<static_cast<unsigned>(grid), threads, 0, stream>>>(W, fmt, nblocks, q, sc, d);
    return cudaGetLastError();
}

// Split-K combine: y[j][r] = sum over K ranges s = 0..S-1 (in that order)
// of partial[s][j][r].  Launched after gemv_kernel on the same stream.
__global__ void splitk_combine_kernel(const float* __restrict__ partial, int S, int ncol, int64_t N, float* y,
                                      int64_t ldy) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= ncol * N) return;
    const int64_t j = t / N, r = t - j * N;
    float v = 0.f;
    for (int s = 0; s < S; ++s) v += partial[(static_cast<int64_t>(s) * ncol + j) * N + r];
    y[j * ldy + r] = v;
}

cudaError_t launch_splitk_combine(const float* partial, int S, int ncol, int64_t N, float* y, int64_t ldy,
                                  cudaStream_t stream) {
    const int64_t n = static_cast<int64_t>(ncol) * N;
    const int threads = 256;
    const int64_t grid = (n + threads - 1) / threads;
    splitk_combine_kernel<<<static_cast<unsigned>(grid), threads, 0, stream>>>(partial, S, ncol, N, y, ldy);
    return cudaGetLastError();
}

// Counter pairs of multi-step launches: pair i = (step completions, CTAs
// finished).  Every pair is zero between launches: the last CTA of a launch
// to finish resets its pair.  Launches take pairs round-robin, so two
// launches share a pair only kSyncPairs launches apart.
__device__ int g_kq_steps_sync[2 * kSyncPairs] = {};

cudaError_t steps_sync_pair(int** out) {
    static int* base[64] = {};
    static std::atomic<unsigned> next[64];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!base[dev]) {
        int* b = nullptr;
        err = cudaGetSymbolAddress(reinterpret_cast<void**>(&b), g_kq_steps_sync);
        if (err != cudaSuccess) return err;
        base[dev] = b;
    }
    *out = base[dev] + 2 * (next[dev].fetch_add(1u, std::memory_order_relaxed) % kSyncPairs);
    return cudaSuccess;
}

// The fault word's device address, looked up once per device.
cudaError_t fault_word(int** out) {
    static int* cache[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64 && cache[dev]) {
        *out = cache[dev];
        return cudaSuccess;
    }
    err = cudaGetSymbolAddress(reinterpret_cast<void**>(out), g_kq_fault);
    if (err == cudaSuccess && dev >= 0 && dev < 64) cache[dev] = *out;
    return err;
}

cudaError_t read_and_clear_fault(int* out) {
    int zero = 0;
    cudaError_t err = cudaMemcpyFromSymbol(out, g_kq_fault, sizeof(int));
    if (err != cudaSuccess) return err;
    return cudaMemcpyToSymbol(g_kq_fault, &zero, sizeof(int));
}

}  // namespace kq
