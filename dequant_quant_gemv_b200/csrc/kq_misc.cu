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
// helpers the GEMV kernels use.  Each format branch fills the block's quants
// (written at once) and its 16 scale and 16 min bytes, d and dmin; `split`
// selects the output form: the separate arrays of kq_unpack (sc_or_s, m,
// d, dmin, one entry or 16 bytes per block) or the packed form of
// kq_unpack_fields (sc: 16 bytes per block, d: d and dmin per block).
__global__ void unpack_kernel(const uint8_t* W, int fmt, int64_t nblocks, uint8_t* q, uint8_t* sc, uint8_t* m,
                              float* d, float* dmin, bool split) {
    const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (b >= nblocks) return;
    uint8_t S[16], M[16];
    for (int g = 0; g < 16; ++g) S[g] = M[g] = 0;
    float dv = 0.0f, dmv = 0.0f;
    if (fmt == 1 || fmt == 3) {
        // Q4_K, Q5_K: the same header; Q5_K quants sit after its 32 qh bytes
        const uint8_t* blk = W + b * (fmt == 1 ? kQ4Bytes : kQ5Bytes);
        const uint8_t* qs = blk + (fmt == 1 ? 16 : 48);
        const uint4 hd = *reinterpret_cast<const uint4*>(blk);
        for (int H = 0; H < 2; ++H) {
            uint32_t sc4, m4;
            q4k_half_scales(hd.y, hd.z, hd.w, H, sc4, m4);
            for (int k = 0; k < 4; ++k) {
                S[4 * H + k] = static_cast<uint8_t>(sc4 >> (8 * k));
                M[4 * H + k] = static_cast<uint8_t>(m4 >> (8 * k));
            }
        }
        dv = __half2float(__ushort_as_half(static_cast<unsigned short>(hd.x & 0xFFFFu)));
        dmv = __half2float(__ushort_as_half(static_cast<unsigned short>(hd.x >> 16)));
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
        for (int g = 0; g < 16; ++g) {
            S[g] = blk[g] & 15u;
            M[g] = blk[g] >> 4;
        }
        for (int i = 0; i < 64; ++i) {
            const uint32_t v = blk[16 + i];
            const int n = i >> 5, l = i & 31;
            for (int j = 0; j < 4; ++j) q[256 * b + 128 * n + 32 * j + l] = static_cast<uint8_t>((v >> (2 * j)) & 3u);
        }
        const uint32_t dw = *reinterpret_cast<const uint32_t*>(blk + 80);
        dv = __half2float(__ushort_as_half(static_cast<unsigned short>(dw & 0xFFFFu)));
        dmv = __half2float(__ushort_as_half(static_cast<unsigned short>(dw >> 16)));
    } else if (fmt == 6) {
        // Q8_0: a unit of eight 34-byte blocks, read by bytes; S holds the
        // eight fp16 scales as raw little-endian bytes
        const uint8_t* u = W + b * kQ80Bytes;
        for (int j = 0; j < 8; ++j) {
            S[2 * j] = u[34 * j];
            S[2 * j + 1] = u[34 * j + 1];
            for (int i = 0; i < 32; ++i) q[256 * b + 32 * j + i] = u[34 * j + 2 + i];
        }
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
            S[g] = static_cast<uint8_t>(lo | (hi << 4));
        }
        const unsigned short dh = static_cast<unsigned short>(blk[108] | (blk[109] << 8));
        dv = __half2float(__ushort_as_half(dh));
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
        for (int g = 0; g < 16; ++g) S[g] = blk[192 + g];
        const unsigned short dh = static_cast<unsigned short>(blk[208] | (blk[209] << 8));
        dv = __half2float(__ushort_as_half(dh));
    }
    if (split) {
        for (int g = 0; g < 16; ++g) sc[16 * b + g] = S[g];
        if (m)
            for (int g = 0; g < 16; ++g) m[16 * b + g] = M[g];
        d[b] = dv;
        if (dmin) dmin[b] = dmv;
    } else {
        // Q4_K, Q5_K: sc_0..7 then m_0..7; Q2_K: the stored bytes sc | m << 4
        const bool eight = fmt == 1 || fmt == 3;
        for (int g = 0; g < 16; ++g)
            sc[16 * b + g] = eight ? (g < 8 ? S[g] : M[g - 8]) : (fmt == 4 ? static_cast<uint8_t>(S[g] | (M[g] << 4)) : S[g]);
        d[2 * b] = dv;
        d[2 * b + 1] = dmv;
    }
}

cudaError_t launch_unpack(const uint8_t* W, int fmt, int64_t nblocks, uint8_t* q, uint8_t* sc, uint8_t* m, float* d,
                          float* dmin, bool split, cudaStream_t stream) {
    const int threads = 128;
    const int64_t grid = (nblocks + threads - 1) / threads;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    unpack_kernel<<<static_cast<unsigned>(grid), threads, 0, stream>>>(W, fmt, nblocks, q, sc, m, d, dmin, split);
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
