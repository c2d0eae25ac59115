// kq_noalloc.cu — kq_gemv_splitk_noalloc: the split-K GEMV for callers that
// cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is off limits or unwanted --
// a real-time or callback thread that must not take the allocator's locks or
// its implicit device synchronisation, an engine whose every byte of device
// memory belongs to its own arena and must not be taken behind its back, or a
// plugin handed only its inputs and outputs by a host that owns allocation.
// Such callers cannot provide the split-K workspace that kq_gemv_splitk asks
// for, so this entry point keeps its partial sums in a fixed array compiled
// into the library instead.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/kq.h"
#include "kq_internal.h"

namespace {

// The partial sums of every kq_gemv_splitk_noalloc call, 64 KiB per GPU.
// Every GPU that loads the library holds this array until the process
// exits.  A split of S K-ranges over N outputs and k columns needs
// S * k * N floats; on a 148-SM B200 the split planner never asks for more
// than about 14 KiB.
constexpr size_t kScratchFloats = 16384;
static __device__ __align__(256) float kq_noalloc_scratch[kScratchFloats];

// Device address of the array, looked up once per device.  (In host code
// the name kq_noalloc_scratch is only a host-side stand-in for the symbol.)
std::mutex g_mu;
float* g_scratch[64] = {};

}  // namespace

extern "C" {

KQ_API int kq_gemv_splitk_noalloc(const void* W, int fmt, int64_t N, int64_t K, const float* x, int64_t ldx,
                                  int k, float* y, int64_t ldy, kq_stream_t stream) {
    char msg[256];
    const size_t need = kq_splitk_workspace_bytes(fmt, N, K, k);
    if (need > sizeof(float) * kScratchFloats) {
        snprintf(msg, sizeof(msg),
                 "split needs %zu bytes of scratch; the built-in scratch holds %zu bytes "
                 "(use kq_gemv_splitk with a workspace)",
                 need, sizeof(float) * kScratchFloats);
        return kq::set_last_error(KQ_ERR_UNSUPPORTED, msg);
    }
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess || dev < 0 || dev >= 64) {
        snprintf(msg, sizeof(msg), "current device: %s", cudaGetErrorString(err));
        return kq::set_last_error(KQ_ERR_CUDA, msg);
    }
    float* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_scratch[dev]) {
            // set-up on this device's first call, with this device current
            void* p = nullptr;
            err = cudaGetSymbolAddress(&p, kq_noalloc_scratch);
            if (err != cudaSuccess) {
                snprintf(msg, sizeof(msg), "cudaGetSymbolAddress: %s", cudaGetErrorString(err));
                return kq::set_last_error(KQ_ERR_CUDA, msg);
            }
            g_scratch[dev] = static_cast<float*>(p);
        }
        scratch = g_scratch[dev];
    }
    // Every partial sum the combine step reads is written earlier in the
    // same call, so the scratch needs no clearing between calls.
    return kq_gemv_splitk(W, fmt, N, K, x, ldx, k, y, ldy, scratch, sizeof(float) * kScratchFloats, stream);
}

}  // extern "C"
