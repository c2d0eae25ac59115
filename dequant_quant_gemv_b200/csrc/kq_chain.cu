// kq_chain.cu — layer weights streamed from pinned host memory through a
// ring of device slots, overlapped with the fused GEMV kernels.
//
// "Out-of-core LLM inference engine written from scratch in Rust", Approach:
// layer weights move through a ring of VRAM slots while the GPU computes
// nearby layers; "Kortex: Streaming 70B Models on Consumer GPUs", Key
// components 2 (the streaming pipeline overlaps transfers with compute).
//
// Schedule for layer l in slot s = l % n_slots (everything is enqueued up
// front; the host never blocks per layer):
//   copy stream:    wait slot_free[s] (layer l - n_slots done with slot s),
//                   cudaMemcpyAsync every matrix of layer l into slot s,
//                   record slot_ready[s]
//   compute stream: wait slot_ready[s], launch the layer's GEMVs reading the
//                   slot, record slot_free[s]
// The copy engine therefore runs up to n_slots layers ahead of the SMs, and
// the kernels are exactly the resident kq_gemv kernels, so a streamed run
// gives bitwise the same outputs as a resident run.
#include <cuda_runtime.h>

#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <thread>
#include <vector>

#include "../../include/kq.h"
#include "kq_internal.h"

struct kq_chain {
    std::vector<kq_matrix_desc> mats;   // host-pinned weights, n_layers * per_layer
    int n_layers = 0, per_layer = 0, n_slots = 0;
    size_t slot_bytes = 0;
    std::vector<size_t> offsets;        // byte offset of each matrix within its slot
    uint8_t* ring = nullptr;            // n_slots * slot_bytes device bytes
    cudaStream_t copy = nullptr;
    std::vector<cudaEvent_t> ready, freed;
    cudaEvent_t done = nullptr;
    int device = 0;
    int fault_layer = -1;               // KQ_FAULT=copy@L: fail before copying layer L
};

namespace {

thread_local char g_chain_err[256] = "";

int chain_fail(int status, const char* msg, cudaError_t err = cudaSuccess) {
    if (err != cudaSuccess)
        snprintf(g_chain_err, sizeof(g_chain_err), "%s: %s", msg, cudaGetErrorString(err));
    else
        snprintf(g_chain_err, sizeof(g_chain_err), "%s", msg);
    return status;
}

size_t round_up(size_t v, size_t m) { return (v + m - 1) / m * m; }

void destroy(kq_chain* c) {
    if (!c) return;
    for (auto e : c->ready) cudaEventDestroy(e);
    for (auto e : c->freed) cudaEventDestroy(e);
    if (c->done) cudaEventDestroy(c->done);
    if (c->copy) cudaStreamDestroy(c->copy);
    if (c->ring) cudaFree(c->ring);
    delete c;
}

}  // namespace

extern "C" {

KQ_API const char* kq_chain_last_error(void) { return g_chain_err; }

KQ_API int kq_chain_create(const kq_matrix_desc* mats, int n_layers, int mats_per_layer, int n_slots,
                           kq_chain** out) {
    g_chain_err[0] = 0;
    if (!out) return chain_fail(KQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!mats || n_layers < 1 || mats_per_layer < 1 || n_slots < 1)
        return chain_fail(KQ_ERR_INVALID_ARG, "bad layer / slot counts");
    kq_chain* c = new (std::nothrow) kq_chain();
    if (!c) return chain_fail(KQ_ERR_OOM, "host allocation");
    c->n_layers = n_layers;
    c->per_layer = mats_per_layer;
    c->n_slots = n_slots < n_layers ? n_slots : n_layers;
    c->mats.assign(mats, mats + static_cast<size_t>(n_layers) * mats_per_layer);
    c->offsets.resize(mats_per_layer);
    // slot layout: the matrices of a layer one after another, 256-byte
    // aligned; every layer must have the same matrix shapes
    size_t off = 0;
    for (int m = 0; m < mats_per_layer; ++m) {
        const kq_matrix_desc& d = c->mats[m];
        c->offsets[m] = off;
        off = round_up(off + static_cast<size_t>(d.N) * kq_row_bytes(d.fmt, d.K), 256);
    }
    c->slot_bytes = off;
    for (int l = 0; l < n_layers; ++l)
        for (int m = 0; m < mats_per_layer; ++m) {
            const kq_matrix_desc& d = c->mats[static_cast<size_t>(l) * mats_per_layer + m];
            const kq_matrix_desc& d0 = c->mats[m];
            if (d.fmt != d0.fmt || d.N != d0.N || d.K != d0.K || kq_row_bytes(d.fmt, d.K) == 0 || d.N < 1) {
                destroy(c);
                return chain_fail(KQ_ERR_INVALID_ARG, "layers must share matrix formats and shapes");
            }
            if (!d.W) {
                destroy(c);
                return chain_fail(KQ_ERR_INVALID_ARG, "NULL weight pointer");
            }
            cudaPointerAttributes attr;
            cudaError_t err = cudaPointerGetAttributes(&attr, d.W);
            if (err != cudaSuccess || attr.type != cudaMemoryTypeHost) {
                cudaGetLastError();
                destroy(c);
                return chain_fail(KQ_ERR_NOT_PINNED, "weights must be page-locked host memory (cudaHostAlloc)");
            }
        }
    cudaError_t err = cudaGetDevice(&c->device);
    if (err == cudaSuccess) err = cudaMalloc(&c->ring, c->slot_bytes * c->n_slots);
    if (err != cudaSuccess) {
        cudaGetLastError();
        destroy(c);
        return chain_fail(KQ_ERR_OOM, "device ring allocation", err);
    }
    err = cudaStreamCreateWithFlags(&c->copy, cudaStreamNonBlocking);
    c->ready.resize(c->n_slots, nullptr);
    c->freed.resize(c->n_slots, nullptr);
    for (int s = 0; s < c->n_slots && err == cudaSuccess; ++s) {
        err = cudaEventCreateWithFlags(&c->ready[s], cudaEventDisableTiming);
        if (err == cudaSuccess) err = cudaEventCreateWithFlags(&c->freed[s], cudaEventDisableTiming);
    }
    if (err == cudaSuccess) err = cudaEventCreateWithFlags(&c->done, cudaEventDisableTiming);
    if (err != cudaSuccess) {
        destroy(c);
        return chain_fail(KQ_ERR_CUDA, "stream/event creation", err);
    }
    const char* f = getenv("KQ_FAULT");
    if (f && strncmp(f, "copy@", 5) == 0) c->fault_layer = atoi(f + 5);
    *out = c;
    return KQ_OK;
}

KQ_API size_t kq_chain_slot_bytes(const kq_chain* c) { return c ? c->slot_bytes : 0; }

KQ_API int kq_chain_run(kq_chain* c, const float* const* x, float* const* y, kq_stream_t compute) {
    g_chain_err[0] = 0;
    if (!c || !x || !y) return chain_fail(KQ_ERR_INVALID_ARG, "NULL argument");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(compute);
    // the copy stream starts after whatever the caller queued before this run
    cudaError_t err = cudaEventRecord(c->done, cs);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(c->copy, c->done, 0);
    if (err != cudaSuccess) return chain_fail(KQ_ERR_CUDA, "stream ordering", err);
    for (int l = 0; l < c->n_layers; ++l) {
        const int s = l % c->n_slots;
        uint8_t* slot = c->ring + static_cast<size_t>(s) * c->slot_bytes;
        if (l == c->fault_layer) {
            // injected failure: stop issuing; what is queued drains normally
            // and kq_chain_wait still covers it
            cudaEventRecord(c->done, cs);
            return chain_fail(KQ_ERR_INJECTED, "KQ_FAULT: copy of the requested layer refused");
        }
        if (l >= c->n_slots) {
            err = cudaStreamWaitEvent(c->copy, c->freed[s], 0);
            if (err != cudaSuccess) return chain_fail(KQ_ERR_CUDA, "wait slot free", err);
        }
        for (int m = 0; m < c->per_layer; ++m) {
            const kq_matrix_desc& d = c->mats[static_cast<size_t>(l) * c->per_layer + m];
            err = cudaMemcpyAsync(slot + c->offsets[m], d.W, static_cast<size_t>(d.N) * kq_row_bytes(d.fmt, d.K),
                                  cudaMemcpyHostToDevice, c->copy);
            if (err != cudaSuccess) return chain_fail(KQ_ERR_CUDA, "H2D copy", err);
        }
        err = cudaEventRecord(c->ready[s], c->copy);
        if (err == cudaSuccess) err = cudaStreamWaitEvent(cs, c->ready[s], 0);
        if (err != cudaSuccess) return chain_fail(KQ_ERR_CUDA, "slot ready", err);
        for (int m = 0; m < c->per_layer; ++m) {
            const size_t i = static_cast<size_t>(l) * c->per_layer + m;
            const kq_matrix_desc& d = c->mats[i];
            int st = kq_gemv(slot + c->offsets[m], d.fmt, d.N, d.K, x[i], y[i], compute);
            if (st != KQ_OK) return chain_fail(st, kq_last_error());
        }
        err = cudaEventRecord(c->freed[s], cs);
        if (err != cudaSuccess) return chain_fail(KQ_ERR_CUDA, "slot free", err);
    }
    err = cudaEventRecord(c->done, cs);
    if (err != cudaSuccess) return chain_fail(KQ_ERR_CUDA, "done event", err);
    return KQ_OK;
}

KQ_API int kq_chain_wait(kq_chain* c, int64_t timeout_ms) {
    g_chain_err[0] = 0;
    if (!c) return chain_fail(KQ_ERR_INVALID_ARG, "NULL chain");
    const auto t0 = std::chrono::steady_clock::now();
    while (true) {
        cudaError_t err = cudaEventQuery(c->done);
        if (err == cudaSuccess) break;
        if (err != cudaErrorNotReady) return chain_fail(KQ_ERR_CUDA, "chain completion", err);
        const auto ms =
            std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count();
        if (timeout_ms >= 0 && ms > timeout_ms) return chain_fail(KQ_ERR_TIMEOUT, "chain did not finish in time");
        std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
    // the copy stream must be idle too (a run stopped by an injected fault
    // leaves earlier copies queued)
    cudaError_t err = cudaStreamSynchronize(c->copy);
    if (err != cudaSuccess) return chain_fail(KQ_ERR_CUDA, "copy stream", err);
    return KQ_OK;
}

KQ_API void kq_chain_destroy(kq_chain* c) {
    if (!c) return;
    cudaStreamSynchronize(c->copy);
    destroy(c);
}

}  // extern "C"
