// kq_chain.cu — layer weights streamed from pinned host memory through a
// ring of device slots, overlapped with the fused GEMV kernels.
//
// "Out-of-core LLM inference engine written from scratch in Rust", Approach:
// layers are copied into a fixed set of device slots and run while other
// layers compute; "Kortex: Streaming 70B Models on Consumer GPUs", Key
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
//
// Residency ("Kortex: Streaming 70B Models on Consumer GPUs", Key components:
// the layers that fit stay in VRAM, the rest stream): the first n_resident
// layers are copied once, when the chain is created, into device memory of
// their own; a run launches their GEMVs straight away and streams only the
// remaining layers, layer l through slot (l - n_resident) % n_slots.
// kq_chain_plan picks n_resident and n_slots for a device-memory budget.
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
    int n_resident = 0;                 // leading layers kept in `resident`
    uint8_t* resident = nullptr;        // n_resident * slot_bytes device bytes
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

// Bytes of one layer as the chain lays it out (each matrix 256-byte
// aligned), and the matrices' offsets; 0 if a layer's shapes are invalid.
size_t layer_layout(const kq_matrix_desc* mats, int per_layer, std::vector<size_t>* offsets) {
    size_t off = 0;
    for (int m = 0; m < per_layer; ++m) {
        const kq_matrix_desc& d = mats[m];
        const size_t rb = kq_row_bytes(d.fmt, d.K);
        if (rb == 0 || d.N < 1) return 0;
        if (offsets) (*offsets)[m] = off;
        off = round_up(off + static_cast<size_t>(d.N) * rb, 256);
    }
    return off;
}

void destroy(kq_chain* c) {
    if (!c) return;
    for (auto e : c->ready) cudaEventDestroy(e);
    for (auto e : c->freed) cudaEventDestroy(e);
    if (c->done) cudaEventDestroy(c->done);
    if (c->copy) cudaStreamDestroy(c->copy);
    if (c->ring) cudaFree(c->ring);
    if (c->resident) cudaFree(c->resident);
    delete c;
}

}  // namespace

extern "C" {

KQ_API const char* kq_chain_last_error(void) { return g_chain_err; }

KQ_API int kq_chain_plan(const kq_matrix_desc* mats, int n_layers, int mats_per_layer, size_t budget_bytes,
                         int max_slots, int* n_resident, int* n_slots) {
    g_chain_err[0] = 0;
    if (!mats || !n_resident || !n_slots || n_layers < 1 || mats_per_layer < 1 || max_slots < 1)
        return chain_fail(KQ_ERR_INVALID_ARG, "bad arguments");
    const size_t lb = layer_layout(mats, mats_per_layer, nullptr);
    if (lb == 0) return chain_fail(KQ_ERR_INVALID_ARG, "bad matrix shape or format");
    if (static_cast<size_t>(n_layers) * lb <= budget_bytes) {  // everything stays resident
        *n_resident = n_layers;
        *n_slots = 0;
        return KQ_OK;
    }
    if (budget_bytes < lb) return chain_fail(KQ_ERR_OOM, "the budget does not hold one layer");
    size_t slots = static_cast<size_t>(max_slots < n_layers ? max_slots : n_layers);
    while (slots > 1 && slots * lb > budget_bytes) --slots;
    size_t res = (budget_bytes - slots * lb) / lb;
    if (res > static_cast<size_t>(n_layers) - slots) res = static_cast<size_t>(n_layers) - slots;
    *n_resident = static_cast<int>(res);
    *n_slots = static_cast<int>(slots);
    return KQ_OK;
}

KQ_API int kq_chain_create_resident(const kq_matrix_desc* mats, int n_layers, int mats_per_layer, int n_resident,
                                    int n_slots, kq_chain** out) {
    g_chain_err[0] = 0;
    if (!out) return chain_fail(KQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!mats || n_layers < 1 || mats_per_layer < 1 || n_resident < 0 || n_resident > n_layers || n_slots < 0 ||
        (n_resident < n_layers && n_slots < 1))
        return chain_fail(KQ_ERR_INVALID_ARG, "bad layer / resident / slot counts");
    kq_chain* c = new (std::nothrow) kq_chain();
    if (!c) return chain_fail(KQ_ERR_OOM, "host allocation");
    c->n_layers = n_layers;
    c->per_layer = mats_per_layer;
    c->n_resident = n_resident;
    const int streamed = n_layers - n_resident;
    c->n_slots = streamed == 0 ? 0 : (n_slots < streamed ? n_slots : streamed);
    c->mats.assign(mats, mats + static_cast<size_t>(n_layers) * mats_per_layer);
    c->offsets.resize(mats_per_layer);
    // slot layout: the matrices of a layer one after another, 256-byte
    // aligned; every layer must have the same matrix shapes
    c->slot_bytes = layer_layout(c->mats.data(), mats_per_layer, &c->offsets);
    if (c->slot_bytes == 0) {
        destroy(c);
        return chain_fail(KQ_ERR_INVALID_ARG, "layers must share matrix formats and shapes");
    }
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
    if (err == cudaSuccess && c->n_slots > 0) err = cudaMalloc(&c->ring, c->slot_bytes * c->n_slots);
    if (err == cudaSuccess && n_resident > 0) err = cudaMalloc(&c->resident, c->slot_bytes * n_resident);
    if (err != cudaSuccess) {
        cudaGetLastError();
        destroy(c);
        return chain_fail(KQ_ERR_OOM, "device slot / resident allocation", err);
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
    // the resident layers, copied once
    for (int l = 0; l < n_resident && err == cudaSuccess; ++l)
        for (int m = 0; m < mats_per_layer && err == cudaSuccess; ++m) {
            const kq_matrix_desc& d = c->mats[static_cast<size_t>(l) * mats_per_layer + m];
            err = cudaMemcpyAsync(c->resident + static_cast<size_t>(l) * c->slot_bytes + c->offsets[m], d.W,
                                  static_cast<size_t>(d.N) * kq_row_bytes(d.fmt, d.K), cudaMemcpyHostToDevice,
                                  c->copy);
        }
    if (err == cudaSuccess) err = cudaStreamSynchronize(c->copy);
    if (err != cudaSuccess) {
        destroy(c);
        return chain_fail(KQ_ERR_CUDA, "resident layer copy", err);
    }
    const char* f = getenv("KQ_FAULT");
    if (f && strncmp(f, "copy@", 5) == 0) c->fault_layer = atoi(f + 5);
    *out = c;
    return KQ_OK;
}

KQ_API int kq_chain_create(const kq_matrix_desc* mats, int n_layers, int mats_per_layer, int n_slots,
                           kq_chain** out) {
    if (n_slots < 1) {
        g_chain_err[0] = 0;
        if (out) *out = nullptr;
        return chain_fail(KQ_ERR_INVALID_ARG, "bad layer / slot counts");
    }
    return kq_chain_create_resident(mats, n_layers, mats_per_layer, 0, n_slots, out);
}

KQ_API int kq_chain_resident_layers(const kq_chain* c) { return c ? c->n_resident : 0; }

KQ_API size_t kq_chain_slot_bytes(const kq_chain* c) { return c ? c->slot_bytes : 0; }

KQ_API int kq_chain_run(kq_chain* c, const float* const* x, float* const* y, kq_stream_t compute) {
    g_chain_err[0] = 0;
    if (!c || !x || !y) return chain_fail(KQ_ERR_INVALID_ARG, "NULL argument");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(compute);
    // the copy stream starts after whatever the caller queued before this run
    cudaError_t err = cudaEventRecord(c->done, cs);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(c->copy, c->done, 0);
    if (err != cudaSuccess) return chain_fail(KQ_ERR_CUDA, "stream ordering", err);
    // A run that stops part-way re-records `done` on the compute stream
    // first, so that kq_chain_wait covers every GEMV already queued.
    auto stop = [&](int status, const char* what, cudaError_t e) {
        cudaEventRecord(c->done, cs);
        return chain_fail(status, what, e);
    };
    for (int l = 0; l < c->n_layers; ++l) {
        if (l < c->n_resident) {  // a resident layer: its GEMVs only
            const uint8_t* base = c->resident + static_cast<size_t>(l) * c->slot_bytes;
            for (int m = 0; m < c->per_layer; ++m) {
                const size_t i = static_cast<size_t>(l) * c->per_layer + m;
                const kq_matrix_desc& d = c->mats[i];
                int st = kq_gemv(base + c->offsets[m], d.fmt, d.N, d.K, x[i], y[i], compute);
                if (st != KQ_OK) return stop(st, kq_last_error(), cudaSuccess);
            }
            continue;
        }
        const int j = l - c->n_resident;  // streamed layer number
        const int s = j % c->n_slots;
        uint8_t* slot = c->ring + static_cast<size_t>(s) * c->slot_bytes;
        if (l == c->fault_layer) {
            // injected failure: stop issuing; what is queued drains normally
            // and kq_chain_wait still covers it
            return stop(KQ_ERR_INJECTED, "KQ_FAULT: copy of the requested layer refused", cudaSuccess);
        }
        if (j >= c->n_slots) {
            err = cudaStreamWaitEvent(c->copy, c->freed[s], 0);
            if (err != cudaSuccess) return stop(KQ_ERR_CUDA, "wait slot free", err);
        }
        for (int m = 0; m < c->per_layer; ++m) {
            const kq_matrix_desc& d = c->mats[static_cast<size_t>(l) * c->per_layer + m];
            err = cudaMemcpyAsync(slot + c->offsets[m], d.W, static_cast<size_t>(d.N) * kq_row_bytes(d.fmt, d.K),
                                  cudaMemcpyHostToDevice, c->copy);
            if (err != cudaSuccess) return stop(KQ_ERR_CUDA, "H2D copy", err);
        }
        err = cudaEventRecord(c->ready[s], c->copy);
        if (err == cudaSuccess) err = cudaStreamWaitEvent(cs, c->ready[s], 0);
        if (err != cudaSuccess) return stop(KQ_ERR_CUDA, "slot ready", err);
        for (int m = 0; m < c->per_layer; ++m) {
            const size_t i = static_cast<size_t>(l) * c->per_layer + m;
            const kq_matrix_desc& d = c->mats[i];
            int st = kq_gemv(slot + c->offsets[m], d.fmt, d.N, d.K, x[i], y[i], compute);
            if (st != KQ_OK) return stop(st, kq_last_error(), cudaSuccess);
        }
        err = cudaEventRecord(c->freed[s], cs);
        if (err != cudaSuccess) return stop(KQ_ERR_CUDA, "slot free", err);
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

KQ_API int kq_stream_chain_create(const kq_layer_desc* layers, int n_layers, int n_slots, kq_chain** out) {
    g_chain_err[0] = 0;
    if (out) *out = nullptr;
    if (!layers || !out || n_layers < 1 || n_slots < 1) return chain_fail(KQ_ERR_INVALID_ARG, "bad arguments");
    const int per = layers[0].n_mats;
    if (per < 1) return chain_fail(KQ_ERR_INVALID_ARG, "a layer without matrices");
    std::vector<kq_matrix_desc> flat;
    flat.reserve(static_cast<size_t>(n_layers) * per);
    for (int l = 0; l < n_layers; ++l) {
        if (layers[l].n_mats != per || !layers[l].mats)
            return chain_fail(KQ_ERR_INVALID_ARG, "layers must share matrix formats and shapes");
        for (int m = 0; m < per; ++m) flat.push_back(layers[l].mats[m]);
    }
    return kq_chain_create(flat.data(), n_layers, per, n_slots, out);
}

KQ_API int kq_stream_chain(kq_chain* c, const float* const* x_in, float* const* y_out, kq_stream_t compute,
                           int64_t timeout_ms) {
    const int st = kq_chain_run(c, x_in, y_out, compute);
    if (st != KQ_OK) {
        // what was queued still completes; wait for it (bounded) so that the
        // caller gets the run's own error, not a busy chain
        if (c) kq_chain_wait(c, timeout_ms);
        return st;
    }
    return kq_chain_wait(c, timeout_ms);
}

KQ_API void kq_stream_chain_destroy(kq_chain* c) { kq_chain_destroy(c); }

}  // extern "C"
