// kq_moe_stream.cu — routed experts streamed from pinned host memory.
//
// "RunNburn - Run a 295B MoE from a 98GB GGUF on a 64GB RAM Desktop": only
// the experts a token selects are fetched, on demand; "Out-of-core LLM
// inference engine written from scratch in Rust", Approach: weight copies
// into device slots overlap the computation.
//
// Schedule of run r in slot set t = r % n_sets (everything enqueued up
// front; the host never blocks):
//   copy stream:    wait set_free[t] (run r - n_sets done reading set t),
//                   one cudaMemcpyAsync per routed expert into slot i of the
//                   set, record set_ready[t]
//   compute stream: wait set_ready[t], kq_moe_gemv over the set with ids
//                   0..n_ids-1 (slot i holds the expert of routed id i),
//                   record set_free[t]
// The kernel is the resident routed GEMV, reading the slot set as an expert
// stack, so the outputs equal those of device-resident experts bitwise.
#include <cuda_runtime.h>

#include <chrono>
#include <cstdio>
#include <new>
#include <thread>
#include <vector>

#include "../../include/kq.h"

struct kq_moe_stream {
    const uint8_t* host = nullptr;  // page-locked expert stack
    int fmt = 0, E = 0, max_ids = 0, n_sets = 0;
    int64_t N = 0, K = 0;
    size_t stride = 0;              // host bytes between experts
    size_t expert_bytes = 0;        // N * row_bytes
    size_t slot_bytes = 0;          // expert_bytes rounded up to 256
    uint8_t* slots = nullptr;       // n_sets * max_ids * slot_bytes device bytes
    int32_t* iota = nullptr;        // device ids 0..max_ids-1
    cudaStream_t copy = nullptr;
    std::vector<cudaEvent_t> ready, freed;
    cudaEvent_t done = nullptr;
    long long runs = 0;
};

namespace {

thread_local char g_moe_err[256] = "";

int moe_fail(int status, const char* msg, cudaError_t err = cudaSuccess) {
    if (err != cudaSuccess)
        snprintf(g_moe_err, sizeof(g_moe_err), "%s: %s", msg, cudaGetErrorString(err));
    else
        snprintf(g_moe_err, sizeof(g_moe_err), "%s", msg);
    return status;
}

void destroy(kq_moe_stream* m) {
    if (!m) return;
    for (auto e : m->ready) cudaEventDestroy(e);
    for (auto e : m->freed) cudaEventDestroy(e);
    if (m->done) cudaEventDestroy(m->done);
    if (m->copy) cudaStreamDestroy(m->copy);
    if (m->slots) cudaFree(m->slots);
    if (m->iota) cudaFree(m->iota);
    delete m;
}

}  // namespace

extern "C" {

KQ_API const char* kq_moe_stream_last_error(void) { return g_moe_err; }

KQ_API int kq_moe_stream_create(const void* W_host, int fmt, int E, int64_t N, int64_t K,
                                size_t expert_stride_bytes, int max_ids, int n_sets, kq_moe_stream** out) {
    g_moe_err[0] = 0;
    if (!out) return moe_fail(KQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    const size_t rb = kq_row_bytes(fmt, K);
    if (!W_host || E < 1 || N < 1 || K < 256 || rb == 0 || max_ids < 1 || n_sets < 1)
        return moe_fail(KQ_ERR_INVALID_ARG, "bad format, shape, id or set count");
    const size_t eb = static_cast<size_t>(N) * rb;
    if (expert_stride_bytes < eb) return moe_fail(KQ_ERR_INVALID_ARG, "expert stride < N * row_bytes");
    cudaPointerAttributes attr;
    cudaError_t err = cudaPointerGetAttributes(&attr, W_host);
    if (err != cudaSuccess || attr.type != cudaMemoryTypeHost) {
        cudaGetLastError();
        return moe_fail(KQ_ERR_NOT_PINNED, "experts must be page-locked host memory (cudaHostAlloc)");
    }
    kq_moe_stream* m = new (std::nothrow) kq_moe_stream();
    if (!m) return moe_fail(KQ_ERR_OOM, "host allocation");
    m->host = static_cast<const uint8_t*>(W_host);
    m->fmt = fmt;
    m->E = E;
    m->N = N;
    m->K = K;
    m->stride = expert_stride_bytes;
    m->expert_bytes = eb;
    m->slot_bytes = (eb + 255) / 256 * 256;
    m->max_ids = max_ids;
    m->n_sets = n_sets;
    err = cudaMalloc(&m->slots, m->slot_bytes * static_cast<size_t>(max_ids) * n_sets);
    if (err == cudaSuccess) err = cudaMalloc(&m->iota, sizeof(int32_t) * max_ids);
    if (err != cudaSuccess) {
        cudaGetLastError();
        destroy(m);
        return moe_fail(KQ_ERR_OOM, "device slot allocation", err);
    }
    std::vector<int32_t> iota(static_cast<size_t>(max_ids));
    for (int i = 0; i < max_ids; ++i) iota[static_cast<size_t>(i)] = i;
    err = cudaMemcpy(m->iota, iota.data(), sizeof(int32_t) * max_ids, cudaMemcpyHostToDevice);
    if (err == cudaSuccess) err = cudaStreamCreateWithFlags(&m->copy, cudaStreamNonBlocking);
    m->ready.resize(static_cast<size_t>(n_sets), nullptr);
    m->freed.resize(static_cast<size_t>(n_sets), nullptr);
    for (int t = 0; t < n_sets && err == cudaSuccess; ++t) {
        err = cudaEventCreateWithFlags(&m->ready[static_cast<size_t>(t)], cudaEventDisableTiming);
        if (err == cudaSuccess) err = cudaEventCreateWithFlags(&m->freed[static_cast<size_t>(t)], cudaEventDisableTiming);
    }
    if (err == cudaSuccess) err = cudaEventCreateWithFlags(&m->done, cudaEventDisableTiming);
    if (err != cudaSuccess) {
        destroy(m);
        return moe_fail(KQ_ERR_CUDA, "stream/event creation", err);
    }
    *out = m;
    return KQ_OK;
}

KQ_API int kq_moe_stream_run(kq_moe_stream* m, const int32_t* ids_host, int n_ids, const float* x,
                             int64_t x_stride, float* y, kq_stream_t compute) {
    g_moe_err[0] = 0;
    if (!m) return moe_fail(KQ_ERR_INVALID_ARG, "NULL stream object");
    if (n_ids < 0 || n_ids > m->max_ids) return moe_fail(KQ_ERR_INVALID_ARG, "n_ids outside 0..max_ids");
    if (n_ids == 0) return KQ_OK;
    if (!ids_host) return moe_fail(KQ_ERR_INVALID_ARG, "ids is NULL");
    for (int i = 0; i < n_ids; ++i)
        if (ids_host[i] < 0 || ids_host[i] >= m->E) return moe_fail(KQ_ERR_INVALID_ARG, "expert id outside [0, E)");
    if (!x || !y) return moe_fail(KQ_ERR_INVALID_ARG, "x or y is NULL");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(compute);
    const int t = static_cast<int>(m->runs % m->n_sets);
    uint8_t* set = m->slots + static_cast<size_t>(t) * m->max_ids * m->slot_bytes;
    // the copies wait only for the GEMV that last read this set, so they
    // overlap the GEMVs of the other sets
    cudaError_t err = cudaSuccess;
    if (m->runs >= m->n_sets) err = cudaStreamWaitEvent(m->copy, m->freed[static_cast<size_t>(t)], 0);
    if (err != cudaSuccess) return moe_fail(KQ_ERR_CUDA, "stream ordering", err);
    for (int i = 0; i < n_ids; ++i) {
        err = cudaMemcpyAsync(set + static_cast<size_t>(i) * m->slot_bytes,
                              m->host + static_cast<size_t>(ids_host[i]) * m->stride, m->expert_bytes,
                              cudaMemcpyHostToDevice, m->copy);
        if (err != cudaSuccess) return moe_fail(KQ_ERR_CUDA, "H2D expert copy", err);
    }
    err = cudaEventRecord(m->ready[static_cast<size_t>(t)], m->copy);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(cs, m->ready[static_cast<size_t>(t)], 0);
    if (err != cudaSuccess) return moe_fail(KQ_ERR_CUDA, "set ready", err);
    int st = kq_moe_gemv(set, m->fmt, n_ids, m->N, m->K, m->slot_bytes, m->iota, n_ids, x, x_stride, y, nullptr,
                         compute);
    if (st != KQ_OK) return moe_fail(st, kq_last_error());
    err = cudaEventRecord(m->freed[static_cast<size_t>(t)], cs);
    if (err == cudaSuccess) err = cudaEventRecord(m->done, cs);
    if (err != cudaSuccess) return moe_fail(KQ_ERR_CUDA, "set free", err);
    ++m->runs;
    return KQ_OK;
}

KQ_API int kq_moe_stream_wait(kq_moe_stream* m, int64_t timeout_ms) {
    g_moe_err[0] = 0;
    if (!m) return moe_fail(KQ_ERR_INVALID_ARG, "NULL stream object");
    const auto t0 = std::chrono::steady_clock::now();
    while (true) {
        cudaError_t err = cudaEventQuery(m->done);
        if (err == cudaSuccess) break;
        if (err != cudaErrorNotReady) return moe_fail(KQ_ERR_CUDA, "run completion", err);
        const auto ms =
            std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count();
        if (timeout_ms >= 0 && ms > timeout_ms) return moe_fail(KQ_ERR_TIMEOUT, "run did not finish in time");
        std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
    cudaError_t err = cudaStreamSynchronize(m->copy);
    if (err != cudaSuccess) return moe_fail(KQ_ERR_CUDA, "copy stream", err);
    return KQ_OK;
}

KQ_API void kq_moe_stream_destroy(kq_moe_stream* m) {
    if (!m) return;
    cudaStreamSynchronize(m->copy);
    destroy(m);
}

}  // extern "C"
