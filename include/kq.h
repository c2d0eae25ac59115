/*
 * kq.h — libkq: decode-time matrix-vector products over GGUF K-quant
 * weights (Q2_K, Q3_K, Q4_K, Q5_K, Q6_K, and Q8_0) on NVIDIA B200 (sm_100a), with the weights
 * dequantised only in registers inside the fused kernels.
 *
 * What the method is (by page):
 *  - "Out-of-core LLM inference engine written from scratch in Rust",
 *    Approach: quantised weights are dequantised inside fused matmul kernels;
 *    speculative decoding verifies several positions with one pass; each
 *    layer is copied into one of a fixed set of device slots and runs there
 *    while copies of other layers proceed.  Results: Llama-3.3-70B Q4_K_M;
 *    a fully resident 30B MoE.
 *  - "Kortex: Streaming 70B Models on Consumer GPUs", Key components 2-3:
 *    the streaming pipeline overlaps transfers with compute; weights are
 *    dequantised only in GPU registers.  Token generation is memory-bandwidth
 *    bound (the paragraph before the first table).
 *  - "RunNburn - Run a 295B MoE from a 98GB GGUF ...": only the experts the
 *    router selects for a token are touched; native K-quant kernels.
 *
 * Weight layout.  A matrix has N output rows and K inputs (K % 256 == 0).
 * Row r is K/256 consecutive super-blocks; rows follow each other with no
 * gap, so row r starts at W + r * kq_row_bytes(fmt, K).
 *   Q4_K super-block, 144 bytes, 256 weights in 8 sub-blocks of 32:
 *     fp16 d | fp16 dmin | 12 bytes of 6-bit scales sc_j and mins m_j |
 *     128 bytes of 4-bit quants q.   w = d*sc_j*q - dmin*m_j.
 *   Q5_K super-block, 176 bytes, 256 weights in 8 sub-blocks of 32:
 *     fp16 d | fp16 dmin | 12 bytes of scales and mins (as Q4_K) |
 *     32 bytes qh of 5th bits | 128 bytes of low 4 bits.  Weight 64c+l
 *     (l < 32) takes the low nibble of byte 32c+l and bit 2c of qh[l];
 *     weight 64c+32+l the high nibble and bit 2c+1.
 *     w = d*sc_j*q - dmin*m_j, q in 0..31.  (A K-quant of the Q2_K..Q6_K
 *     family "RunNburn - Run a 295B MoE ..." runs natively.)
 *   Q2_K super-block, 84 bytes, 256 weights in 16 groups of 16:
 *     16 bytes sc_g | m_g << 4 | 64 bytes of 2-bit quants | fp16 d | fp16
 *     dmin.  Weight 128n+32j+l is bits 2j..2j+1 of quant byte 32n+l; its
 *     group is g = i/16.   w = d*sc_g*q - dmin*m_g, q in 0..3.
 *   Q3_K super-block, 110 bytes, 256 weights in 16 groups of 16:
 *     32 bytes hmask | 64 bytes of low 2 bits | 12 bytes of 6-bit scales
 *     v_g | fp16 d.  Weight 128n+32j+l: low bits as Q2_K, third bit = bit
 *     4n+j of hmask[l], q = (low | third << 2) - 4 in -4..3; v_g: low 4 bits
 *     from scale byte g (g < 8, low nibble) or g-8 (high nibble), top 2
 *     bits from bits 2(g/4) of byte 8 + g%4.   w = d*(v_g - 32)*q.
 *   Q6_K super-block, 210 bytes, 256 weights in 16 groups of 16:
 *     128 bytes low 4 bits | 64 bytes high 2 bits | 16 int8 scales s_g |
 *     fp16 d.   w = d*s_g*(q - 32), q in 0..63.
 *   Q8_0 blocks, 34 bytes per 32 weights: fp16 d | 32 int8 quants q.
 *     w = d*q.  A row is K/32 consecutive blocks; the library takes them
 *     in units of 8 blocks (256 weights, 272 bytes), so K % 256 == 0 here
 *     too.
 *   (The GGUF bit layout; the pages name the formats but print no
 *   layout.)
 *
 * Conventions for every entry point:
 *  - All pointers named W, x, y, ids, status are DEVICE pointers owned by the
 *    caller; libkq never frees or retains them past the call (the chain object
 *    below is the exception and says so).
 *  - W must be 16-byte aligned; its rows need not be (a Q6_K row of K = 2560
 *    is 2100 bytes, of K = 2304 1890): weights are copied in whole 16-byte
 *    units from the boundary at or below a stage's first byte, so a call
 *    may read up to 15 bytes past the last row, never past the 16-byte
 *    granule that holds the matrix's last byte.  Two or more columns of
 *    Q6_K with K % 2048 != 0 (any format whose rows are not a multiple of 16
 *    bytes) run one single-column launch per column.  x and
 *    y must be 4-byte aligned.
 *  - Calls are asynchronous on `stream` (0 = the legacy default stream).  The
 *    return value reports argument validation and launch errors only
 *    (KQ_ERR_CUDA carries cudaGetLastError()); kq_last_error() gives text.
 *  - Arithmetic: quants are unpacked exactly; sums are fp32 (or exact
 *    integers).  A single column rounds each activation to a 14-bit
 *    integer on a power-of-two grid per group of 32 (error at most 2^-14 of
 *    the group's largest |x|), every format alike; two or
 *    more columns run on the tensor cores with exact fp16 weight operands
 *    (sc*q; Q8_0 the int8 q, its d applied per block in fp32; Q3_K the code
 *    0..7, its -4 offset a separate term over the same rounded activations;
 *    Q6_K scales beyond +-64 rounded to fp16) and each activation rounded to
 *    fp16 after a power-of-two scale per column and super-block (relative
 *    error at most 2^-11, so |y - y_exact| <= 2^-11 * sum_i |w_i x_i| from
 *    the activations); shapes whose rows are not a multiple of 16 bytes run
 *    one single-column launch per column.  Every output satisfies
 *    |y - y_exact| <= 1e-3 * sum_i |w_i x_i| + 1e-6 for activations of
 *    comparable magnitude within each group of 32.
 *    Results are deterministic: the same inputs give bitwise-equal outputs;
 *    column c of a kq_gemv_multi call with k >= 2 does not depend on the
 *    other columns or on k, and k = 1 equals kq_gemv.
 *  - No C++ exception crosses this interface.  Functions without shared state
 *    are thread-safe; a kq_chain must not be used by two threads at once.
 */
#ifndef KQ_H_
#define KQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KQ_API __attribute__((visibility("default")))
#else
#define KQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA runtime's cudaStream_t, without pulling in the CUDA headers. */
typedef struct CUstream_st* kq_stream_t;

typedef enum {
    KQ_FMT_Q4_K = 1,
    KQ_FMT_Q6_K = 2,
    KQ_FMT_Q5_K = 3,
    KQ_FMT_Q2_K = 4,
    KQ_FMT_Q3_K = 5,
    KQ_FMT_Q8_0 = 6
} kq_fmt;

typedef enum {
    KQ_OK = 0,
    KQ_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad format, misalignment */
    KQ_ERR_UNSUPPORTED = 2,   /* valid but not handled (e.g. K > 32768, or beyond shared memory) */
    KQ_ERR_NOT_PINNED = 3,    /* host memory that must be page-locked is not */
    KQ_ERR_OOM = 4,           /* a device or pinned allocation failed */
    KQ_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
    KQ_ERR_TIMEOUT = 6,       /* a bounded wait ran out */
    KQ_ERR_DEVICE_CHECK = 7,  /* a device-side check failed (see kq_moe_gemv) */
    KQ_ERR_INJECTED = 8       /* a failure requested through KQ_FAULT (tests) */
} kq_status;

/* Library version as 10000*major + 100*minor + patch. */
KQ_API int kq_version(void);

/* Static text for a status code. */
KQ_API const char* kq_status_str(int status);

/* Text describing the last failure on the calling thread ("" if none). */
KQ_API const char* kq_last_error(void);

/* Reads and clears the current device's fault word (0 if no fault): a
 * kernel whose bounded wait ran out sets it to KQ_ERR_TIMEOUT instead of
 * hanging.  Synchronous.  *out is a HOST int. */
KQ_API int kq_device_fault(int* out);

/* Test hook for the failure-detection tests: a device-side wait that runs
 * out.  spec "hold@S" (S >= 1): the next single-column GEMV launch (kq_gemv,
 * or a one-column group of kq_gemv_multi) does not copy the S-th weight stage
 * of its first CTA, and that CTA's bounded waits give up after 1 ms instead
 * of 2 s;
 * the consumers waiting for that stage then time out, the CTA stops, lets
 * the copies it issued land, and the launch ends with the fault word set to
 * KQ_ERR_TIMEOUT (read it with kq_device_fault); that CTA's outputs are
 * undefined.  One-shot; NULL or "" cancels.  No trap, no hang: the context
 * stays usable.  Process-wide; KQ_ERR_INVALID_ARG for another spec. */
KQ_API int kq_inject(const char* spec);

/* Measurement helper: reads `bytes` (a multiple of 16) at src (DEVICE,
 * 16-byte aligned) once and XORs what it read into *out (DEVICE uint32), so
 * that the time of the call is the device's read-only bandwidth -- the
 * ceiling of a GEMV, which only reads its weights (decode is bound by the
 * weight bytes: "Kortex: Streaming 70B Models on Consumer GPUs", the
 * paragraph before the first table).  mode 0: 16-byte loads from every
 * thread of a full grid; mode 1: the GEMV kernels' weight path, one CTA per
 * SM bulk-copying (TMA, no multicast) 48 KiB stages of a contiguous range
 * into a 4-slot shared-memory ring, one warp reading each stage from shared
 * memory and releasing it (no other work).  Asynchronous on `stream`.  Errors: KQ_ERR_INVALID_ARG,
 * KQ_ERR_CUDA; a bounded wait that runs out sets the fault word. */
KQ_API int kq_read_probe(const void* src, size_t bytes, int mode, uint32_t* out, kq_stream_t stream);

/* Bytes per super-block (Q2_K 84, Q3_K 110, Q4_K 144, Q5_K 176, Q6_K 210;
 * Q8_0 272, per 8 blocks of 32 weights) or 0 for an unknown format. */
KQ_API size_t kq_block_bytes(int fmt);

/* Bytes per weight row: (K/256) * kq_block_bytes(fmt); 0 if K % 256 != 0. */
KQ_API size_t kq_row_bytes(int fmt, int64_t K);

/*
 * kq_gemv — y = W x for one quantised matrix.
 *   W: N x K matrix in `fmt` (device).  x: K floats (device).  y: N floats
 *   (device, written).  N >= 1, K >= 256, K % 256 == 0.
 * The fused dequant-matmul of "Out-of-core LLM inference engine written from
 * scratch in Rust" (Approach) and "Kortex: Streaming 70B Models on Consumer
 * GPUs" (Key components 3): each weight is read from HBM once and
 * dequantised in registers.
 */
KQ_API int kq_gemv(const void* W, int fmt, int64_t N, int64_t K, const float* x, float* y,
            kq_stream_t stream);

/*
 * kq_gemv_multi — Y = W X for k activation columns sharing one weight read.
 *   X column c is x + c*ldx (K floats each, ldx >= K); Y column c is
 *   y + c*ldy (N floats each, ldy >= N); 1 <= k <= 8.
 * The verify pass of speculative decoding ("Out-of-core LLM inference engine
 * ...", Approach: several positions verified with one pass of the large
 * model).  With k >= 2 the products run on the tensor cores (every format,
 * rows a multiple of 16 bytes); column c then equals column c of any other
 * k >= 2 call on the same activations bitwise, and kq_gemv within the
 * tolerance.  Rows off the 16-byte grid run one single-column launch per
 * column (each column equal to kq_gemv bitwise).  k = 1 equals kq_gemv
 * bitwise.
 */
KQ_API int kq_gemv_multi(const void* W, int fmt, int64_t N, int64_t K, const float* x, int64_t ldx,
                  int k, float* y, int64_t ldy, kq_stream_t stream);

/* Activation prologues applied inside kq_gemv_fused (never written back). */
typedef enum {
    KQ_PRO_NONE = 0,
    /* x'_i = x_i * gamma_i / sqrt(mean_j(x_j^2) + eps), per column: the norm
     * in front of a layer's qkv and gate|up matmuls. */
    KQ_PRO_RMSNORM = 1,
    /* Each column holds 2K values [g; u]; x'_i = silu(g_i) * u_i with
     * silu(g) = g / (1 + exp(-g)): the gated activation in front of down,
     * taking the gate|up matmul's stacked output as is. */
    KQ_PRO_SWIGLU = 2
} kq_prologue_kind;

typedef struct {
    int kind;            /* kq_prologue_kind */
    const float* gamma;  /* KQ_PRO_RMSNORM: K weights (device); else unused */
    float eps;           /* KQ_PRO_RMSNORM: > 0 */
} kq_prologue;

/*
 * kq_gemv_fused — Y = W P(X): kq_gemv_multi with a prologue P applied to the
 * activations as they are staged, so the normalised or gated vector never
 * goes through HBM.
 *   pro: HOST pointer, NULL = KQ_PRO_NONE.  For KQ_PRO_SWIGLU, column c is
 *   x + c*ldx with 2K floats (ldx >= 2K); otherwise as kq_gemv_multi.
 * The pages do not spell these steps out: they are the RMSNorm and SiLU-gated
 * MLP of the Llama and Qwen model families whose decode the pages benchmark
 * ("Kortex: Streaming 70B Models on Consumer GPUs", the tables; "Out-of-core
 * LLM inference engine written from scratch in Rust", Results).  Each CTA
 * computes the column's sum of squares over all K itself (fixed order), so
 * results are deterministic and independent of the grid.
 * Errors: KQ_ERR_INVALID_ARG for an unknown kind, a NULL gamma, eps <= 0 or
 * ldx < 2K for SwiGLU; otherwise as kq_gemv_multi.
 */
KQ_API int kq_gemv_fused(const void* W, int fmt, int64_t N, int64_t K, const float* x, int64_t ldx, int k,
                         const kq_prologue* pro, float* y, int64_t ldy, kq_stream_t stream);

/* One GEMV of a kq_gemv_steps call (one activation column). */
typedef struct kq_step {
    const void* W;       /* device: N rows of K/256 blocks of `fmt`, as kq_gemv */
    int fmt;             /* kq_fmt */
    int64_t N, K;
    const float* x;      /* device: K floats (2K for KQ_PRO_SWIGLU), 4-byte aligned */
    float* y;            /* device: N floats */
    kq_prologue pro;     /* prologue of this step (kind KQ_PRO_NONE: none) */
    int after;           /* nonzero: x (or gamma) is written by an earlier step of this call */
} kq_step;

/*
 * kq_gemv_steps — run n_steps single-column GEMVs (each y = W P(x) as
 * kq_gemv_fused with k = 1) in order, in as few launches as possible: one
 * persistent grid streams the weights of step after step without a gap
 * while the steps are computed.  A step with `after` set starts only when
 * every earlier step of the call has finished on the whole GPU (its x may
 * be an earlier step's y); other steps may overlap the step before them,
 * so a step without `after` must not read what an earlier step of the call
 * writes.  This is the decode chain of the pages' engines -- a token's
 * matvecs one after another, each reading the weights once ("Kortex:
 * Streaming 70B Models on Consumer GPUs", the paragraph before the first
 * table; "Out-of-core LLM inference engine written from scratch in Rust",
 * Approach) -- without a kernel boundary between matvecs.
 *   steps: HOST array of n_steps descriptors (read during the call only).
 * Results equal, bit for bit, the same steps run one by one with
 * kq_gemv_fused (k = 1).  Asynchronous on `stream`; the call returns once
 * the launches are queued.
 * Errors: KQ_ERR_INVALID_ARG (n_steps < 0, a NULL steps array, or any step's
 * arguments as kq_gemv_fused would reject them), KQ_ERR_UNSUPPORTED (a
 * step's shape the single-column kernel does not take, or steps whose
 * activations and stages do not fit shared memory together), KQ_ERR_CUDA.
 * Nothing is launched unless every step is valid.
 */
KQ_API int kq_gemv_steps(const kq_step* steps, int n_steps, kq_stream_t stream);

/*
 * kq_gemv_splitk — kq_gemv_multi for tall-skinny matrices: when the matrix
 * has fewer row pairs than the GPU has SMs, K is also split across CTAs.
 * Each CTA writes the partial sums of its K range to `workspace`, and a
 * second kernel adds the ranges in a fixed order (deterministic, but not
 * bitwise equal to kq_gemv, whose summation order differs).  For matrices
 * that need no split it is exactly kq_gemv_multi and ignores the workspace.
 *   workspace: DEVICE scratch of at least kq_splitk_workspace_bytes(fmt, N,
 *   K, k) bytes, owned by the caller; calls that share a workspace must not
 *   overlap on the GPU.  Other arguments as kq_gemv_multi.
 * Split-K for tall-skinny shapes; the pages' decode matvecs ("Kortex:
 * Streaming 70B Models on Consumer GPUs", the paragraph before the first
 * table) include narrow projections such as the grouped k/v heads.
 */
KQ_API size_t kq_splitk_workspace_bytes(int fmt, int64_t N, int64_t K, int k);
KQ_API int kq_gemv_splitk(const void* W, int fmt, int64_t N, int64_t K, const float* x, int64_t ldx, int k,
                          float* y, int64_t ldy, void* workspace, size_t workspace_bytes, kq_stream_t stream);

/*
 * kq_gemv_splitk_noalloc — kq_gemv_splitk for callers that cannot allocate
 * device memory: a real-time or callback thread that must not enter the
 * allocator (its locks, its implicit synchronisation), an engine whose device
 * memory is all owned by its own arena, or a plugin given only its inputs and
 * outputs.  Such callers cannot supply the split-K workspace, so this call
 * keeps the partial sums in a 64 KiB array built into the library (every GPU
 * that loads libkq holds it until the process exits).  It calls no cudaMalloc,
 * cudaFree or allocating routine (the first call per device aside: see
 * below).
 *   Arguments, layout and results are those of kq_gemv_splitk (the same
 *   kernels and summation order, so the outputs are identical).
 *   Errors: KQ_ERR_UNSUPPORTED when the split would need more partial sums
 *   than the 64 KiB hold (16384 floats = ranges * k * N); the text is in
 *   kq_last_error().  Other errors as kq_gemv_splitk.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current.  With CUDA's lazy
 *   module loading (the default) that lookup may load the library's device
 *   module, which allocates device memory and takes driver locks, so make
 *   the first call per device outside real-time and capture code (a
 *   warm-up call at start-up); every later call allocates nothing.  The
 *   looked-up address is cached per device: after cudaDeviceReset the
 *   library must be unloaded and loaded again.
 *   All calls share the one array: calls that overlap on the GPU (other
 *   streams, other threads) race on it and must be ordered by the caller.
 *   Nothing in it needs clearing between calls: each call writes every
 *   partial sum it later reads.
 * The pages have no counterpart to this entry point.
 */
KQ_API int kq_gemv_splitk_noalloc(const void* W, int fmt, int64_t N, int64_t K, const float* x, int64_t ldx,
                                  int k, float* y, int64_t ldy, kq_stream_t stream);

/*
 * kq_moe_gemv — routed-expert GEMV.
 *   W_experts: E matrices, each N x K in `fmt`, matrix e at
 *   W_experts + e*expert_stride_bytes (stride >= N*row_bytes, 16-byte
 *   multiple).  ids: n_ids int32 expert ids (DEVICE memory, read by the
 *   kernel).  x: if x_stride == 0 one K-vector shared by all ids, else id i
 *   uses x + i*x_stride (x_stride >= K).  y: n_ids x N floats, row-major
 *   (y + i*N is the output for the i-th id).
 *   An id outside [0, E) is not dereferenced: its N outputs are set to 0 and,
 *   if status is not NULL, *status (device int32) is set to
 *   KQ_ERR_DEVICE_CHECK.  The kernel never traps.
 * Only the selected experts' weights are read ("RunNburn ...": the selected
 * experts for each token; "Out-of-core LLM inference engine ...", Results:
 * a fully resident 30B MoE).  Output i equals kq_gemv on expert ids[i].
 */
KQ_API int kq_moe_gemv(const void* W_experts, int fmt, int E, int64_t N, int64_t K,
                size_t expert_stride_bytes, const int32_t* ids, int n_ids, const float* x,
                int64_t x_stride, float* y, int32_t* status, kq_stream_t stream);

/*
 * Streamed MoE — the routed experts' weights stay in PAGE-LOCKED HOST memory
 * and only the selected experts are copied to the device, per call
 * ("RunNburn - Run a 295B MoE from a 98GB GGUF on a 64GB RAM Desktop": the
 * experts a token selects are gathered on demand; "Out-of-core LLM
 * inference engine ...", Approach: weight copies into device slots proceed
 * alongside the computation).
 *
 * kq_moe_stream_create: the expert stack W_host (HOST pointer, page-locked,
 *   owned by the caller and kept alive and unchanged until destroy): E
 *   matrices of N x K in `fmt`, matrix e at W_host + e*expert_stride_bytes
 *   (stride >= N*row_bytes).  max_ids: the most ids one run routes; n_sets
 *   (>= 1): sets of max_ids device slots used in turn, so the copies of the
 *   next run overlap the GEMV of this one.  Allocates n_sets*max_ids slots of
 *   N*row_bytes (rounded up to 256) bytes, a copy stream and events.
 *   KQ_ERR_NOT_PINNED if W_host is not page-locked, KQ_ERR_OOM if the slots
 *   do not fit.
 * kq_moe_stream_run: ids_host (HOST int32, n_ids <= max_ids, each in [0, E),
 *   else KQ_ERR_INVALID_ARG and nothing is enqueued); x, y as kq_moe_gemv
 *   (DEVICE).  Enqueues, on the object's copy stream, the H2D copies of the
 *   routed experts into the next slot set (after the GEMV that last read
 *   that set), then on `compute` the routed GEMV over the set.  Asynchronous.
 *   y[i] equals, bitwise, kq_moe_gemv with the same experts resident in
 *   device memory.  The copies wait only for the GEMV that last read their
 *   set, so they overlap the GEMVs of the other sets.
 * kq_moe_stream_wait: host-side polling until the last run finished;
 *   KQ_ERR_TIMEOUT after timeout_ms (negative: no limit).
 * kq_moe_stream_destroy: waits for the copies, frees slots, stream, events.
 * One object must not be used by two threads at once.
 */
typedef struct kq_moe_stream kq_moe_stream;

KQ_API int kq_moe_stream_create(const void* W_host, int fmt, int E, int64_t N, int64_t K,
                                size_t expert_stride_bytes, int max_ids, int n_sets, kq_moe_stream** out);
KQ_API int kq_moe_stream_run(kq_moe_stream* s, const int32_t* ids_host, int n_ids, const float* x,
                             int64_t x_stride, float* y, kq_stream_t compute);
KQ_API int kq_moe_stream_wait(kq_moe_stream* s, int64_t timeout_ms);
KQ_API void kq_moe_stream_destroy(kq_moe_stream* s);
/* Text describing the last streamed-MoE failure on the calling thread. */
KQ_API const char* kq_moe_stream_last_error(void);

/*
 * GGUF reader (host only) — the tensor table of a GGUF model file (versions
 * 2 and 3) and its tensors' bytes on demand, so that a weight stored in the
 * file can be handed to the GEMV entry points.  A 2-D weight of N rows and
 * K inputs has dims {K, N} (dims[0] innermost); its rows follow one another
 * in the file, which is libkq's matrix layout: copy its bytes to the device
 * (16-byte aligned) and call kq_gemv(W, kq_gguf_kq_format(type), N, K, ...).
 * The pages load GGUF files ("Out-of-core LLM inference engine ...",
 * Results: Q4_K_M; "RunNburn - Run a 295B MoE from a 98GB GGUF ...") but
 * print no format; this follows the public GGUF layout.
 *
 * kq_gguf_open: reads the header, skips the metadata (except
 *   general.alignment) and reads the tensor table.  KQ_ERR_INVALID_ARG for a
 *   missing file, a bad magic or version, a truncated or malformed table, or
 *   tensor data past the end of the file.  The object keeps the file open
 *   until kq_gguf_close; one object must not be read by two threads at once.
 * kq_gguf_tensor_info: name (valid until close), ggml type id, dims (unused
 *   ones 1), absolute file offset and byte size (0 for a type this reader
 *   does not size: F32, F16, BF16, Q8_0 and Q2_K..Q6_K are sized).
 * kq_gguf_find: index of the named tensor, or -1.
 * kq_gguf_kq_format: the KQ_FMT_* of a ggml type id (Q4_K 12, Q5_K 13,
 *   Q6_K 14, Q2_K 10, Q3_K 11, Q8_0 8), 0 for none.
 * kq_gguf_read: copies tensor i (nbytes must equal its size) into dst
 *   (HOST memory, page-locked or not).
 */
typedef struct kq_gguf kq_gguf;

KQ_API int kq_gguf_open(const char* path, kq_gguf** out);
KQ_API int kq_gguf_tensor_count(const kq_gguf* g);
KQ_API int kq_gguf_tensor_info(const kq_gguf* g, int i, const char** name, int* ggml_type, int* n_dims,
                               int64_t dims[4], uint64_t* file_offset, uint64_t* nbytes);
KQ_API int kq_gguf_find(const kq_gguf* g, const char* name);
KQ_API int kq_gguf_kq_format(int ggml_type);
KQ_API int kq_gguf_read(const kq_gguf* g, int i, void* dst, uint64_t nbytes);
KQ_API void kq_gguf_close(kq_gguf* g);
/* Text describing the last GGUF failure on the calling thread. */
KQ_API const char* kq_gguf_last_error(void);

/*
 * kq_unpack — debug: the integer fields of n_blocks consecutive super-blocks
 * as the GEMV kernels decode them, for bit-exact comparison with a plain
 * decoder (the pages ask that quants be unpacked exactly: "Kortex: Streaming
 * 70B Models on Consumer GPUs", Key components 3, dequantisation in
 * registers; the block layouts are those above).
 *   q:       n_blocks*256 int8, quant of weight i of block b at q[256b+i]
 *            (Q2_K 0..3; Q3_K -4..3; Q4_K 0..15; Q5_K 0..31; Q6_K 0..63,
 *            before the -32 offset; Q8_0 the int8 quants)
 *   sc_or_s: n_blocks*16 bytes, the block's group scales at 16b+g: Q4_K and
 *            Q5_K sc_0..7 (bytes 8..15 zero); Q2_K the 16 4-bit sc_g; Q3_K
 *            the 16 6-bit v_g (before the -32 offset); Q6_K the 16 int8 s_g
 *            as two's-complement bytes; Q8_0 its eight fp16 d as raw
 *            little-endian bytes
 *   m:       n_blocks*16 bytes or NULL: Q4_K and Q5_K m_0..7 (bytes 8..15
 *            zero); Q2_K the 16 4-bit m_g; other formats zeros
 *   d:       n_blocks floats: d widened exactly from fp16 (Q8_0: 0)
 *   dmin:    n_blocks floats or NULL: dmin of Q2_K, Q4_K and Q5_K (else 0)
 *   For Q8_0 a "block" here is a unit of 8 blocks (256 weights).
 * All device pointers; W must be 16-byte aligned, d and dmin 4-byte aligned.
 * Errors: KQ_ERR_INVALID_ARG (unknown format, n_blocks < 0, a NULL q,
 * sc_or_s or d, misalignment), KQ_ERR_CUDA.
 */
KQ_API int kq_unpack(const void* W, int fmt, int64_t n_blocks, int8_t* q, uint8_t* sc_or_s, uint8_t* m, float* d,
                     float* dmin, kq_stream_t stream);

/*
 * kq_unpack_fields — the same decode in a packed form (three arrays):
 *   q:  n_blocks*256 bytes, as kq_unpack
 *   sc: n_blocks*16 bytes; Q4_K, Q5_K: sc_0..7 then m_0..7; Q2_K: the 16
 *       bytes sc_g | m_g << 4 as stored; Q3_K, Q6_K, Q8_0: as kq_unpack
 *   d:  n_blocks*2 floats: d, dmin (0 where the format has none)
 * Errors as kq_unpack.
 */
KQ_API int kq_unpack_fields(const void* W, int fmt, int64_t n_blocks, uint8_t* q, uint8_t* sc, float* d,
                            kq_stream_t stream);

/* ------------------------------------------------------------------------
 * Streamed layer chain ("Out-of-core LLM inference engine written from
 * scratch in Rust", Approach: layers are copied into a fixed set of device
 * slots and run while other layers compute; "Kortex: Streaming 70B Models
 * on Consumer GPUs", Key components 2: the pipeline overlaps transfers with
 * compute).
 *
 * A chain holds n_layers layers of mats_per_layer matrices whose weights
 * stay in PAGE-LOCKED HOST memory.  kq_chain_run copies layer l into device
 * slot l % n_slots on the chain's own copy stream and runs that layer's
 * GEMVs (the kq_gemv kernels) on the caller's stream as soon as its copy has
 * landed; the copy of layer l + n_slots waits until layer l's GEMVs are done
 * with the slot.  Outputs equal a resident kq_gemv run bitwise.
 * ---------------------------------------------------------------------- */

/* One weight matrix: W is HOST page-locked memory (cudaHostAlloc or
 * cudaHostRegister), N x K in format fmt. */
typedef struct kq_matrix_desc {
    const void* W;
    int fmt;
    int64_t N;
    int64_t K;
} kq_matrix_desc;

typedef struct kq_chain kq_chain;

/* Creates a chain.  mats: n_layers * mats_per_layer descriptors, layer
 * major; every layer must have the same formats and shapes (matrix m of
 * each layer alike).  The chain copies the descriptor array (not the
 * weights: they must stay valid and pinned for the chain's lifetime) and
 * allocates n_slots device slots of kq_chain_slot_bytes() bytes each, one
 * copy stream and its events on the current device.
 * Errors: KQ_ERR_INVALID_ARG, KQ_ERR_NOT_PINNED (a W that is not
 * page-locked), KQ_ERR_OOM, KQ_ERR_CUDA.  On error *out is NULL. */
KQ_API int kq_chain_create(const kq_matrix_desc* mats, int n_layers, int mats_per_layer, int n_slots,
                           kq_chain** out);

/* Residency for a device-memory budget ("Kortex: Streaming 70B Models on
 * Consumer GPUs", Key components: layers that fit stay in VRAM, the rest
 * stream): *n_resident leading layers stay resident next to a ring of
 * *n_slots slots (1 <= *n_slots <= max_slots), together within
 * budget_bytes of device memory (layer bytes as kq_chain_slot_bytes counts
 * them; activations and outputs are not counted).  Every layer fits:
 * *n_resident = n_layers, *n_slots = 0.  Host arithmetic only.
 * Errors: KQ_ERR_INVALID_ARG, KQ_ERR_OOM (the budget does not hold one
 * layer). */
KQ_API int kq_chain_plan(const kq_matrix_desc* mats, int n_layers, int mats_per_layer, size_t budget_bytes,
                         int max_slots, int* n_resident, int* n_slots);

/* kq_chain_create with the first n_resident layers (0..n_layers) copied
 * once, during this call, into device memory of their own; a run launches
 * their GEMVs directly and streams only the other layers, through n_slots
 * slots (>= 1 unless every layer is resident).  Outputs equal a resident
 * run bitwise.  Errors as kq_chain_create. */
KQ_API int kq_chain_create_resident(const kq_matrix_desc* mats, int n_layers, int mats_per_layer, int n_resident,
                                    int n_slots, kq_chain** out);

/* Resident leading layers of a chain. */
KQ_API int kq_chain_resident_layers(const kq_chain* c);

/* Device bytes of one slot (one layer's matrices, 256-byte aligned each). */
KQ_API size_t kq_chain_slot_bytes(const kq_chain* c);

/* Enqueues one pass over every layer.  x, y: HOST arrays of n_layers *
 * mats_per_layer DEVICE pointers (activation K floats, output N floats per
 * matrix).  Asynchronous: returns once everything is queued; the copy
 * stream starts after the work already queued on `compute`.  The
 * environment variable KQ_FAULT=copy@L makes the run stop before copying
 * layer L and return KQ_ERR_INJECTED (what was queued still completes). */
KQ_API int kq_chain_run(kq_chain* c, const float* const* x, float* const* y, kq_stream_t compute);

/* Waits (host-side polling, no device spin) until the last run finished;
 * KQ_ERR_TIMEOUT if it takes longer than timeout_ms (negative: no limit). */
KQ_API int kq_chain_wait(kq_chain* c, int64_t timeout_ms);

/* Text describing the last chain failure on the calling thread. */
KQ_API const char* kq_chain_last_error(void);

/* Waits for the chain's copies, then frees its slots, stream and events. */
KQ_API void kq_chain_destroy(kq_chain* c);

/* The streamed chain by layer (the same object and schedule as kq_chain_*,
 * for callers that hold their weights per layer). */
typedef struct kq_layer_desc {
    const kq_matrix_desc* mats;  /* HOST array of n_mats matrices (weights page-locked) */
    int n_mats;
} kq_layer_desc;

/* kq_chain_create over n_layers layer descriptors (every layer with the same
 * n_mats, formats and shapes; the descriptor arrays are read during the call
 * only).  Errors as kq_chain_create; on error *out is NULL. */
KQ_API int kq_stream_chain_create(const kq_layer_desc* layers, int n_layers, int n_slots, kq_chain** out);

/* One streamed pass, waited for: kq_chain_run(c, x_in, y_out, compute), then
 * kq_chain_wait(c, timeout_ms).  x_in / y_out: HOST arrays of n_layers *
 * n_mats DEVICE pointers, layer major.  KQ_OK once the pass has finished;
 * KQ_ERR_TIMEOUT if it has not within timeout_ms (negative: no limit) -- the
 * pass then goes on on the device and kq_chain_wait can wait for it again.
 * A run that fails part-way returns its own error after what it queued has
 * drained (bounded by timeout_ms). */
KQ_API int kq_stream_chain(kq_chain* c, const float* const* x_in, float* const* y_out, kq_stream_t compute,
                           int64_t timeout_ms);

/* kq_chain_destroy. */
KQ_API void kq_stream_chain_destroy(kq_chain* c);

#ifdef __cplusplus
}
#endif

#endif /* KQ_H_ */
