// kq_gguf.cu — reader of GGUF model files: header, metadata, tensor table,
// and tensor bytes on demand (host code only).
//
// The pages load "Q4_K_M" GGUF files ("Out-of-core LLM inference engine
// written from scratch in Rust", Results; "RunNburn - Run a 295B MoE from a
// 98GB GGUF ...") but print no format; this follows the public GGUF layout,
// versions 2 and 3, little-endian:
//   "GGUF" | u32 version | u64 tensor count | u64 metadata count
//   metadata: string key | u32 value type | value
//   tensor infos: string name | u32 n_dims | u64 ne[n_dims] | u32 ggml type |
//                 u64 offset (from the start of the data section)
//   data section: at the first multiple of general.alignment (default 32)
//                 after the tensor infos
// A string is u64 length + bytes (no terminator); an array is u32 element
// type + u64 count + elements.  ne[0] is the innermost dimension: a 2-D
// weight of N rows and K inputs has ne = {K, N}, rows stored one after
// another, which is libkq's matrix layout.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/kq.h"

struct kq_gguf {
    FILE* f = nullptr;
    uint32_t version = 0;
    uint64_t alignment = 32;
    uint64_t data_start = 0;
    uint64_t file_size = 0;
    struct Tensor {
        std::string name;
        int type = 0;
        int n_dims = 0;
        int64_t ne[4] = {1, 1, 1, 1};
        uint64_t offset = 0, nbytes = 0;
    };
    std::vector<Tensor> tensors;
};

namespace {

thread_local char g_gguf_err[256] = "";

int gguf_fail(int status, const char* msg) {
    snprintf(g_gguf_err, sizeof(g_gguf_err), "%s", msg);
    return status;
}

// ggml types: weights per block and bytes per block (0: not a type this
// reader sizes)
struct TypeInfo {
    int blck;
    int bytes;
};
TypeInfo type_info(int t) {
    switch (t) {
        case 0: return {1, 4};       // F32
        case 1: return {1, 2};       // F16
        case 8: return {32, 34};     // Q8_0
        case 10: return {256, 84};   // Q2_K
        case 11: return {256, 110};  // Q3_K
        case 12: return {256, 144};  // Q4_K
        case 13: return {256, 176};  // Q5_K
        case 14: return {256, 210};  // Q6_K
        case 30: return {1, 2};      // BF16
        default: return {0, 0};
    }
}

struct Reader {
    FILE* f;
    bool ok = true;
    template <typename T>
    T get() {
        T v{};
        if (ok && fread(&v, sizeof(T), 1, f) != 1) ok = false;
        return v;
    }
    bool skip(uint64_t n) {
        if (!ok) return false;
        if (n > (1ull << 40) || fseeko(f, static_cast<off_t>(n), SEEK_CUR) != 0) ok = false;
        return ok;
    }
    std::string str() {
        const uint64_t n = get<uint64_t>();
        if (!ok || n > (1u << 20)) {
            ok = false;
            return {};
        }
        std::string s(static_cast<size_t>(n), '\0');
        if (n && fread(&s[0], 1, static_cast<size_t>(n), f) != n) ok = false;
        return s;
    }
};

// Bytes of one scalar of GGUF value type t (0 for string / array / unknown).
int scalar_bytes(uint32_t t) {
    switch (t) {
        case 0: case 1: case 7: return 1;   // u8, i8, bool
        case 2: case 3: return 2;           // u16, i16
        case 4: case 5: case 6: return 4;   // u32, i32, f32
        case 10: case 11: case 12: return 8;  // u64, i64, f64
        default: return 0;
    }
}

// Skips one value of type t; reads general.alignment when `align` is set.
bool skip_value(Reader& r, uint32_t t, int depth, uint64_t* align) {
    if (depth > 2) return r.ok = false;
    if (t == 8) {  // string
        const uint64_t n = r.get<uint64_t>();
        return r.skip(n);
    }
    if (t == 9) {  // array
        const uint32_t et = r.get<uint32_t>();
        const uint64_t n = r.get<uint64_t>();
        if (!r.ok || n > (1ull << 32)) return r.ok = false;
        const int sb = scalar_bytes(et);
        if (sb) return r.skip(n * static_cast<uint64_t>(sb));
        for (uint64_t i = 0; i < n && r.ok; ++i) skip_value(r, et, depth + 1, nullptr);
        return r.ok;
    }
    const int sb = scalar_bytes(t);
    if (!sb) return r.ok = false;
    if (align && (t == 4 || t == 10)) {
        *align = t == 4 ? r.get<uint32_t>() : r.get<uint64_t>();
        return r.ok;
    }
    return r.skip(static_cast<uint64_t>(sb));
}

}  // namespace

extern "C" {

KQ_API const char* kq_gguf_last_error(void) { return g_gguf_err; }

KQ_API int kq_gguf_open(const char* path, kq_gguf** out) {
    g_gguf_err[0] = 0;
    if (!out || !path) return gguf_fail(KQ_ERR_INVALID_ARG, "NULL argument");
    *out = nullptr;
    FILE* f = fopen(path, "rb");
    if (!f) return gguf_fail(KQ_ERR_INVALID_ARG, "cannot open the file");
    kq_gguf* g = new (std::nothrow) kq_gguf();
    if (!g) {
        fclose(f);
        return gguf_fail(KQ_ERR_OOM, "host allocation");
    }
    g->f = f;
    auto bad = [&](const char* msg) {
        kq_gguf_close(g);
        return gguf_fail(KQ_ERR_INVALID_ARG, msg);
    };
    fseeko(f, 0, SEEK_END);
    g->file_size = static_cast<uint64_t>(ftello(f));
    fseeko(f, 0, SEEK_SET);
    Reader r{f};
    char magic[4];
    if (fread(magic, 1, 4, f) != 4 || memcmp(magic, "GGUF", 4) != 0) return bad("not a GGUF file (magic)");
    g->version = r.get<uint32_t>();
    if (!r.ok || (g->version != 2 && g->version != 3)) return bad("unsupported GGUF version");
    const uint64_t n_tensors = r.get<uint64_t>();
    const uint64_t n_kv = r.get<uint64_t>();
    if (!r.ok || n_tensors > (1u << 24) || n_kv > (1u << 24)) return bad("implausible tensor or metadata count");
    for (uint64_t i = 0; i < n_kv && r.ok; ++i) {
        const std::string key = r.str();
        const uint32_t t = r.get<uint32_t>();
        if (!r.ok) break;
        skip_value(r, t, 0, key == "general.alignment" ? &g->alignment : nullptr);
    }
    if (!r.ok) return bad("truncated or malformed metadata");
    if (g->alignment == 0 || (g->alignment & (g->alignment - 1)) != 0) return bad("alignment is not a power of two");
    g->tensors.resize(static_cast<size_t>(n_tensors));
    for (auto& t : g->tensors) {
        t.name = r.str();
        const uint32_t nd = r.get<uint32_t>();
        if (!r.ok || nd < 1 || nd > 4) return bad("bad tensor dimension count");
        t.n_dims = static_cast<int>(nd);
        uint64_t count = 1;
        for (uint32_t d = 0; d < nd; ++d) {
            const uint64_t ne = r.get<uint64_t>();
            if (ne == 0 || ne > (1ull << 40)) return bad("bad tensor dimension");
            t.ne[d] = static_cast<int64_t>(ne);
            count *= ne;
        }
        t.type = static_cast<int>(r.get<uint32_t>());
        t.offset = r.get<uint64_t>();
        if (!r.ok) return bad("truncated tensor table");
        const TypeInfo ti = type_info(t.type);
        if (ti.blck == 0 || t.ne[0] % ti.blck != 0) {
            t.nbytes = 0;  // a type this reader does not size: listed, not readable
        } else {
            t.nbytes = count / static_cast<uint64_t>(ti.blck) * static_cast<uint64_t>(ti.bytes);
        }
    }
    const uint64_t pos = static_cast<uint64_t>(ftello(f));
    g->data_start = (pos + g->alignment - 1) / g->alignment * g->alignment;
    for (const auto& t : g->tensors)
        if (t.nbytes && (t.offset % g->alignment != 0 || g->data_start + t.offset + t.nbytes > g->file_size))
            return bad("tensor data misaligned or past the end of the file");
    *out = g;
    return KQ_OK;
}

KQ_API int kq_gguf_tensor_count(const kq_gguf* g) { return g ? static_cast<int>(g->tensors.size()) : 0; }

KQ_API int kq_gguf_tensor_info(const kq_gguf* g, int i, const char** name, int* ggml_type, int* n_dims,
                               int64_t dims[4], uint64_t* file_offset, uint64_t* nbytes) {
    g_gguf_err[0] = 0;
    if (!g || i < 0 || i >= static_cast<int>(g->tensors.size()))
        return gguf_fail(KQ_ERR_INVALID_ARG, "no such tensor");
    const auto& t = g->tensors[static_cast<size_t>(i)];
    if (name) *name = t.name.c_str();
    if (ggml_type) *ggml_type = t.type;
    if (n_dims) *n_dims = t.n_dims;
    if (dims)
        for (int d = 0; d < 4; ++d) dims[d] = t.ne[d];
    if (file_offset) *file_offset = g->data_start + t.offset;
    if (nbytes) *nbytes = t.nbytes;
    return KQ_OK;
}

KQ_API int kq_gguf_find(const kq_gguf* g, const char* name) {
    if (!g || !name) return -1;
    for (size_t i = 0; i < g->tensors.size(); ++i)
        if (g->tensors[i].name == name) return static_cast<int>(i);
    return -1;
}

KQ_API int kq_gguf_kq_format(int ggml_type) {
    switch (ggml_type) {
        case 12: return KQ_FMT_Q4_K;
        case 14: return KQ_FMT_Q6_K;
        case 13: return KQ_FMT_Q5_K;
        case 10: return KQ_FMT_Q2_K;
        case 11: return KQ_FMT_Q3_K;
        case 8: return KQ_FMT_Q8_0;
        default: return 0;
    }
}

KQ_API int kq_gguf_read(const kq_gguf* g, int i, void* dst, uint64_t nbytes) {
    g_gguf_err[0] = 0;
    if (!g || i < 0 || i >= static_cast<int>(g->tensors.size()) || !dst)
        return gguf_fail(KQ_ERR_INVALID_ARG, "no such tensor or NULL destination");
    const auto& t = g->tensors[static_cast<size_t>(i)];
    if (t.nbytes == 0) return gguf_fail(KQ_ERR_UNSUPPORTED, "tensor type not sized by this reader");
    if (nbytes != t.nbytes) return gguf_fail(KQ_ERR_INVALID_ARG, "nbytes differs from the tensor's size");
    if (fseeko(g->f, static_cast<off_t>(g->data_start + t.offset), SEEK_SET) != 0 ||
        fread(dst, 1, static_cast<size_t>(nbytes), g->f) != nbytes)
        return gguf_fail(KQ_ERR_INVALID_ARG, "short read");
    return KQ_OK;
}

KQ_API void kq_gguf_close(kq_gguf* g) {
    if (!g) return;
    if (g->f) fclose(g->f);
    delete g;
}

}  // extern "C"
