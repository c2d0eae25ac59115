// kq_device.cuh — sm_100a device helpers for libkq: mbarrier / bulk-copy
// (TMA) PTX wrappers, bounded waits, and the K-quant unpack primitives the
// GEMV kernels and the debug unpack kernel share.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace kq {

constexpr int kQ4Bytes = 144;      // Q4_K super-block
constexpr int kQ6Bytes = 210;      // Q6_K super-block
constexpr int kQ5Bytes = 176;      // Q5_K super-block
constexpr int kQ2Bytes = 84;       // Q2_K super-block
constexpr int kQ3Bytes = 110;      // Q3_K super-block
constexpr int kQ80Bytes = 272;     // Q8_0: eight 34-byte blocks (256 weights)
// Bytes per 256 weights of format FMT (1 Q4_K, 2 Q6_K, 3 Q5_K, 4 Q2_K, 5
// Q3_K, 6 Q8_0).
template <int FMT>
__host__ __device__ constexpr int block_bytes_of() {
    return FMT == 1 ? kQ4Bytes : FMT == 2 ? kQ6Bytes : FMT == 3 ? kQ5Bytes : FMT == 4 ? kQ2Bytes
         : FMT == 5 ? kQ3Bytes : kQ80Bytes;
}
constexpr int kConsumerWarps = 8;  // warps that dequantise and multiply
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kRegion = 132;       // floats per activation region: 128 x + 4 sums
constexpr int kMaxStages = 8;
constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded-wait limit (2 s)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make initialised barriers visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// try_wait with a suspend-time hint: the warp sleeps in hardware until the
// phase completes or about `kSuspendNs` pass, instead of spinning and
// taking issue slots from the warps that compute.
constexpr uint32_t kSuspendNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, giving up after limit_ns or
// when another thread of the CTA has raised `abort_flag`.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  unsigned long long limit_ns = kWaitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// The producer's last wait before its CTA may exit: phase `parity` of a
// ring slot's `full` barrier, which completes when a bulk copy it issued
// into this CTA's shared memory has landed.  Unlike mbar_wait_bounded it
// does not give up when the CTA has aborted (a copy in flight must land
// before the shared memory can be released), only after kWaitNs.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitNs) return false;
    }
}

// The producer's record of its ring: which slots last received a bulk copy
// (and at which phase).  A slot is reused only after the consumers released
// it, and the producer issues nothing once the CTA has aborted, so each slot
// holds at most one copy that may still be in flight; drain() waits for
// each before the CTA exits, abort or not.
struct RingTrack {
    uint32_t issued = 0, phase = 0;
    __device__ __forceinline__ void issue(int slot, uint32_t ph) {
        issued |= 1u << slot;
        phase = (phase & ~(1u << slot)) | ((ph & 1u) << slot);
    }
    __device__ __forceinline__ void skip(int slot) { issued &= ~(1u << slot); }
    __device__ void drain(uint64_t* full, int ns) const {
        for (int s = 0; s < ns; ++s)
            if ((issued >> s) & 1u) mbar_wait_drain(&full[s], (phase >> s) & 1u);
    }
};

// ------------------------------------------------------------- clusters

// Every thread of every CTA of the cluster: releases this CTA's writes,
// acquires the other CTAs' (also orders mbarrier initialisation before any
// remote arrive).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The shared::cluster address of the same location in CTA `rank`.
__device__ __forceinline__ uint32_t map_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_f32(uint32_t cluster_addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t cluster_addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
    return v;
}

// Release at cluster scope of this thread's earlier shared-memory writes,
// and those it has seen through a CTA barrier, before a remote arrive.
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

// Arrive (release at cluster scope) on an mbarrier of another CTA.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Bounded wait on a local mbarrier whose arrivals come from other CTAs
// (acquire at cluster scope, so their writes before the arrive are seen).
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
            : "memory");
        if (ok) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitNs) return false;
    }
}

// L2 policy for the weight stream: read once per pass, so its lines are
// the first to go, leaving the activations and outputs (small, reused by
// every CTA) in L2.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 1-D bulk copy global -> shared (the TMA engine, no tensor map, no
// multicast) of weights, completing `bytes` of transaction count on `bar`,
// with the L2 policy `policy`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also returns the OR of `pred` over its threads, so a
// decision taken after it is the same in every participating thread.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Programmatic dependent launch: wait for the preceding grid's memory, and
// allow the next grid to start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ float4 lds128f(const float* p) { return *reinterpret_cast<const float4*>(p); }

// Shared-memory loads/stores by 32-bit shared-window address (ld.shared /
// st.shared): the hot loops keep all their addresses in 32-bit registers.
__device__ __forceinline__ uint4 ld_s128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float4 ld_s128f(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float2 ld_s64f(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 ld_s2w(uint32_t a) {  // two words, 8-byte aligned
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ void st_s64u(uint32_t a, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ uint32_t ld_s32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ float ld_s32f(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void st_s32f(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void st_s64f(uint32_t a, float2 v) {
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(v.x), "f"(v.y) : "memory");
}

__device__ __forceinline__ uint32_t u4w(const uint4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// -------------------------------------------------------- integer dots

// Four byte products summed into an int32 (DP4A): unsigned quants with
// signed (us) or unsigned (uu) activation bytes.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
// Byte k of w as a sign-extended int (one byte permute whose selector
// replicates the byte's sign bit into the upper bytes).
__device__ __forceinline__ int sext_byte(uint32_t w, int k) {
    uint32_t r;
    const uint32_t sel = static_cast<uint32_t>(k) | ((8u + static_cast<uint32_t>(k)) * 0x1110u);
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "r"(sel));
    return static_cast<int>(r);
}
// Signed quants (Q8_0) with signed (ss) or unsigned (su) activation bytes.
__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp4a_su(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// ----------------------------------------------------------------- Q4_K

// The four 6-bit scales and four 6-bit mins of half H (sub-blocks
// 4H..4H+3) of a Q4_K super-block, one per byte.  w1, w2, w3 are the 12
// scale bytes (little-endian words).  For j < 4 the scale/min are the low 6
// bits of bytes j / j+4; for j >= 4 the low 4 bits come from byte j+4 (scale
// in its low nibble, min in its high nibble) and the top 2 bits from bits
// 6-7 of byte j-4 (scale) / byte j (min).
__device__ __forceinline__ void q4k_half_scales(uint32_t w1, uint32_t w2, uint32_t w3, int H, uint32_t& sc4,
                                                uint32_t& m4) {
    const uint32_t sc_lo = w1 & 0x3F3F3F3Fu;
    const uint32_t m_lo = w2 & 0x3F3F3F3Fu;
    const uint32_t sc_hi = (w3 & 0x0F0F0F0Fu) | ((w1 >> 2) & 0x30303030u);
    const uint32_t m_hi = ((w3 >> 4) & 0x0F0F0F0Fu) | ((w2 >> 2) & 0x30303030u);
    sc4 = H ? sc_hi : sc_lo;
    m4 = H ? m_hi : m_lo;
}

// ----------------------------------------------------------------- Q6_K

// The 6-bit quants of 4 consecutive positions l..l+3 of a Q6_K half, for
// the four 32-weight quarters t = 0..3, one per byte.  A = ql[l..l+3],
// B = ql[32+l..], Hh = qh[l..] of that half.  Quarter t takes its low 4 bits
// from A (t = 0, 2) or B (t = 1, 3), low nibble for t < 2, high nibble
// otherwise, and its top 2 bits from bits 2t..2t+1 of Hh.
__device__ __forceinline__ void q6k_build(uint32_t A, uint32_t B, uint32_t Hh, uint32_t& q0, uint32_t& q1,
                                          uint32_t& q2, uint32_t& q3) {
    q0 = (A & 0x0F0F0F0Fu) | ((Hh << 4) & 0x30303030u);
    q1 = (B & 0x0F0F0F0Fu) | ((Hh << 2) & 0x30303030u);
    q2 = ((A >> 4) & 0x0F0F0F0Fu) | (Hh & 0x30303030u);
    q3 = ((B >> 4) & 0x0F0F0F0Fu) | ((Hh >> 2) & 0x30303030u);
}

// ------------------------------------------------------ float conversion

// Float with value 1 + b/128 from a byte b|0x80 placed in bits 16..23
// (exponent byte 0x3F supplied by the constant); `sel_k` picks byte k.
__device__ __forceinline__ float magic_unit(uint32_t packed, int k) {
    return __uint_as_float(__byte_perm(packed, 0x3F000000u, 0x7054u | (static_cast<uint32_t>(k) << 8)));
}

// Float with value 2^23 + b for byte k of `packed`.
__device__ __forceinline__ float magic_2p23(uint32_t packed, int k) {
    return __uint_as_float(__byte_perm(packed, 0x4B000000u, 0x7650u | static_cast<uint32_t>(k)));
}

}  // namespace kq
