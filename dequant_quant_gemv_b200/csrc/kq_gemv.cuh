// kq_gemv.cuh — fused dequant-GEMV kernels for GGUF Q4_K / Q6_K on sm_100a.
//
// The product computed is y = W x with W dequantised only in registers
// ("Out-of-core LLM inference engine written from scratch in Rust",
// Approach: dequantisation inside fused matmul kernels; "Kortex: Streaming
// 70B Models on Consumer GPUs", Key components 3).  Decode is bound by
// weight bytes (same page, the paragraph before the first table), so the
// kernel is organised around streaming the weights once from HBM:
//
//  * One persistent CTA per SM owns a contiguous range of row pairs.  Rows
//    are contiguous in memory, so a stage (a few row pairs, ~37-54 KB) is ONE
//    1-D TMA bulk copy into a ring of shared-memory buffers, tracked by
//    mbarriers (full: transaction bytes landed; empty: consumers done).
//  * Warp 0 is the producer.  Warps 1..8 dequantise from shared memory in
//    registers.  A consumer lane owns one unit = (row pair, super-block,
//    half) = 2 x 128 weights, so the activation values it loads serve two
//    rows.  The lane->unit order makes every 16-byte shared load of a
//    quarter-warp hit distinct banks.
//  * Activations are staged once per CTA in a permuted, padded layout that
//    matches the lane's consumption order (pairs for the packed fp32 FMA).
//  * Reduction: butterfly over the lanes of a row pair, then a fixed-order
//    sum over warps.  Every output has one fixed summation order, so results
//    are bitwise reproducible and independent of the column count, the grid
//    and the stage boundaries.
//
// Quant -> float.  Q4_K low nibbles: n becomes 1 + n/128 by one byte
// permute into an exponent-0x7F float.  Q4_K high nibbles: two at a time
// become the fp16 pair (1024 + 16n, 1024 + 16n') by one mask-or, each then
// widened to fp32 (this splits the conversion work between the integer and
// the floating-point pipes, measured +5% over byte permutes alone).  The
// constant offsets (1, 1024) are removed after the dot product by
// subtracting the sub-block's activation sum (times 1024), which the
// staging pass accumulates with the very same fused-multiply-add sequence,
// so all-zero quants cancel exactly.
// Q6_K: q becomes 2^23 + q by a byte permute, then q - 32 exactly by one
// packed add.  Products and sums are fp32 (packed f32x2 FMA on sm_100a).
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {

// Packed fp32 (f32x2) fused multiply-add / add, round to nearest: one
// instruction for two independent lanes on sm_100a.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// ------------------------------------------------------------ the units

// Q4_K unit: rows r0 (and r0+1) of a row pair, super-block b, half H
// (sub-blocks 4H..4H+3, i.e. 32-byte quant chunks c = 2H and 2H+1).
// xr: the unit's activation region for column 0; column j at xr + j*xcs.
template <int NCOL>
__device__ __forceinline__ void q4k_unit(uint32_t row0, int row_bytes, int b, int H, uint32_t xr, int xcs,
                                         float (&out)[2][NCOL]) {
    // all addresses are 32-bit shared-window addresses; xcs in floats
    const uint32_t blk[2] = {row0 + b * kQ4Bytes, row0 + row_bytes + b * kQ4Bytes};
    float2 A2[2][2], NB2[2][2];  // [row][c'] (128 d sc, 16 d sc'), (-dmin m, -dmin m')
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint4 hd = ld_s128(blk[r]);
        uint32_t sc4, m4;
        q4k_half_scales(hd.y, hd.z, hd.w, H, sc4, m4);
        const float2 dd = make_float2(__half2float(__ushort_as_half(static_cast<unsigned short>(hd.x & 0xFFFFu))),
                                      __half2float(__ushort_as_half(static_cast<unsigned short>(hd.x >> 16))));
        const float2 dscale = make_float2(dd.x * 128.0f, dd.x * 0.0625f);
        const float2 nmin = make_float2(-dd.y, -dd.y);
        const float2 m23 = make_float2(-8388608.0f, -8388608.0f);
#pragma unroll
        for (int cp = 0; cp < 2; ++cp) {
            float2 scf = make_float2(magic_2p23(sc4, 2 * cp), magic_2p23(sc4, 2 * cp + 1));
            float2 mf = make_float2(magic_2p23(m4, 2 * cp), magic_2p23(m4, 2 * cp + 1));
            scf = __fadd2_rn(scf, m23);
            mf = __fadd2_rn(mf, m23);
            A2[r][cp] = __fmul2_rn(dscale, scf);
            NB2[r][cp] = __fmul2_rn(nmin, mf);
        }
    }
    float2 y2[2][NCOL];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int j = 0; j < NCOL; ++j) y2[r][j] = make_float2(0.f, 0.f);

#pragma unroll
    for (int cp = 0; cp < 2; ++cp) {
        float2 acc[2][NCOL];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int j = 0; j < NCOL; ++j) acc[r][j] = make_float2(0.f, 0.f);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int qoff = 16 + 64 * H + 32 * cp + 16 * h;
            const uint4 q0 = ld_s128(blk[0] + qoff);
            const uint4 q1 = ld_s128(blk[1] + qoff);
            const uint32_t xp = xr + 4 * ((cp * 2 + h) * 32);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint32_t w0 = u4w(q0, t), w1 = u4w(q1, t);
                const uint32_t lo0 = (w0 & 0x0F0F0F0Fu) | 0x80808080u;
                const uint32_t lo1 = (w1 & 0x0F0F0F0Fu) | 0x80808080u;
                // high nibbles as fp16 1024 + 16n (bytes 0,2 / 1,3), widened
                const uint32_t hA0 = (w0 & 0x00F000F0u) | 0x64006400u;
                const uint32_t hB0 = ((w0 >> 8) & 0x00F000F0u) | 0x64006400u;
                const uint32_t hA1 = (w1 & 0x00F000F0u) | 0x64006400u;
                const uint32_t hB1 = ((w1 >> 8) & 0x00F000F0u) | 0x64006400u;
                float4 xa[NCOL], xb[NCOL];
#pragma unroll
                for (int j = 0; j < NCOL; ++j) {
                    xa[j] = ld_s128f(xp + 4 * (j * xcs + 8 * t));
                    xb[j] = ld_s128f(xp + 4 * (j * xcs + 8 * t + 4));
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t hs0 = (k & 1) ? hB0 : hA0, hs1 = (k & 1) ? hB1 : hA1;
                    const float h0f = (k & 2) ? __high2float(*reinterpret_cast<const __half2*>(&hs0))
                                              : __low2float(*reinterpret_cast<const __half2*>(&hs0));
                    const float h1f = (k & 2) ? __high2float(*reinterpret_cast<const __half2*>(&hs1))
                                              : __low2float(*reinterpret_cast<const __half2*>(&hs1));
                    const float2 f0 = make_float2(magic_unit(lo0, k), h0f);
                    const float2 f1 = make_float2(magic_unit(lo1, k), h1f);
#pragma unroll
                    for (int j = 0; j < NCOL; ++j) {
                        const float2 xv = k == 0   ? make_float2(xa[j].x, xa[j].y)
                                          : k == 1 ? make_float2(xa[j].z, xa[j].w)
                                          : k == 2 ? make_float2(xb[j].x, xb[j].y)
                                                   : make_float2(xb[j].z, xb[j].w);
                        acc[0][j] = fma2(f0, xv, acc[0][j]);
                        acc[1][j] = fma2(f1, xv, acc[1][j]);
                    }
                }
            }
        }
#pragma unroll
        for (int j = 0; j < NCOL; ++j) {
            const float2 X2 = ld_s64f(xr + 4 * (j * xcs + 128 + 2 * cp));
            const float2 nX2 = make_float2(-X2.x, -1024.0f * X2.y);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float2 D = __fadd2_rn(acc[r][j], nX2);
                y2[r][j] = __ffma2_rn(A2[r][cp], D, y2[r][j]);
                y2[r][j] = __ffma2_rn(NB2[r][cp], X2, y2[r][j]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int j = 0; j < NCOL; ++j) out[r][j] = y2[r][j].x + y2[r][j].y;
}

// Activation sums of one Q4_K region, accumulated exactly as q4k_unit
// accumulates a chunk whose quants are all zero (factor 1.0).
__device__ __forceinline__ float2 q4k_region_sum(uint32_t xr, int cp) {
    float2 acc = make_float2(0.f, 0.f);
    const float2 one = make_float2(1.0f, 1.0f);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t xp = xr + 4 * ((cp * 2 + h) * 32);
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 xv = ld_s64f(xp + 4 * (8 * t + 2 * k));
                acc = __ffma2_rn(one, xv, acc);
            }
    }
    return acc;
}

// Q6_K unit: row pair, super-block b, half H (groups 8H..8H+7).  Blocks
// are 210 bytes, so within a 16-byte aligned row a block starts at an even
// but not necessarily 4-byte aligned offset: ODD marks blocks that start 2
// bytes past a 4-byte boundary (b odd).  The warp's blocks all share that
// class, so the branch is uniform and only two code paths exist.  Loads are
// 4-byte words; for ODD blocks each stream word is rebuilt from two loaded
// words with one byte permute.
template <int NCOL, bool ODD>
__device__ __forceinline__ void q6k_unit(uint32_t row0, int row_bytes, int b, int H, uint32_t xr, int xcs,
                                         float (&out)[2][NCOL]) {
    uint32_t QL[2][16], QH[2][8];
    float2 sA[2][2], sB[2][2];
    float dsc[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint32_t bw = row0 + r * row_bytes + b * kQ6Bytes - (ODD ? 2 : 0);  // 4-byte aligned
        auto sw = [&](int i) -> uint32_t {
            if constexpr (ODD) return __byte_perm(ld_s32(bw + 4 * i), ld_s32(bw + 4 * i + 4), 0x5432);
            else return ld_s32(bw + 4 * i);
        };
#pragma unroll
        for (int i = 0; i < 16; ++i) QL[r][i] = sw(16 * H + i);   // ql[64H .. 64H+63]
#pragma unroll
        for (int i = 0; i < 8; ++i) QH[r][i] = sw(32 + 8 * H + i);  // qh[32H .. 32H+31]
        // 8 signed scales of this half (bytes 192+8H..) as floats: flip the
        // sign bit to get s+128 as an unsigned byte, 2^23 + (s+128) by byte
        // permute, then subtract 2^23 + 128.
        const uint32_t s0 = sw(48 + 2 * H) ^ 0x80808080u;
        const uint32_t s1 = sw(49 + 2 * H) ^ 0x80808080u;
        const uint32_t dword = ODD ? (ld_s32(bw + 208) >> 16) : ld_s32(bw + 208);  // d = bytes 208..209
        const float2 off = make_float2(-8388736.0f, -8388736.0f);
        // groups: sh = 0 -> (8H+0, 8H+4) / (8H+2, 8H+6); sh = 1 -> +1
        sA[r][0] = __fadd2_rn(make_float2(magic_2p23(s0, 0), magic_2p23(s1, 0)), off);
        sA[r][1] = __fadd2_rn(make_float2(magic_2p23(s0, 1), magic_2p23(s1, 1)), off);
        sB[r][0] = __fadd2_rn(make_float2(magic_2p23(s0, 2), magic_2p23(s1, 2)), off);
        sB[r][1] = __fadd2_rn(make_float2(magic_2p23(s0, 3), magic_2p23(s1, 3)), off);
        dsc[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(dword & 0xFFFFu)));
    }
    float2 accA[2][2][NCOL], accB[2][2][NCOL];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int sh = 0; sh < 2; ++sh)
#pragma unroll
            for (int j = 0; j < NCOL; ++j) accA[r][sh][j] = accB[r][sh][j] = make_float2(0.f, 0.f);
    const float2 c32 = make_float2(-8388640.0f, -8388640.0f);  // -(2^23 + 32)
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        const int sh = s >> 2;
        uint32_t qv[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r) q6k_build(QL[r][s], QL[r][8 + s], QH[r][s], qv[r][0], qv[r][1], qv[r][2], qv[r][3]);
        const uint32_t xp = xr + 4 * (16 * s);
        float4 xa0[NCOL], xa1[NCOL], xb0[NCOL], xb1[NCOL];
#pragma unroll
        for (int j = 0; j < NCOL; ++j) {
            xa0[j] = ld_s128f(xp + 4 * (j * xcs));
            xa1[j] = ld_s128f(xp + 4 * (j * xcs + 4));
            xb0[j] = ld_s128f(xp + 4 * (j * xcs + 8));
            xb1[j] = ld_s128f(xp + 4 * (j * xcs + 12));
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float2 fA = fadd2(make_float2(magic_2p23(qv[r][0], k), magic_2p23(qv[r][2], k)), c32);
                const float2 fB = fadd2(make_float2(magic_2p23(qv[r][1], k), magic_2p23(qv[r][3], k)), c32);
#pragma unroll
                for (int j = 0; j < NCOL; ++j) {
                    const float2 xA = k == 0   ? make_float2(xa0[j].x, xa0[j].y)
                                      : k == 1 ? make_float2(xa0[j].z, xa0[j].w)
                                      : k == 2 ? make_float2(xa1[j].x, xa1[j].y)
                                               : make_float2(xa1[j].z, xa1[j].w);
                    const float2 xB = k == 0   ? make_float2(xb0[j].x, xb0[j].y)
                                      : k == 1 ? make_float2(xb0[j].z, xb0[j].w)
                                      : k == 2 ? make_float2(xb1[j].x, xb1[j].y)
                                               : make_float2(xb1[j].z, xb1[j].w);
                    accA[r][sh][j] = fma2(fA, xA, accA[r][sh][j]);
                    accB[r][sh][j] = fma2(fB, xB, accB[r][sh][j]);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int j = 0; j < NCOL; ++j) {
            float2 y2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int sh = 0; sh < 2; ++sh) {
                y2 = __ffma2_rn(sA[r][sh], accA[r][sh][j], y2);
                y2 = __ffma2_rn(sB[r][sh], accB[r][sh][j], y2);
            }
            out[r][j] = dsc[r] * (y2.x + y2.y);
        }
}

// ------------------------------------------------------- stage sequence

struct Stage {
    int64_t seg;    // segment (matrix or routed id) index
    int64_t row0;   // first row within the segment
    int nrp;        // row pairs in the stage
    int nrows;      // real rows (nrp*2, or one less at an odd tail)
};

// The CTA's stages: consecutive groups of at most `ps` row pairs of its
// range [rp, rp_end), never crossing a segment boundary.
// (One division at construction; next() only adds and compares.)  Also
// tracks the ring slot and mbarrier phase of the stage it returns.
struct StageIter {
    // 32-bit counters: a CTA's range, the row pairs of a segment (N <= 2^31
    // rows) and the segment count (an int at the ABI) all fit
    int left;            // row pairs still to hand out
    int seg, off;        // segment and row-pair offset within it
    int rps;
    int64_t N;
    int ps, ns;
    int slot = -1;       // ring slot of the last stage returned
    uint32_t phase = 0;  // its mbarrier phase parity
    int count = 0;       // stages returned so far
    __device__ StageIter(int64_t rp_begin, int64_t rp_end, int64_t rps_, int64_t N_, int ps_, int ns_)
        : left(static_cast<int>(rp_end - rp_begin)), seg(static_cast<int>(rp_begin / rps_)),
          off(static_cast<int>(rp_begin - (rp_begin / rps_) * rps_)), rps(static_cast<int>(rps_)), N(N_), ps(ps_),
          ns(ns_) {}
    __device__ bool next(Stage& st) {
        if (left <= 0) return false;
        if (off == rps) {
            ++seg;
            off = 0;
        }
        int n = left < ps ? left : ps;
        if (n > rps - off) n = rps - off;
        st.seg = seg;
        st.row0 = 2 * static_cast<int64_t>(off);
        st.nrp = n;
        const int64_t rows = N - st.row0;
        st.nrows = static_cast<int>(rows < 2 * n ? rows : 2 * n);
        off += n;
        left -= n;
        if (++slot == ns) {
            slot = 0;
            phase ^= 1u;
        }
        ++count;
        return true;
    }
};

__device__ __forceinline__ void raise_fault(const GemvArgs& a, volatile int* abort_flag, int code) {
    *abort_flag = 1;
    if (a.status) atomicExch(a.status, code);
    if (a.fault) atomicExch(a.fault, code);
}

// ------------------------------------------------------------ producer

// Ask L2 for the bytes the consumers will stage: every column's K range
// [kb0, kb0 + nbl) blocks of a shared activation copy, and the prologue's
// second operand (gamma, or the u half of [g; u]).  Issued by the producer
// at the CTA's start, before the previous grid has finished: a hint only
// (L2 is where the previous grid's writes land, so nothing stale can be
// read); the staging then reads from L2 instead of HBM.  16-byte aligned
// ranges only.
__device__ __forceinline__ void prefetch_l2(const float* p, uint32_t bytes) {
    if ((reinterpret_cast<uintptr_t>(p) & 15u) == 0)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ inline void prefetch_activations(const GemvArgs& a, int kb0, int nbl) {
    if (a.x_seg_stride != 0) return;  // one copy per segment: staged as the segments come
    const int64_t k0 = static_cast<int64_t>(kb0) * 256;
    const uint32_t bytes = static_cast<uint32_t>(nbl) * 1024u;
    for (int j = 0; j < a.ncol_real; ++j) {
        prefetch_l2(a.x + j * a.ldx + k0, bytes);
        if (a.pro == 2) prefetch_l2(a.x + j * a.ldx + a.K + k0, bytes);
    }
    if (a.pro == 1) prefetch_l2(a.gamma + k0, bytes);
}

// The producer thread: walks the CTA's stages and brings each one's rows
// into its ring slot with 1-D bulk copies (no multicast), waiting for the
// consumers to release a slot before reusing it.  `contiguous`: whole rows
// stored back to back (one copy per stage); otherwise each row's K range
// [kb0, kb0 + nbl) blocks is copied to its own smem row `srow` bytes apart,
// from the 16-byte boundary at or below the range start (bulk copies move
// whole 16-byte units), so the range begins (kb0 * BS) % 16 bytes into the
// smem row.  Rows are multiples of 16 bytes, so no copy leaves its row.
// `staged` (single-matrix kernel): after its first `lead` stages the
// producer waits until the consumers have staged the activations (they set
// *staged), so that the activation loads do not queue behind a full ring of
// weight copies; the wait is a hint and gives up after kStagedWaitNs.
constexpr unsigned long long kStagedWaitNs = 100000ull;

template <int BS>
__device__ void produce_stages(const GemvArgs& a, uint64_t* full, uint64_t* empty, volatile int* abort_flag,
                               uint8_t* sbuf, int64_t rp_begin, int64_t rp_end, int64_t rps, int ns, int kb0,
                               int nbl, int srow, bool contiguous, volatile int* staged = nullptr, int lead = 0) {
    if (a.ids) pdl_wait();  // routed ids may come from the previous grid
    const uint64_t pol = l2_evict_first();
    const unsigned long long lim = a.wait_ns && blockIdx.x == 0 ? a.wait_ns : kWaitNs;
    StageIter it(rp_begin, rp_end, rps, a.N, a.ps, ns);
    Stage st;
    RingTrack ring;
    while (it.next(st)) {
        const int slot = it.slot;
        // a reused slot: wait until the consumers released its last stage
        if (it.count > ns && !mbar_wait_bounded(&empty[slot], it.phase ^ 1u, abort_flag, lim)) {
            raise_fault(a, abort_flag, 6);
            break;
        }
        if (*abort_flag) break;  // nothing more is issued once the CTA has aborted
        if (a.test_hold && blockIdx.x == 0 && it.count == a.test_hold) {
            // test hook (kq_inject "hold@S"): this stage is never copied, so
            // the consumers' bounded wait for it runs out
            ring.skip(slot);
            continue;
        }
        int64_t e = st.seg;
        if (a.ids) e = a.ids[st.seg];
        if (e >= 0 && e < a.E) {
            const uint8_t* src = a.W + e * a.seg_stride + st.row0 * a.row_bytes;
            uint8_t* dst = sbuf + static_cast<size_t>(slot) * a.stage_bytes;
            if (contiguous) {
                // rows need not be 16-byte aligned: copy whole 16-byte units
                // from the boundary at or below the stage's first byte (the
                // consumers index from src % 16); the last unit never reaches
                // past the 16-byte granule of the stage's last byte
                const uintptr_t s0 = reinterpret_cast<uintptr_t>(src);
                const uintptr_t b0 = s0 & ~uintptr_t(15);
                const uintptr_t e0 = (s0 + static_cast<uintptr_t>(st.nrows * a.row_bytes) + 15) & ~uintptr_t(15);
                const uint32_t bytes = static_cast<uint32_t>(e0 - b0);
                mbar_arrive_expect_tx(&full[slot], bytes);
                bulk_g2s(dst, reinterpret_cast<const void*>(b0), bytes, &full[slot], pol);
            } else {
                const int64_t off = static_cast<int64_t>(kb0) * BS;
                const int64_t off16 = off & ~int64_t(15);
                const uint32_t rbytes = static_cast<uint32_t>((off + nbl * BS - off16 + 15) & ~int64_t(15));
                mbar_arrive_expect_tx(&full[slot], rbytes * st.nrows);
                for (int i = 0; i < st.nrows; ++i)
                    bulk_g2s(dst + i * srow, src + i * a.row_bytes + off16, rbytes, &full[slot], pol);
            }
            ring.issue(slot, it.phase);
        } else {
            mbar_arrive(&full[slot]);
            ring.skip(slot);
        }
        if (staged && it.count == lead) {
            const unsigned long long t0 = globaltimer_ns();
            while (!*staged && !*abort_flag && globaltimer_ns() - t0 < kStagedWaitNs) {
            }
        }
    }
    // Let every copy this CTA issued land before the CTA can exit, abort or
    // not (bounded).
    ring.drain(full, ns);
}

// ------------------------------------------------------------- prologue
//
// RMSNorm: W (x o gamma o inv) = inv * W (x o gamma), inv = 1/sqrt(sum(x^2)/K
// + eps) per column.  The staging pass applies gamma and collects partial
// sums of squares of the raw x as it loads them; after it, one warp per
// column combines the partials into inv, and the outputs are scaled by it.
// SiLU-gated product: the column holds [g; u] (2K floats) and the staging
// replaces x_i by silu(g_i) * u_i.  Both fetch their second operand (gamma,
// or u) in the same pass as x.

// Prologue scratch of the single-column kernel: per consumer group, partial
// sums of up to kProParts warps for each of 8 columns, then 8 inverse norms.
constexpr int kProParts = 16;
constexpr int kProRegion = 4 * (8 * kProParts + 8);
static_assert(2 * kProRegion <= kProBytes, "prologue scratch");
__device__ __forceinline__ uint32_t pro_inv_addr(uint32_t region) { return region + 4 * 8 * kProParts; }

// silu(g) * u with the fast exponential and division (relative error of a
// few 1e-7 for the activations' range; g -> -inf gives -0, g -> +inf g*u).
__device__ __forceinline__ float silu_gate(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Activation loads of the staging passes go to L2 only (ld.global.cg): a CTA
// of a multi-step launch may read a buffer that another CTA rewrote since
// this one last read it, and a line left in its L1 would be stale.
__device__ __forceinline__ float ld_x(const float* p) { return __ldcg(p); }

// A float4 at p, one 16-byte load when p is 16-byte aligned.
__device__ __forceinline__ float4 ld_f4(const float* p) {
    if ((reinterpret_cast<uintptr_t>(p) & 15u) == 0) return __ldcg(reinterpret_cast<const float4*>(p));
    return make_float4(ld_x(p), ld_x(p + 1), ld_x(p + 2), ld_x(p + 3));
}

// inv[c] = 1/sqrt(sum_i part[c][i] / K + eps) for the columns c < ncol from
// `count` partial sums per column, `stride` floats apart: warp c of the
// staging warps, lane l summing i = l, l + 32, ... in order, then a fixed
// butterfly; then the staging threads' barrier.  With `nbs` > 0 partial i
// lives in the shared memory of cluster rank i / nbs (the same offset).
__device__ inline void rms_finish(float K, float eps, uint32_t part, int stride, int count, uint32_t inv, int ncol,
                                  int warp, int lane, int bar, int nthr, int nbs) {
    if (warp < ncol) {
        float s = 0.f;
        for (int i = lane; i < count; i += 32) {
            const uint32_t ad = part + 4 * (warp * stride + i);
            s += nbs > 0 ? ld_cluster_f32(map_rank(ad, static_cast<uint32_t>(i / nbs))) : ld_s32f(ad);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) st_s32f(inv + 4 * warp, 1.0f / sqrtf(s / K + eps));
    }
    named_bar_sync(bar, nthr);
}

// Sum of squares of one 256-activation block held two float4 per lane (lane
// l: elements 4l..4l+3 and 128+4l..128+4l+3), in one fixed order: lane-local
// then a butterfly.  Every warp gets the same value for the same block.
__device__ __forceinline__ float block_sq(const float4& p, const float4& q) {
    float s = p.x * p.x;
    s = fmaf(p.y, p.y, s);
    s = fmaf(p.z, p.z, s);
    s = fmaf(p.w, p.w, s);
    s = fmaf(q.x, q.x, s);
    s = fmaf(q.y, q.y, s);
    s = fmaf(q.z, q.z, s);
    s = fmaf(q.w, q.w, s);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

// ------------------------------------------------------ activation stage

// Where activation i (0..256*nb-1 of a K range) of a column sits in its
// fp32 regions (a float offset; the 4 activations i..i+3 sit 2 floats apart,
// pair members alternating).
template <int FMT>
__device__ __forceinline__ int x_offset(int i, int nb) {
    const int b = i >> 8, within = i & 255;
    if constexpr (FMT == 1) {
        // weight 64c + 32*hi + 16h + 4t + k of block b -> region 2b + c/2,
        // pair (c%2, h, t, k), member hi
        const int c = within >> 6, w64 = within & 63, hi = w64 >> 5, l = w64 & 31;
        const int h = l >> 4, t = (l >> 2) & 3;
        return (2 * b + (c >> 1)) * kRegion + ((c & 1) * 2 + h) * 32 + 8 * t + hi;
    } else {
        // weight 128H + 32t + 4s + k of block b = 8i + kappa -> region
        // (kappa*nb8 + i)*2 + H; pair A = (t0, t2), pair B = (t1, t3)
        const int H = within >> 7, w128 = within & 127, t = w128 >> 5, sidx = (w128 & 31) >> 2;
        const int kappa = b & 7, ib = b >> 3;
        return ((kappa * (nb >> 3) + ib) * 2 + H) * kRegion + 16 * sidx + ((t & 1) ? 8 : 0) + (t >> 1);
    }
}

template <int FMT>
__device__ __forceinline__ void st_x4(uint32_t dst, const float4& v) {
    st_s32f(dst, v.x);
    st_s32f(dst + 8, v.y);
    st_s32f(dst + 16, v.z);
    st_s32f(dst + 24, v.w);
}

// Q4_K: the sub-block sums of each staged region (after the fill's barrier).
template <int FMT, int NCOL>
__device__ __forceinline__ void stage_x_sums(uint32_t xs, int ct, int nthr, int bar, int nbl, int xcs) {
    if constexpr (FMT == 1) {
        const int sums = NCOL * 2 * nbl * 2;
        for (int it = ct; it < sums; it += nthr) {
            const int j = it / (2 * nbl * 2);
            const int rem = it - j * 2 * nbl * 2;
            const int reg = rem >> 1, cp = rem & 1;
            const uint32_t xr = xs + 4 * (j * xcs + reg * kRegion);
            st_s64f(xr + 4 * (128 + 2 * cp), q4k_region_sum(xr, cp));
        }
        named_bar_sync(bar, nthr);
    }
}

// Stage the activations of segment `seg` (all NCOL columns) into the
// padded, permuted layout the units read, then (Q4_K) the region sums.
template <int FMT, int NCOL>
__device__ void stage_x(const GemvArgs& a, int64_t seg, uint32_t xs, int ct, int nthr, int bar, int kb0,
                        int nbl) {
    // the K range [256*kb0, 256*(kb0+nbl)) in regions laid out for a.nbs blocks
    const float* xg = a.x + seg * a.x_seg_stride + static_cast<int64_t>(kb0) * 256;
    const int nb = a.nbs;
    const int nreg = 2 * nb;
    const int xcs = nreg * kRegion;
    // fill: one item = 4 consecutive activations (a coalesced 16-byte load
    // when the column is 16-byte aligned), scattered into the region layout;
    // the 4 values land 2 floats apart (pair members alternate).
    const int k4 = nbl * 64;
    const int items = NCOL * k4;
    for (int it = ct; it < items; it += nthr) {
        const int j = it / k4;
        const int i = 4 * (it - j * k4);
        const float* xc = xg + (j < a.ncol_real ? j : a.ncol_real - 1) * a.ldx;
        float4 v;
        if ((reinterpret_cast<uintptr_t>(xc) & 15u) == 0) v = __ldcg(reinterpret_cast<const float4*>(xc + i));
        else v = make_float4(ld_x(xc + i), ld_x(xc + i + 1), ld_x(xc + i + 2), ld_x(xc + i + 3));
        st_x4<FMT>(xs + 4 * (j * xcs + x_offset<FMT>(i, nb)), v);
    }
    named_bar_sync(bar, nthr);
    stage_x_sums<FMT, NCOL>(xs, ct, nthr, bar, nbl, xcs);
}

// What the prologue staging reads, by value (the staging below is kept out
// of line, so that the kernel's main loop compiles as it does without it).
struct ProStage {
    const float* xg;   // column 0 of the segment at the K range start
    const float* gg;   // RMSNorm: gamma at the K range start
    int64_t K, ldx;
    int ncol_real, pro, nbs;
    float eps;
};

// stage_x with the prologue: the same layout, U items per thread with their
// loads (x, and gamma or u) in flight together; RMSNorm's partial sums of
// squares (raw x, per thread in item order, then a butterfly) go to
// part[column][warp], the inverse norms to pro_inv_addr(part).
template <int FMT, int NCOL>
__device__ __noinline__ void stage_x_pro(const ProStage p, uint32_t xs, int ct, int nthr, int bar, int nbl,
                                         uint32_t part) {
    constexpr int U = 4;
    const bool rms = p.pro == 1;
    const int nb = p.nbs;
    const int xcs = 2 * nb * kRegion;
    const int k4 = nbl * 64;
    const int items = NCOL * k4;
    float sq[NCOL];
#pragma unroll
    for (int j = 0; j < NCOL; ++j) sq[j] = 0.f;
    for (int it0 = ct; it0 < items; it0 += U * nthr) {
        float4 v[U], w[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int it = it0 + u * nthr;
            v[u] = w[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (it < items) {
                const int j = it / k4;
                const int i = 4 * (it - j * k4);
                const float* xc = p.xg + (j < p.ncol_real ? j : p.ncol_real - 1) * p.ldx;
                v[u] = ld_f4(xc + i);
                w[u] = ld_f4(rms ? p.gg + i : xc + p.K + i);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int it = it0 + u * nthr;
            if (it >= items) break;
            const int j = it / k4;
            const int i = 4 * (it - j * k4);
            float4 t = v[u];
            if (rms) {
                const float s = fmaf(t.w, t.w, fmaf(t.z, t.z, fmaf(t.y, t.y, t.x * t.x)));
#pragma unroll
                for (int c = 0; c < NCOL; ++c)
                    if (c == j) sq[c] += s;
                t = make_float4(t.x * w[u].x, t.y * w[u].y, t.z * w[u].z, t.w * w[u].w);
            } else {
                t = make_float4(silu_gate(t.x, w[u].x), silu_gate(t.y, w[u].y), silu_gate(t.z, w[u].z),
                                silu_gate(t.w, w[u].w));
            }
            st_x4<FMT>(xs + 4 * (j * xcs + x_offset<FMT>(i, nb)), t);
        }
    }
    if (rms) {
        const int warp = ct >> 5, lane = ct & 31;
#pragma unroll
        for (int c = 0; c < NCOL; ++c) {
            float s = sq[c];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (lane == 0) st_s32f(part + 4 * (c * kProParts + warp), s);
        }
    }
    named_bar_sync(bar, nthr);
    stage_x_sums<FMT, NCOL>(xs, ct, nthr, bar, nbl, xcs);
    if (rms)
        rms_finish(static_cast<float>(p.K), p.eps, part, kProParts, nthr >> 5, pro_inv_addr(part), p.ncol_real,
                   ct >> 5, ct & 31, bar, nthr, 0);
}

// ------------------------------- single column: the integer dot path
//
// One column of any format runs its inner products on DP4A (four byte
// products per instruction, exact int32 sums).  The activations of each
// group of 32 consecutive weights are scaled by a power of two 2^sh that
// puts the group's largest |x| in [2^13, 2^14), rounded to integers xi
// (|xi| <= 2^14) and stored as a signed high byte xi >> 8 and an unsigned
// low byte xi & 255 (xi = 256*hi + lo).  Per group the staging also keeps
// P = 2^-sh and Xg = P * sum of the xi (an exact integer sum, |sum| <=
// 2^19), and for formats whose scales cover 16 weights the integer sums of
// the group's two halves.  A sub-block's sum S of q*xi is then exact (for
// Q5_K's 5-bit codes |S| <= 31 * 32 * 2^14 < 2^24, so exact in fp32 too),
// and for Q4_K y = sum over sub-blocks of d*sc*P*S - dmin*m*Xg in fp32: the
// exact dot product of the dequantised weights with the rounded activations
// P*xi, up to fp32 rounding of the per-sub-block terms (the other formats'
// units state their own forms).  |x - P*xi| <= P/2 <= 2^-14 * (largest |x|
// of the group), so |y - y_exact| <= 2^-14 * sum over groups of
// (max_g |x|) * sum_{i in g} |w_i|.  All-zero quants with zero mins give
// y = 0 exactly.

constexpr int kXGroupBytes = 64;  // 32 high bytes, then 32 low bytes
constexpr int kXInfoBytes = 16;   // Xg, P; with S16 also the int sums of xi 0..15 and 16..31
// A region holds the 4 groups of one half super-block (its bytes, then its
// 4 info records) plus 16 bytes of padding: 336 bytes = 21 16-byte units,
// an odd count, so the regions of 8 consecutive lanes (consecutive halves
// of consecutive blocks) fall on distinct banks.
constexpr int kXRegionBytes = 4 * (kXGroupBytes + kXInfoBytes) + 16;

__device__ __forceinline__ uint32_t x_region(uint32_t xs, int b, int H) {
    return xs + kXRegionBytes * (2 * b + H);
}

// Block-parity lane order over `par` blocks (single-column Q6_K, par even):
// each parity's par/2 blocks (block pair index i, block 2i + p) take
// round_up(par, 32) lanes of their own, so that a warp never mixes the two
// alignment classes.  Within a parity the lanes come in pairs of warps over
// 32 consecutive i: lane l of the first warp takes block i = 32c + l, half
// l % 2, and lane l of the second the other half of the same block.  A
// lane's words of one kind lie at bank 9i + 8H + const (qh; ql 16H, scales
// 2H): blocks of one parity are 420 bytes = 105 words apart.  Two lanes of
// one warp with the same half are an even number 0 < |i - j| < 32 of block
// pairs apart, with different halves an odd number, so their banks differ
// by 9(i - j) or by an odd number plus an even offset: never 0 mod 32, and
// every ql, qh and scale load of a warp hits 32 distinct banks (the old
// order, two lanes per block, put lanes i and i + 8 of different halves on
// one qh bank).  A last warp without a partner
// (round_up(par, 32) / 32 odd) keeps two lanes per block, (i, half) = (l/2,
// l%2), as a lone warp of 16 blocks cannot avoid the 8-word overlap.
//
// Position of the region of block b, half H: 2b + H, or in the
// block-parity order the lane's index among the parity's active lanes after
// the previous parity's par regions (consecutive lanes read consecutive
// regions, the first warp of a pair its nc blocks' regions and then the
// second warp its nc).
__device__ __forceinline__ int x_pos(int b, int H, int par) {
    if (!par) return 2 * b + H;
    const int p = b & 1, i = b >> 1, c = i >> 5, l = i & 31;
    const int m = (par + 31) >> 5;  // warps per parity
    int d;
    if (2 * c + 1 < m) {
        const int rest = (par >> 1) - 32 * c;  // blocks of this parity from 32c
        const int nc = rest < 32 ? rest : 32;
        d = 64 * c + (((H ^ l) & 1) ? nc : 0) + l;
    } else {
        d = 64 * c + 2 * l + H;
    }
    return p * par + d;
}

// The unit of consumer thread ct in the single-column lane layout: LR lanes
// per row pair; lane u of a row pair takes block u/2, half u%2, or with the
// block-parity order (par > 0; LR = 2 round_up(par, 32)) one half of the
// row pair's lanes take its even blocks and the other half the odd ones
// (which half, alternating per 128 lanes of the group), in the warp-pair
// order above.  pos: the unit's activation region (x_pos).
struct LaneUnit {
    int rp, b, H, pos;
    bool active;
};
__device__ __forceinline__ LaneUnit lane_unit(int ct, int LR, int nbl, int par) {
    LaneUnit L;
    L.rp = ct / LR;
    const int u = ct - L.rp * LR;
    if (par) {
        const int LRp = LR >> 1;
        const int hi = u >= LRp ? 1 : 0;
        const int up = u - hi * LRp;
        // the parity of the lanes' blocks, swapped for every other 128
        // lanes of the group: the warps of a row pair alternate between the
        // 4 schedulers (warp w on w % 4), and odd blocks cost more (their
        // words are realigned), so each scheduler gets both kinds
        const int p = hi ^ (((L.rp * LR) >> 7) & 1);
        const int w = up >> 5, l = up & 31, c = w >> 1;
        int i;
        if ((w | 1) < (LRp >> 5)) {  // a warp of a pair
            i = 32 * c + l;
            L.H = (l ^ w) & 1;
        } else {
            i = 32 * c + (l >> 1);
            L.H = l & 1;
        }
        L.b = 2 * i + p;
        L.active = L.b < nbl;
        L.pos = x_pos(L.b, L.H, par);
    } else {
        L.b = u >> 1;
        L.H = u & 1;
        L.active = u < 2 * nbl;
        L.pos = u;
    }
    return L;
}

// Stage the K range [256*kb0, 256*(kb0+nbl)) of segment `seg` as above,
// into the regions at `xs` (positions by x_pos).  A warp takes 4 groups of 32 activations (one
// region) per pass: lane l holds 4 consecutive values of group l / 8, loaded
// as one float4; a group's largest |x| and the sum of its xi are butterflies
// over its 8 lanes, and each lane writes its 4 high and 4 low bytes as one
// word each.  U passes' loads in flight.  PRO: with the prologue a.pro, its
// second operand (gamma, or u) loaded beside x; RMSNorm's partial sums of
// squares (raw x, per lane, then a butterfly) go to part[0][warp] and the
// inverse norm to pro_inv_addr(part).  S16: the info record also holds the
// integer sums of the group's first and last 16 xi (for formats whose
// scales and offsets cover 16 weights).
template <bool PRO, bool S16 = false>
__device__ inline void stage_x_int(const GemvArgs& a, int64_t seg, uint32_t xs, int warp, int nwarps, int lane,
                                   int bar, int nthr, int kb0, int nbl, uint32_t part, int par = 0) {
    constexpr int U = PRO ? 4 : 8;  // one round of loads for K up to 16384 (8 with a prologue) and 16 warps
    const float* xg = a.x + seg * a.x_seg_stride + static_cast<int64_t>(kb0) * 256;
    const int quads = 2 * nbl;  // passes of 4 groups (128 activations)
    const bool rms = PRO && a.pro == 1;
    const float* sg = PRO ? (rms ? a.gamma + static_cast<int64_t>(kb0) * 256 : xg + a.K) : nullptr;
    const int sub = lane >> 3;     // the lane's group within the pass
    const int e = 4 * (lane & 7);  // its first position in the group
    float sq = 0.f;
    for (int base = warp; base < quads; base += nwarps * U) {
        float4 v[U], w[U];
        // the region positions of the U passes loaded together here, in the
        // block-parity order: one pass per lane (lane u: pass u), then
        // broadcast per pass
        int pos_l = 0;
        if (par) {
            const int Ql = base + nwarps * (lane & (U - 1));
            pos_l = x_pos(Ql >> 1, Ql & 1, par);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int Q = base + nwarps * u;
            const int off = 128 * Q + 32 * sub + e;
            v[u] = Q < quads ? ld_f4(xg + off) : make_float4(0.f, 0.f, 0.f, 0.f);
            if constexpr (PRO) w[u] = Q < quads ? ld_f4(sg + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if constexpr (PRO) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (rms) {
                    sq = fmaf(v[u].x, v[u].x, sq);
                    sq = fmaf(v[u].y, v[u].y, sq);
                    sq = fmaf(v[u].z, v[u].z, sq);
                    sq = fmaf(v[u].w, v[u].w, sq);
                    v[u] = make_float4(v[u].x * w[u].x, v[u].y * w[u].y, v[u].z * w[u].z, v[u].w * w[u].w);
                } else {
                    v[u] = make_float4(silu_gate(v[u].x, w[u].x), silu_gate(v[u].y, w[u].y),
                                       silu_gate(v[u].z, w[u].z), silu_gate(v[u].w, w[u].w));
                }
            }
        }
        // the passes advance two at a time in lockstep (a pair past the end
        // is skipped; a pass past the end inside a pair works on zeros and
        // stores nothing), so that their shuffle and conversion latencies
        // overlap
#pragma unroll
        for (int c = 0; c < U; c += 2) {
            if (base + nwarps * c >= quads) break;  // warp-uniform
            float m[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float4 w4 = v[c + u];
                m[u] = fmaxf(fmaxf(fabsf(w4.x), fabsf(w4.y)), fmaxf(fabsf(w4.z), fabsf(w4.w)));
            }
#pragma unroll
            for (int off = 1; off <= 4; off <<= 1)
#pragma unroll
                for (int u = 0; u < 2; ++u) m[u] = fmaxf(m[u], __shfl_xor_sync(0xffffffffu, m[u], off));
            int sh[2], t[2], first[2];
            uint32_t hb[2], lb[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t mb = __float_as_uint(m[u]);
                int ex = 0;
                if (mb != 0u) {
                    ex = 13 - (static_cast<int>(mb >> 23) - 127);
                    ex = ex > 100 ? 100 : ex < -100 ? -100 : ex;
                }
                sh[u] = ex;
                const float sc = __int_as_float((ex + 127) << 23);
                const float4 w4 = v[c + u];
                const int x0 = __float2int_rn(w4.x * sc), x1 = __float2int_rn(w4.y * sc);
                const int x2 = __float2int_rn(w4.z * sc), x3 = __float2int_rn(w4.w * sc);
                t[u] = (x0 + x1) + (x2 + x3);
                // byte 1 of each xi (the signed high byte), then byte 0
                hb[u] = __byte_perm(__byte_perm(x0, x1, 0x0051u), __byte_perm(x2, x3, 0x0051u), 0x5410u);
                lb[u] = __byte_perm(__byte_perm(x0, x1, 0x0040u), __byte_perm(x2, x3, 0x0040u), 0x5410u);
            }
#pragma unroll
            for (int off = 1; off <= 4; off <<= 1) {
#pragma unroll
                for (int u = 0; u < 2; ++u) t[u] += __shfl_xor_sync(0xffffffffu, t[u], off);
                if (off == 2) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) first[u] = t[u];  // on lanes 0..3 of a group: its first 16
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int Q = base + nwarps * (c + u);
                if (Q >= quads) break;  // warp-uniform
                const int pos = par ? __shfl_sync(0xffffffffu, pos_l, c + u) : Q;
                const uint32_t xr = xs + kXRegionBytes * pos;
                asm volatile("st.shared.u32 [%0], %1;" ::"r"(xr + kXGroupBytes * sub + e), "r"(hb[u]) : "memory");
                asm volatile("st.shared.u32 [%0], %1;" ::"r"(xr + kXGroupBytes * sub + 32 + e), "r"(lb[u])
                             : "memory");
                if ((lane & 7) == 0) {
                    const float X = static_cast<float>(t[u]) * __int_as_float((127 - sh[u]) << 23);
                    const uint32_t ir = xr + 4 * kXGroupBytes + kXInfoBytes * sub;
                    if constexpr (S16) {
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ir), "r"(__float_as_uint(X)),
                                     "r"(static_cast<uint32_t>((127 - sh[u]) << 23)), "r"(first[u]),
                                     "r"(t[u] - first[u])
                                     : "memory");
                    } else {
                        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(ir), "r"(__float_as_uint(X)),
                                     "r"(static_cast<uint32_t>((127 - sh[u]) << 23))
                                     : "memory");
                    }
                }
            }
        }
    }
    if (rms) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
        if (lane == 0) st_s32f(part + 4 * warp, sq);
    }
    named_bar_sync(bar, nthr);
    if (rms)
        rms_finish(static_cast<float>(a.K), a.eps, part, kProParts, nwarps, pro_inv_addr(part), 1, warp, lane, bar,
                   nthr, 0);
}

__device__ __forceinline__ float byte_f(uint32_t w, int k) { return static_cast<float>((w >> (8 * k)) & 0xFFu); }

// Q4_K unit, one column: row pair at row0 (rows row_bytes apart), super-block
// b, half H (sub-blocks 4H..4H+3).  Chunk c = 2H + cc holds sub-block 2c in
// its low nibbles (x group 8b + 2c) and 2c+1 in its high nibbles.
__device__ __forceinline__ void q4k_unit_int(uint32_t row0, int row_bytes, int b, int H, uint32_t xr,
                                             float (&out)[2][1]) {
    const uint32_t blk[2] = {row0 + b * kQ4Bytes, row0 + row_bytes + b * kQ4Bytes};
    float dd[2], dm[2];
    uint32_t sc4[2], m4[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint4 hd = ld_s128(blk[r]);
        q4k_half_scales(hd.y, hd.z, hd.w, H, sc4[r], m4[r]);
        dd[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(hd.x & 0xFFFFu)));
        dm[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(hd.x >> 16)));
    }
    float y[2] = {0.f, 0.f};
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * H + cc;
        const uint32_t gL = xr + kXGroupBytes * (2 * cc), gH = gL + kXGroupBytes;  // groups 2cc, 2cc+1 of the half
        int hL[2] = {0, 0}, hH[2] = {0, 0};
        uint32_t lL[2] = {0u, 0u}, lH[2] = {0u, 0u};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 q0 = ld_s128(blk[0] + 16 + 32 * c + 16 * h), q1 = ld_s128(blk[1] + 16 + 32 * c + 16 * h);
            const uint4 xhL = ld_s128(gL + 16 * h), xlL = ld_s128(gL + 32 + 16 * h);
            const uint4 xhH = ld_s128(gH + 16 * h), xlH = ld_s128(gH + 32 + 16 * h);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const uint32_t w = u4w(r ? q1 : q0, t);
                    // high nibbles in place: 16*q, the 1/16 folded into the scale
                    const uint32_t lo = w & 0x0F0F0F0Fu, hi = w & 0xF0F0F0F0u;
                    hL[r] = dp4a_us(lo, u4w(xhL, t), hL[r]);
                    lL[r] = dp4a_uu(lo, u4w(xlL, t), lL[r]);
                    hH[r] = dp4a_us(hi, u4w(xhH, t), hH[r]);
                    lH[r] = dp4a_uu(hi, u4w(xlH, t), lH[r]);
                }
            }
        }
        const float4 iL = ld_s128f(xr + 4 * kXGroupBytes + kXInfoBytes * (2 * cc));
        const float4 iH = ld_s128f(xr + 4 * kXGroupBytes + kXInfoBytes * (2 * cc + 1));
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const float sL = static_cast<float>(hL[r] * 256 + static_cast<int>(lL[r]));
            const float sH = static_cast<float>(hH[r] * 256 + static_cast<int>(lH[r]));
            y[r] = fmaf(dd[r] * byte_f(sc4[r], 2 * cc) * iL.y, sL, y[r]);
            y[r] = fmaf(-dm[r] * byte_f(m4[r], 2 * cc), iL.x, y[r]);
            y[r] = fmaf(dd[r] * byte_f(sc4[r], 2 * cc + 1) * (iH.y * 0.0625f), sH, y[r]);
            y[r] = fmaf(-dm[r] * byte_f(m4[r], 2 * cc + 1), iH.x, y[r]);
        }
    }
    out[0][0] = y[0];
    out[1][0] = y[1];
}

// Q5_K unit, one column, on DP4A: as q4k_unit_int, with each code's 5th bit
// merged in.  Bytes: header 0..15 (as Q4_K), qh 16..47, quants 48..175.
// Weight 64c+l takes bit 2c of qh[l] (low nibble) and 64c+32+l bit 2c+1
// (high nibble); the lane's 16-byte half h of a chunk covers l = 16h..16h+15,
// so one 16-byte load of qh serves both of its chunks.
__device__ __forceinline__ void q5k_unit_int(uint32_t row0, int row_bytes, int b, int H, uint32_t xr,
                                             float (&out)[2][1]) {
    const uint32_t blk[2] = {row0 + b * kQ5Bytes, row0 + row_bytes + b * kQ5Bytes};
    float dd[2], dm[2];
    uint32_t sc4[2], m4[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint4 hd = ld_s128(blk[r]);
        q4k_half_scales(hd.y, hd.z, hd.w, H, sc4[r], m4[r]);
        dd[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(hd.x & 0xFFFFu)));
        dm[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(hd.x >> 16)));
    }
    float y[2] = {0.f, 0.f};
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * H + cc;
        const uint32_t gL = xr + kXGroupBytes * (2 * cc), gH = gL + kXGroupBytes;  // groups 2cc, 2cc+1 of the half
        int hL[2] = {0, 0}, hH[2] = {0, 0};
        uint32_t lL[2] = {0u, 0u}, lH[2] = {0u, 0u};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 q0 = ld_s128(blk[0] + 48 + 32 * c + 16 * h), q1 = ld_s128(blk[1] + 48 + 32 * c + 16 * h);
            const uint4 e0 = ld_s128(blk[0] + 16 + 16 * h), e1 = ld_s128(blk[1] + 16 + 16 * h);
            const uint4 xhL = ld_s128(gL + 16 * h), xlL = ld_s128(gL + 32 + 16 * h);
            const uint4 xhH = ld_s128(gH + 16 * h), xlH = ld_s128(gH + 32 + 16 * h);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const uint32_t w = u4w(r ? q1 : q0, t), e = u4w(r ? e1 : e0, t);
                    const uint32_t lo = (w & 0x0F0F0F0Fu) | (((e >> (2 * c)) & 0x01010101u) << 4);
                    const uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) | (((e >> (2 * c + 1)) & 0x01010101u) << 4);
                    hL[r] = dp4a_us(lo, u4w(xhL, t), hL[r]);
                    lL[r] = dp4a_uu(lo, u4w(xlL, t), lL[r]);
                    hH[r] = dp4a_us(hi, u4w(xhH, t), hH[r]);
                    lH[r] = dp4a_uu(hi, u4w(xlH, t), lH[r]);
                }
            }
        }
        const float4 iL = ld_s128f(xr + 4 * kXGroupBytes + kXInfoBytes * (2 * cc));
        const float4 iH = ld_s128f(xr + 4 * kXGroupBytes + kXInfoBytes * (2 * cc + 1));
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const float sL = static_cast<float>(hL[r] * 256 + static_cast<int>(lL[r]));
            const float sH = static_cast<float>(hH[r] * 256 + static_cast<int>(lH[r]));
            y[r] = fmaf(dd[r] * byte_f(sc4[r], 2 * cc) * iL.y, sL, y[r]);
            y[r] = fmaf(-dm[r] * byte_f(m4[r], 2 * cc), iL.x, y[r]);
            y[r] = fmaf(dd[r] * byte_f(sc4[r], 2 * cc + 1) * iH.y, sH, y[r]);
            y[r] = fmaf(-dm[r] * byte_f(m4[r], 2 * cc + 1), iH.x, y[r]);
        }
    }
    out[0][0] = y[0];
    out[1][0] = y[1];
}

// Q2_K unit, one column, on DP4A: row pair at row0, super-block b (84
// bytes: 16 scale|min bytes, 64 quant bytes, d, dmin; 4-byte aligned), half
// H.  Weight 128H + 32j + l is bits 2j of quant byte 32H + l, in 16-weight
// group 8H + 2j + l/16.  The codes of plane j are used in place (4^j * q,
// no shift), the 4^-j folded into the group's factor.  Per group the exact
// S = sum q*xi, then y += d*sc*P*S - dmin*m*P*(the group's 16-sum of xi).
__device__ __forceinline__ void q2k_unit_int(uint32_t row0, int row_bytes, int b, int H, uint32_t xr,
                                             float (&out)[2][1]) {
    uint32_t Q[2][8], sw[2][2];
    float dd[2], dm[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint32_t blk = row0 + r * row_bytes + b * kQ2Bytes;
#pragma unroll
        for (int t = 0; t < 8; ++t) Q[r][t] = ld_s32(blk + 16 + 32 * H + 4 * t);
        sw[r][0] = ld_s32(blk + 8 * H);
        sw[r][1] = ld_s32(blk + 8 * H + 4);
        const uint32_t dw = ld_s32(blk + 80);
        dd[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(dw & 0xFFFFu)));
        dm[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(dw >> 16)));
    }
    // per 32-group j and row: the exact int32 sums sc*S and m*(16-sum) of
    // its two 16-groups (|.| < 2^31), folded into fp32 once per j
    float yd[2] = {0.f, 0.f}, ym[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 info = ld_s128(xr + 4 * kXGroupBytes + kXInfoBytes * j);  // X, P, 16-sums
        const float P = __uint_as_float(info.y);
        const float Pj = P * (1.0f / static_cast<float>(1 << (2 * j)));  // undoes the 4^j of the in-place codes
        int isum[2] = {0, 0}, msum[2] = {0, 0};
#pragma unroll
        for (int sh = 0; sh < 2; ++sh) {
            const uint4 xh = ld_s128(xr + kXGroupBytes * j + 16 * sh);
            const uint4 xl = ld_s128(xr + kXGroupBytes * j + 32 + 16 * sh);
            int hi[2] = {0, 0};
            uint32_t lo[2] = {0u, 0u};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const uint32_t q = Q[r][4 * sh + m] & (0x03030303u << (2 * j));  // 4^j * q
                    hi[r] = dp4a_us(q, u4w(xh, m), hi[r]);
                    lo[r] = dp4a_uu(q, u4w(xl, m), lo[r]);
                }
            }
            const int x16 = static_cast<int>(sh ? info.w : info.z);
            const int g = 2 * j + sh;  // group within the half
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int sb = static_cast<int>((sw[r][g >> 2] >> (8 * (g & 3))) & 0xFFu);
                isum[r] += (sb & 15) * (hi[r] * 256 + static_cast<int>(lo[r]));
                msum[r] += (sb >> 4) * x16;
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            yd[r] = fmaf(Pj, static_cast<float>(isum[r]), yd[r]);
            ym[r] = fmaf(P, static_cast<float>(msum[r]), ym[r]);
        }
    }
    out[0][0] = dd[0] * yd[0] - dm[0] * ym[0];
    out[1][0] = dd[1] * yd[1] - dm[1] * ym[1];
}

// Q3_K unit, one column, on DP4A: row pair at row0, super-block b (110
// bytes: hmask[32], 64 quant bytes, 12 scale bytes, d), half H.  Blocks are
// 2-byte aligned only and the parity of b varies across the lanes, so each
// stream of words is loaded from the 4-byte aligned address at or below
// its start (one word more than it needs) and every word rebuilt by a byte
// permute whose selector is picked by b's parity.  Weight 128H + 32j + l:
// q + 4 = (bits 2j of quant byte 32H + l) | (bit 4H + j of hmask[l]) << 2,
// in 0..7, assembled in place as 4^jj * (q + 4) with jj = min(j, 2) (the
// 4^-jj folded into the group's factor).  Per 16-weight group the exact
// S = sum (q+4)*xi - 4*(16-sum of xi); per 32-group the int32 sum of
// (v - 32)*S over its two groups (|.| < 2^31, v the 6-bit scale); y = d *
// sum over 32-groups of P*(that sum), in fp32.
__device__ __forceinline__ void q3k_unit_int(uint32_t row0, int row_bytes, int b, int H, uint32_t xr,
                                             float (&out)[2][1]) {
    uint32_t Q[2][8], M[2][8], sc[2][2], hs[2];
    float dd[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        // the block's alignment class, read off its address (per row)
        const uint32_t addr = row0 + r * row_bytes + b * kQ3Bytes;
        const bool odd = (addr & 2u) != 0;
        const uint32_t sel = odd ? 0x5432u : 0x3210u;
        const uint32_t bw = addr - (odd ? 2u : 0u);  // 4-byte aligned
        uint32_t L[9];
#pragma unroll
        for (int t = 0; t < 9; ++t) L[t] = ld_s32(bw + 32 + 32 * H + 4 * t);
#pragma unroll
        for (int t = 0; t < 8; ++t) Q[r][t] = __byte_perm(L[t], L[t + 1], sel);
#pragma unroll
        for (int t = 0; t < 9; ++t) L[t] = ld_s32(bw + 4 * t);
#pragma unroll
        for (int t = 0; t < 8; ++t) M[r][t] = __byte_perm(L[t], L[t + 1], sel);
#pragma unroll
        for (int t = 0; t < 4; ++t) L[t] = ld_s32(bw + 96 + 4 * t);
        // the half's 8 groups: low 4 bits from scale bytes 0..7 (nibble H),
        // high 2 bits from bytes 8..11 (bits 2(g/4)+4H .. of byte 8 + g%4)
        sc[r][0] = (__byte_perm(L[0], L[1], sel) >> (4 * H)) & 0x0F0F0F0Fu;
        sc[r][1] = (__byte_perm(L[1], L[2], sel) >> (4 * H)) & 0x0F0F0F0Fu;
        hs[r] = __byte_perm(L[2], L[3], sel) >> (4 * H);
        dd[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(L[3] >> (odd ? 16 : 0))));
    }
    // per 32-group j and row: the exact int32 sum of (v - 32)*S over its two
    // 16-groups (|.| < 2^31), folded into fp32 once per j
    float y[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 info = ld_s128(xr + 4 * kXGroupBytes + kXInfoBytes * j);  // X, P, 16-sums
        const int jj = j < 3 ? j : 2;  // the plane's codes sit at bits 2jj..2jj+2
        const float Pj = __uint_as_float(info.y) * (1.0f / static_cast<float>(1 << (2 * jj)));
        int isum[2] = {0, 0};
#pragma unroll
        for (int sh = 0; sh < 2; ++sh) {
            const uint4 xh = ld_s128(xr + kXGroupBytes * j + 16 * sh);
            const uint4 xl = ld_s128(xr + kXGroupBytes * j + 32 + 16 * sh);
            int hi[2] = {0, 0};
            uint32_t lo[2] = {0u, 0u};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int t = 4 * sh + m;
                    // 4^jj * (q + 4): the low bits in place (plane 3 moved down to
                    // plane 2's bits, so that the three bits fit a byte), the third
                    // bit rotated next to them (a rotation keeps each byte's bit
                    // 4H + j inside its byte)
                    const uint32_t lowb = j < 3 ? Q[r][t] : Q[r][t] >> 2;
                    const uint32_t hb = __funnelshift_l(M[r][t], M[r][t], (2 * jj + 2 - 4 * H - j) & 31);
                    const uint32_t q = (lowb & (0x03030303u << (2 * jj))) | (hb & (0x04040404u << (2 * jj)));
                    hi[r] = dp4a_us(q, u4w(xh, m), hi[r]);
                    lo[r] = dp4a_uu(q, u4w(xl, m), lo[r]);
                }
            }
            const int x16 = static_cast<int>(sh ? info.w : info.z) << (2 * jj);
            const int g = 2 * j + sh;  // group within the half
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t lo4 = (sc[r][g >> 2] >> (8 * (g & 3))) & 15u;
                const uint32_t hi2 = (hs[r] >> (8 * (g & 3) + 2 * (g >> 2))) & 3u;
                const int v = static_cast<int>(lo4 | (hi2 << 4)) - 32;
                isum[r] += v * (hi[r] * 256 + static_cast<int>(lo[r]) - 4 * x16);
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) y[r] = fmaf(Pj, static_cast<float>(isum[r]), y[r]);
    }
    out[0][0] = dd[0] * y[0];
    out[1][0] = dd[1] * y[1];
}

// Q8_0 unit, one column, on DP4A: row pair at row0, unit b of eight
// 34-byte blocks (272 bytes, 256 weights), half H = blocks 4H..4H+3 (136
// bytes from an 8-byte boundary).  Block k of the half (weights 128H + 32k +
// l, activation group k of the region) starts at byte 34k: fp16 d, then 32
// int8 quants.  Blocks 0 and 2 start on a 4-byte boundary (their quant
// words are rebuilt from two loaded words by a byte permute), blocks 1 and
// 3 two bytes past one (their quant words are aligned).  The half is read as
// two runs of 18 words (8-byte loads), one per pair of blocks.  Per block
// the exact int32 S = sum q*xi (|S| <= 2^26) and y += d*P*S.
__device__ __forceinline__ void q80_unit_int(uint32_t row0, int row_bytes, int b, int H, uint32_t xr,
                                             float (&out)[2][1]) {
    float y[2] = {0.f, 0.f};
#pragma unroll
    for (int p = 0; p < 2; ++p) {  // blocks 2p and 2p+1: bytes 68p .. 68p+67 of the half
        uint32_t Wd[2][18];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint32_t base = row0 + r * row_bytes + b * kQ80Bytes + 136 * H + 64 * p;  // 8-byte aligned
#pragma unroll
            for (int i = 0; i < 9; ++i) {
                const uint2 v = ld_s2w(base + 8 * i);
                Wd[r][2 * i] = v.x;
                Wd[r][2 * i + 1] = v.y;
            }
        }
        // block 2p starts at word p (byte 4p of the run), block 2p+1 at byte
        // 34 + 4p: word 8 + p, two bytes in
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int k = 2 * p + kk;
            const uint4 info = ld_s128(xr + 4 * kXGroupBytes + kXInfoBytes * k);  // X, P
            const float P = __uint_as_float(info.y);
            int hi[2] = {0, 0}, lo[2] = {0, 0};
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const uint4 xh = ld_s128(xr + kXGroupBytes * k + 16 * s);
                const uint4 xl = ld_s128(xr + kXGroupBytes * k + 32 + 16 * s);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int i = 4 * s + m;  // quant word i of the block
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const uint32_t q = kk == 0 ? __byte_perm(Wd[r][p + i], Wd[r][p + i + 1], 0x5432u)
                                                   : Wd[r][9 + p + i];
                        hi[r] = dp4a_ss(q, u4w(xh, m), hi[r]);
                        lo[r] = dp4a_su(q, u4w(xl, m), lo[r]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t dw = kk == 0 ? (Wd[r][p] & 0xFFFFu) : (Wd[r][8 + p] >> 16);
                const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(dw)));
                const int S = hi[r] * 256 + lo[r];
                y[r] = fmaf(d * P, static_cast<float>(S), y[r]);
            }
        }
    }
    out[0][0] = y[0];
    out[1][0] = y[1];
}

// Q6_K unit, one column, on DP4A: row pair at row0, super-block b (210
// bytes: ql[128], qh[64], 16 int8 scales, d), half H.  Blocks are 2-byte
// aligned only: a block at an even index of a 16-byte aligned row starts on
// a 4-byte boundary, one at an odd index 2 bytes past one (rows whose
// length is not a multiple of 16 bytes shift this per row).  ODD = 0: an
// aligned block, its words loaded as they are; ODD = 1: each stream is
// loaded from the 4-byte boundary below its start, one word more than it
// needs, and every word rebuilt by a byte permute; ODD = 2: the class is
// read off each row's block address (the lanes of a warp mix both; the
// extra word is the block's own or its neighbour's bytes, or at the end of
// a stage the slot's slack).  Weight 128H + 32t + l: low 4 bits from ql[64H + 32(t%2) + l]
// (nibble t/2), top 2 bits from bits 2t of qh[32H + l]; 16-weight group
// 2t + l/16 of the half has scale s = scales[8H + 2t + l/16].  Per group the
// exact S = sum q*xi - 32*(its 16-sum of xi) = sum (q - 32)*xi, |S| <= 2^23,
// and T = s*S (|T| <= 2^30, an exact int32); y = d * sum over groups of
// P*T in fp32.
template <int ODD>
__device__ __forceinline__ void q6k_unit_int(uint32_t row0, int row_bytes, int b, int H, uint32_t xr,
                                             float (&out)[2][1]) {
    // each row's alignment class: fixed by ODD, or (ODD == 2) read off the
    // block's shared-memory address, which also covers rows whose length is
    // not a multiple of 4 bytes (the two rows of a pair then differ)
    bool odd[2];
    uint32_t sel[2], bw[2], sc[2][2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint32_t addr = row0 + r * row_bytes + b * kQ6Bytes;
        odd[r] = ODD == 2 ? (addr & 2u) != 0 : ODD == 1;
        sel[r] = odd[r] ? 0x5432u : 0x3210u;
        bw[r] = addr - (odd[r] ? 2u : 0u);  // 4-byte aligned
    }
    // the 4 words at base (4-byte aligned) of a stream of row r starting at
    // base + 2*odd[r]
    auto words = [&](int r, uint32_t base, uint32_t (&w)[4]) {
        if constexpr (ODD == 0) {
#pragma unroll
            for (int m = 0; m < 4; ++m) w[m] = ld_s32(base + 4 * m);
        } else {
            uint32_t L[5];
#pragma unroll
            for (int k = 0; k < 5; ++k) L[k] = ld_s32(base + 4 * k);
#pragma unroll
            for (int m = 0; m < 4; ++m) w[m] = __byte_perm(L[m], L[m + 1], sel[r]);
        }
    };
    float dd[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (ODD == 0) {
            sc[r][0] = ld_s32(bw[r] + 192 + 8 * H);
            sc[r][1] = ld_s32(bw[r] + 196 + 8 * H);
        } else {
            const uint32_t s0 = ld_s32(bw[r] + 192 + 8 * H), s1 = ld_s32(bw[r] + 196 + 8 * H),
                           s2 = ld_s32(bw[r] + 200 + 8 * H);
            sc[r][0] = __byte_perm(s0, s1, sel[r]);
            sc[r][1] = __byte_perm(s1, s2, sel[r]);
        }
        dd[r] = __half2float(
            __ushort_as_half(static_cast<unsigned short>(ld_s32(bw[r] + 208) >> (odd[r] ? 16 : 0))));
    }
    // the half's 4 groups: P and 32 times the integer sums of their two
    // 16-weight halves (loaded once for both s)
    float Pg[4];
    uint32_t x32[4][2];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const uint4 info = ld_s128(xr + 4 * kXGroupBytes + kXInfoBytes * t);  // X, P, 16-sums
        Pg[t] = __uint_as_float(info.y);
        x32[t][0] = 32u * info.z;
        x32[t][1] = 32u * info.w;
    }
    float y[2] = {0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        // positions l = 16s .. 16s+15: words of ql (A: t = 0, 2; B: t = 1, 3) and qh
        uint32_t A[2][4], B[2][4], Hh[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            words(r, bw[r] + 64 * H + 16 * s, A[r]);
            words(r, bw[r] + 64 * H + 32 + 16 * s, B[r]);
            words(r, bw[r] + 128 + 32 * H + 16 * s, Hh[r]);
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const uint4 xh = ld_s128(xr + kXGroupBytes * t + 16 * s);
            const uint4 xl = ld_s128(xr + kXGroupBytes * t + 32 + 16 * s);
            // the low-byte sums start at -32 * (16-sum of xi), mod 2^32: the
            // exact int32 S = 256*hi + lo - 32*sum below (|each| < 2^31)
            int hi[2] = {0, 0};
            uint32_t lo[2] = {0u - x32[t][s], 0u - x32[t][s]};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const uint32_t src = (t & 1) ? B[r][m] : A[r][m];
                    const uint32_t low = ((t & 2) ? (src >> 4) : src) & 0x0F0F0F0Fu;
                    const uint32_t top = t == 0 ? (Hh[r][m] << 4) : t == 1 ? (Hh[r][m] << 2)
                                                      : t == 2 ? Hh[r][m] : (Hh[r][m] >> 2);
                    const uint32_t q = low | (top & 0x30303030u);
                    hi[r] = dp4a_us(q, u4w(xh, m), hi[r]);
                    lo[r] = dp4a_uu(q, u4w(xl, m), lo[r]);
                }
            }
            const int g = 2 * t + s;  // group within the half
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int S = hi[r] * 256 + static_cast<int>(lo[r]);
                const int sv = sext_byte(sc[r][g >> 2], g & 3);  // the group's int8 scale
                y[r] = fmaf(Pg[t], static_cast<float>(sv * S), y[r]);
            }
        }
    }
    out[0][0] = y[0] * dd[0];
    out[1][0] = y[1] * dd[1];
}

// Dispatch a Q6_K unit to the code path of its alignment class.
template <int NCOL>
__device__ __forceinline__ void q6k_unit_dispatch(int kappa, uint32_t row0, int row_bytes, int b, int H,
                                                  uint32_t xr, int xcs, float (&out)[2][NCOL]) {
    if (kappa & 1) q6k_unit<NCOL, true>(row0, row_bytes, b, H, xr, xcs, out);
    else q6k_unit<NCOL, false>(row0, row_bytes, b, H, xr, xcs, out);
}

// Stage a segment's activations for the kernel below: threads ct of nthr
// (whole warps), integer regions (INT) or fp32 regions, with or without the
// prologue (PRO).
// PAR: the launch may use the block-parity region order (a.par; only
// single-column Q6_K), otherwise the regions are in plain order at compile time.
template <int FMT, int NCOL, bool INT, bool PRO, bool PAR = (FMT == 2)>
__device__ __forceinline__ void stage_all(const GemvArgs& a, int64_t seg, uint32_t xs, int ct, int nthr, int bar,
                                          int kb0, int nbl, uint32_t part) {
    if constexpr (INT)
        stage_x_int<PRO, (FMT == 2 || FMT == 4 || FMT == 5)>(a, seg, xs, ct >> 5, nthr >> 5, ct & 31, bar, nthr, kb0,
                                                             nbl, part, PAR ? a.par : 0);
    else if constexpr (PRO)
        stage_x_pro<FMT, NCOL>(ProStage{a.x + seg * a.x_seg_stride + static_cast<int64_t>(kb0) * 256,
                                        a.pro == 1 ? a.gamma + static_cast<int64_t>(kb0) * 256 : nullptr, a.K, a.ldx,
                                        a.ncol_real, a.pro, a.nbs, a.eps},
                               xs, ct, nthr, bar, nbl, part);
    else stage_x<FMT, NCOL>(a, seg, xs, ct, nthr, bar, kb0, nbl);
}

// ------------------------------------------------------------ the kernel

// NG consumer groups of 8 warps each: group g consumes the stages whose
// index is g mod NG, so two groups work on consecutive stages of one ring
// while the producer keeps filling it (more warps per SM to hide shared-memory
// latency, one activation copy, a deeper ring than two CTAs could hold).
// PRO: the instantiation that applies the prologue a.pro while staging
// (kept apart so that the plain kernel carries none of its code).
template <int FMT, int NCOL, int NG, bool PRO>
__global__ void __launch_bounds__(32 + NG * kConsumers, 1) gemv_kernel(const __grid_constant__ GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 2 * kMaxStages * 8);
    float* wp = reinterpret_cast<float*>(smem + a.wp_offset);
    float* xs = reinterpret_cast<float*>(smem + a.xs_offset);
    uint8_t* sbuf = smem + a.sbuf_offset;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ns = a.nstage;

    if (tid == 0) {
        for (int s = 0; s < ns; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int64_t rps = (a.N + 1) / 2;
    const int64_t P = static_cast<int64_t>(a.n_seg) * rps;
    // split-K: CTA c covers K range c % ksplit of row-pair range c / ksplit
    const int ks = static_cast<int>(blockIdx.x) % a.ksplit;
    const int64_t rc = blockIdx.x / a.ksplit, G = gridDim.x / a.ksplit;
    const int64_t rp_begin = P * rc / G;
    const int64_t rp_end = P * (rc + 1) / G;
    constexpr int BS = block_bytes_of<FMT>();
    static_assert(FMT <= 2 || NCOL == 1, "Q5_K, Q2_K, Q3_K and Q8_0: one column per launch in this kernel");
    const int kb0 = ks * a.nbs;
    const int nbl = a.nb - kb0 < a.nbs ? a.nb - kb0 : a.nbs;       // blocks in this range
    const int srow = a.ksplit > 1 ? a.nbs * BS : static_cast<int>(a.row_bytes);  // staged row stride

    if (warp == 0) {
        if (lane == 0) {
            prefetch_activations(a, kb0, nbl);
            produce_stages<BS>(a, full, empty, abort_flag, sbuf, rp_begin, rp_end, rps, ns, kb0, nbl, srow,
                               a.ksplit == 1);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int ct_all = tid - 32;             // 0 .. NG*256-1
    const int g = NG == 2 ? (ct_all >> 8) : 0;
    const int ct = ct_all & (kConsumers - 1);  // thread within the group
    const int cw = ct >> 5;                   // warp within the group
    const int gbar = 1 + g;                   // the group's named barrier
    const int nb = a.nbs;                     // lane layout: blocks of a full K range
    const int xcs = 2 * nb * kRegion;
    const bool shared_x = a.x_seg_stride == 0;
    pdl_wait();                      // activations may come from the previous grid
    pdl_launch_dependents();

    // this lane's unit within a stage
    int u_rp, u_b, u_H, group, part;
    bool u_active;
    int kappa = 0;
    int u_pos = 0;  // the lane's integer activation region (single column)
    if (FMT != 2 || NCOL == 1) {  // lanes take (row pair, block, half)
        const int LR = a.lanes_per_rp;
        const LaneUnit L = lane_unit(ct, LR, nbl, a.par);
        u_rp = L.rp;
        u_b = L.b;
        u_H = L.H;
        u_active = L.active;
        u_pos = L.pos;
        group = LR < 32 ? LR : 32;
        part = LR > 32 ? ((ct - u_rp * LR) >> 5) : 0;
    } else {
        const int LRw = a.lanes_per_rp;  // lanes per row pair inside one warp
        kappa = cw;
        u_rp = lane / LRw;
        const int u = lane - u_rp * LRw;
        u_active = u < 2 * (nbl >> 3);
        const int i = u >> 1;
        u_H = u & 1;
        u_b = 8 * i + kappa;
        group = LRw;
        part = kappa;
    }
    const int parts = a.parts;
    // single column with whole row pairs per warp: no cross-warp reduction
    const bool direct = NCOL == 1 && parts == 1;
    int region;
    if (FMT != 2 || NCOL == 1) region = 2 * u_b + u_H;
    else region = ((kappa * (nb >> 3) + (u_b >> 3)) << 1) + u_H;
    const int wp_group = 2 * a.ps * parts * 2 * NCOL;     // floats of one group's double buffer
    // activation copy: fp32 regions (several columns) or the integer groups
    // of the single-column path (kXGroupBytes + kXInfoBytes per 32 weights),
    // which serves every format
    constexpr bool INT = NCOL == 1;
    const uint32_t xcopy = INT ? kXRegionBytes * 2 * nb : 4 * NCOL * xcs;
    const uint32_t xs_s = smem_u32(xs) + (shared_x ? 0 : g * xcopy);
    const uint32_t xri = xs_s + kXRegionBytes * u_pos;  // this lane's integer region
    const uint32_t sbuf_s = smem_u32(sbuf), wp_s = smem_u32(wp) + 4 * g * wp_group;
    const uint32_t xr = xs_s + 4 * (region * kRegion);

    StageIter it(rp_begin, rp_end, rps, a.N, a.ps, ns);
    Stage st;
    const unsigned long long wait_lim = a.wait_ns && blockIdx.x == 0 ? a.wait_ns : kWaitNs;
    int64_t staged_seg = -1;
    // prologue scratch: one region for a shared copy, else the group's own
    const uint32_t pro_r = smem_u32(smem + a.pro_offset) + (shared_x ? 0 : g * kProRegion);
    const uint32_t pro_inv = pro_inv_addr(pro_r);  // RMSNorm: the columns' 1/rms
    float rinv = 1.f;  // RMSNorm: the column's 1/rms, read once per staging (single column)
    if (shared_x) {
        // one activation copy for all groups, staged by all consumer threads
        stage_all<FMT, NCOL, INT, PRO>(a, 0, xs_s, ct_all, NG * kConsumers, NG == 2 ? 3 : 1, kb0, nbl, pro_r);
        if (PRO && a.pro == 1) rinv = ld_s32f(pro_inv);
        staged_seg = 0;
    }
    int own = 0;  // stages this group has consumed
    while (it.next(st)) {
        if (NG == 2 && ((it.count - 1) & 1) != g) continue;
        if (!shared_x && st.seg != staged_seg) {
            // (with warps running free between stages, all of the group must
            // be done with the previous segment's activations first)
            if (direct && staged_seg >= 0) named_bar_sync(gbar, kConsumers);
            stage_all<FMT, NCOL, INT, PRO>(a, st.seg, xs_s, ct, kConsumers, gbar, kb0, nbl, pro_r);
            if (PRO && a.pro == 1) rinv = ld_s32f(pro_inv);
            staged_seg = st.seg;
        }
        const int slot = it.slot;
        // Two groups take alternate stages.  With an odd ring depth a slot
        // alternates between them, so a group first waits until the other
        // group has released the slot's previous stage: only then can the
        // parity wait on `full` not pass on a phase two ahead (it cannot
        // tell phase k from phase k + 2).
        if (NG == 2 && (ns & 1) && it.count > ns &&
            !mbar_wait_bounded(&empty[slot], it.phase ^ 1u, abort_flag, wait_lim))
            raise_fault(a, abort_flag, 6);
        if (!mbar_wait_bounded(&full[slot], it.phase, abort_flag, wait_lim)) raise_fault(a, abort_flag, 6);
        float out[2][NCOL];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int j = 0; j < NCOL; ++j) out[r][j] = 0.f;
        const bool work = u_active && u_rp < st.nrp && !*abort_flag;
        if (work) {
            uint32_t row0 = sbuf_s + slot * a.stage_bytes + 2 * u_rp * srow;
            if (a.ksplit == 1) {  // a contiguous stage starts src % 16 bytes into its slot
                int64_t e = st.seg;
                if (a.ids) e = a.ids[st.seg];
                row0 += static_cast<uint32_t>(
                    reinterpret_cast<uintptr_t>(a.W + e * a.seg_stride + st.row0 * a.row_bytes) & 15u);
            }
            if constexpr (INT && FMT == 1) {
                q4k_unit_int(row0, srow, u_b, u_H, xri, out);
            } else if constexpr (INT && FMT == 3) {
                q5k_unit_int(row0, srow, u_b, u_H, xri, out);
            } else if constexpr (INT && FMT == 4) {
                q2k_unit_int(row0, srow, u_b, u_H, xri, out);
            } else if constexpr (INT && FMT == 5) {
                q3k_unit_int(row0, srow, u_b, u_H, xri, out);
            } else if constexpr (INT && FMT == 6) {
                q80_unit_int(row0, srow, u_b, u_H, xri, out);
            } else if constexpr (INT) {
                if (a.par == 0) q6k_unit_int<2>(row0, srow, u_b, u_H, xri, out);
                else if (u_b & 1) q6k_unit_int<1>(row0, srow, u_b, u_H, xri, out);
                else q6k_unit_int<0>(row0, srow, u_b, u_H, xri, out);
            } else if constexpr (FMT == 1) {
                q4k_unit<NCOL>(row0, srow, u_b, u_H, xr, xcs, out);
            } else {
                q6k_unit_dispatch<NCOL>(kappa, row0, srow, u_b, u_H, xr, xcs, out);
            }
        }
        // butterfly over the lanes of this row pair (fixed order)
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            if (off < group) {
#pragma unroll
                for (int r = 0; r < 2; ++r)
#pragma unroll
                    for (int j = 0; j < NCOL; ++j) out[r][j] += __shfl_xor_sync(0xffffffffu, out[r][j], off);
            }
        }
        if (direct) {
            // one warp holds all units of each of its row pairs: its lead
            // lanes write y, and warps need not wait for each other between
            // stages (the shuffles above have ended the warp's reads)
            // (after a fault the warps keep walking the stages -- every wait
            // then returns at once and no unit runs -- so that all of them
            // reach the same barriers)
            if (lane == 0) mbar_arrive(&empty[slot]);
            if ((lane & (group - 1)) == 0 && u_rp < st.nrp) {
                int64_t e = st.seg;
                if (a.ids) e = a.ids[st.seg];
                const bool valid = e >= 0 && e < a.E;
                if (!valid && a.status) atomicExch(a.status, 7);
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int row = 2 * u_rp + r;
                    if (row >= st.nrows) continue;
                    float v = valid ? out[r][0] : 0.f;
                    if constexpr (PRO) v *= rinv;
                    if (a.ksplit == 1) a.y[st.seg * a.y_seg_stride + st.row0 + row] = v;
                    else a.partial[static_cast<int64_t>(ks) * a.N + st.row0 + row] = v;
                }
            }
            continue;
        }
        // the group's own stages alternate between two partial-sum buffers
        const uint32_t wb = wp_s + 4 * ((own & 1) * (a.ps * parts * 2 * NCOL));
        ++own;
        if ((lane & (group - 1)) == 0 && u_rp < a.ps) {
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int j = 0; j < NCOL; ++j) st_s32f(wb + 4 * (((u_rp * parts + part) * 2 + r) * NCOL + j), out[r][j]);
        }
        const bool stop = named_bar_or(gbar, kConsumers, *abort_flag != 0);
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (stop) break;
        // fixed-order sum over parts, then store
        int64_t e = st.seg;
        if (a.ids) e = a.ids[st.seg];
        const bool valid = e >= 0 && e < a.E;
        if (!valid && ct == 0 && a.status) atomicExch(a.status, 7);
        for (int t = ct; t < st.nrows * NCOL; t += kConsumers) {
            const int row = t / NCOL, j = t - row * NCOL;
            const int rp = row >> 1, r = row & 1;
            float v = 0.f;
            if (valid) {
                for (int p = 0; p < parts; ++p) v += ld_s32f(wb + 4 * (((rp * parts + p) * 2 + r) * NCOL + j));
                if constexpr (PRO) v *= NCOL == 1 ? rinv : (a.pro == 1 ? ld_s32f(pro_inv + 4 * j) : 1.f);
            }
            if (j < a.ncol_real) {
                if (a.ksplit == 1) a.y[st.seg * a.y_seg_stride + j * a.ldy + st.row0 + row] = v;
                else a.partial[(static_cast<int64_t>(ks) * a.ncol_real + j) * a.N + st.row0 + row] = v;
            }
        }
    }
}


// ----------------------------------------------------------- launchers

template <int FMT, int NCOL, int NG>
cudaError_t launch_one(const GemvArgs& a, const LaunchPlan& p, cudaStream_t stream) {
    auto kern = a.pro ? gemv_kernel<FMT, NCOL, NG, true> : gemv_kernel<FMT, NCOL, NG, false>;
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void*>(kern), p.smem_bytes);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(32 + NG * kConsumers);
    cfg.dynamicSmemBytes = p.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = p.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace kq
