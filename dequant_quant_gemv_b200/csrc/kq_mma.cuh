// kq_mma.cuh — the fused K-quant GEMV for 2..8 activation columns on the
// tensor cores: the speculative-verify shape, where k token columns share
// one read of every weight block (Kortex and runNburn pages: the
// multi-token verify matvec).
//
// With k columns the per-weight work of the CUDA-core kernel grows with k
// (one FMA per weight per column); here the multiply-adds go to mma.sync
// m16n8k16 (f16 inputs, f32 accumulation) and the per-weight cost is the
// dequantisation alone, whatever k is.
//
// Exactness.  The A operand (weights) is the integer product sc*q of a
// sub-block scale and a quant, which fp16 represents exactly for Q4_K
// (|sc*q| <= 63*15 < 2048): one fp16 FMA per two weights turns a nibble
// placed in the mantissa of 1024 (0x6400 | n) into sc*n with no rounding.
// The B operand (activations) is each fp32 value rounded to fp16 after a
// power-of-two scale per column and super-block that keeps the largest |x|
// of the block in [2^14, 2^15): a relative error of at most 2^-11 per
// activation, so with exact weights |y - y_exact| <= 2^-11 sum_i |w_i x_i|
// (half the stated bound), and one n-tile of 8 B columns carries 8
// activation columns.  d and the min term are applied per super-block in
// fp32: y = sum_b 2^-e_b d_b S_b - sum_b 2^(5-e_b) dmin_b M_b, where S_b =
// sum sc*q*x (16 K-steps) and M_b = sum_j m_j X_j (two m16n8k8 steps whose
// A holds the 8 mins and B the sub-block sums of x, scaled by 2^(e_b-5) and
// split into a high and a low fp16 term, so that the min term, which may
// nearly cancel the other, keeps 22 bits).
//
// Schedule.  The persistent CTA and its TMA ring are those of gemv_kernel;
// a stage is 16 rows (one m16 tile), copied row by row into smem rows
// `a.sp` bytes apart (a.sp = 64 mod 128 for the 16-byte loads of Q4_K and
// 16 mod 128 for the 4-byte loads of Q6_K keep them free of bank
// conflicts).  The 8 consumer warps split the stage's super-blocks
// (warp w takes blocks w, w+8, ...) and add their partial sums in a fixed
// order, so results are deterministic and each column's value does not
// depend on the other columns.
#pragma once

#include <cuda_fp16.h>

#include "kq_gemv.cuh"

namespace kq {

constexpr int kMmaRowPairs = 8;  // 16 rows per stage
// B fragments of one super-block (256 weights): 16 K-steps of quants
// (m16n8k16: 8 bytes per lane and n-tile), plus for Q4_K and Q5_K two of mins (m16n8k8, the
// activation sums split into a high and a low fp16 term: 4 bytes per lane
// and n-tile)
template <int FMT>
__host__ __device__ constexpr int xb_block_bytes(int nt) {
    return nt * (16 * 256 + (FMT == 2 || FMT == 6 ? 0 : FMT == 4 || FMT == 5 ? 2 * 256 : 2 * 128));
}

// D += A * B for one m16n8k8 tile (the min steps: A = the 8 mins of rows
// g and g+8, B = the sub-block sums of x).
__device__ __forceinline__ void mma1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

// D += A * B for one m16n8k16 tile (row-major A, column-major B).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t hfma2u(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t hmul2u(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hadd2u(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ __half2 u2h2(uint32_t v) { return *reinterpret_cast<const __half2*>(&v); }
__device__ __forceinline__ uint32_t h22u(__half2 v) { return *reinterpret_cast<const uint32_t*>(&v); }
__device__ __forceinline__ uint32_t pack_h2(__half lo, __half hi) {
    return static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
}
__device__ __forceinline__ void st_s32u(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void st_s16u(uint32_t a, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(v) : "memory");
}
__device__ __forceinline__ uint2 ld_s64u(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

constexpr uint32_t kH2_1024 = 0x64006400u;    // (1024, 1024)
constexpr uint32_t kH2_m1024 = 0xE400E400u;   // (-1024, -1024)
constexpr uint32_t kH2_1_16 = 0x2C002C00u;    // (1/16, 1/16)
constexpr uint32_t kH2_m64 = 0xD400D400u;     // (-64, -64)

// Two 6-bit values (bytes p and p+1 of `packed`) as the fp16 pair
// (v_p, v_p+1), exactly: 1024 + v by byte permute, then minus 1024.
__device__ __forceinline__ uint32_t byte_pair_h2(uint32_t packed, uint32_t sel) {
    return hadd2u(__byte_perm(packed, 0x64646464u, sel), kH2_m1024);
}

// ------------------------------------------------------ activation stage

// Power-of-two scale exponent that brings a largest |x| (amax) into
// [2^14, 2^15): 14 - floor(log2(amax)), clamped so 2^+-sh stays a normal
// float.  Zero columns get 0.
__device__ __forceinline__ int col_shift(uint32_t amax_bits) {
    if (amax_bits == 0) return 0;
    int sh = 14 - (static_cast<int>(amax_bits >> 23) - 127);
    return sh > 120 ? 120 : sh < -120 ? -120 : sh;
}
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }

// B-fragment entry of K-step s for one column: the column is B column
// col%8 of n-tile col/8, i.e. lane 4*(col%8) + q.  reg0 holds the K
// positions 2q, 2q+1 and reg1 2q+8, 2q+9: activations 0, 2 and 1, 3 of the
// group of four that feeds the quant word at those positions, each rounded
// to fp16 (relative error at most 2^-11; the block's power-of-two scale
// keeps them normal fp16 numbers unless far below the block's largest).
template <int FMT, int NT>
__device__ __forceinline__ void store_b_entry(uint32_t xb, int bl, int s, int q, int col, float4 v) {
    const int nt = col >> 3, gc = col & 7;
    const __half h0 = __float2half_rn(v.x), h1 = __float2half_rn(v.y), h2 = __float2half_rn(v.z),
                 h3 = __float2half_rn(v.w);
    const uint32_t step = xb + static_cast<uint32_t>(bl * xb_block_bytes<FMT>(NT)) + 8u * (s * 32 * NT + nt);
    st_s64u(step + 8u * NT * (4 * gc + q), pack_h2(h0, h2), pack_h2(h1, h3));
}

// Where 4 consecutive activations w..w+3 (w a multiple of 4) of a block go:
// the K-step s and lane q whose quant word holds weights w..w+3.
//
// Q4_K: weight w is quant byte beta = 32*(w/64) + w%32, low nibble for
// (w/32) even, high otherwise; byte beta is word (beta/4)%4 of 16-byte
// chunk beta/16.  Lane q reads chunks q and q+4; word u of chunk q+4c feeds
// K-step pair j = 4c + u: step 2j (low nibbles) or 2j+1 (high).
//
// Q2_K, Q3_K: weight w = 128n + 32j + l has its 2 low bits at bits 2j of
// quant byte 32n + l, so quant word u (bytes 4u..4u+3) holds weights
// 128n + 32j + 4(u%8) .. +3 of n = u/8 for every j.  K-step s reads word s;
// lane q takes the bits of j = q, so that each lane's weights of a step sit
// in one 16-weight group (8n + 2q + (u%8)/4) and one shift.
//
// Q8_0: the unit of 256 weights is 8 blocks of 32 (fp16 d, then 32 int8
// quants); block j's quant word u (weights 32j + 4u .. +3) feeds K-step
// 2j + u/4, lane u%4, so that a K-step holds 16 weights of one block.
//
// Q6_K: weight w = 128n + 32t + l takes its low bits from ql[64n + l +
// 32(t%2)] (nibble t/2) and its top bits from bits 2t of qh[32n + l].  Lane
// q reads the 4-byte groups lg = q and q+4 of each half n, l = 4lg..4lg+3;
// group (n, lg) is combination c = 2n + lg/4, and the quants of quarter t
// feed K-step s = 4c + t.
template <int FMT>
__device__ __forceinline__ void b_slot(int w, int& s, int& q) {
    if constexpr (FMT == 4 || FMT == 5) {  // Q2_K, Q3_K: weight 128n + 32j + l: step 8n + l/4, lane j
        q = (w >> 5) & 3;
        s = 8 * (w >> 7) + ((w & 31) >> 2);
    } else if constexpr (FMT == 6) {  // Q8_0: word u = (w%32)/4 of block w/32 feeds step 2*(w/32) + u/4, lane u%4
        const int u = (w & 31) >> 2;
        q = u & 3;
        s = 2 * (w >> 5) + (u >> 2);
    } else if constexpr (FMT != 2) {  // Q4_K and Q5_K share the quant order
        const int hi = (w >> 5) & 1;
        const int beta = 32 * (w >> 6) + (w & 31);
        const int ch = beta >> 4, u = (beta >> 2) & 3;
        q = ch & 3;
        s = 2 * (((ch >> 2) << 2) | u) + hi;
    } else {
        const int n = w >> 7, t = (w >> 5) & 3, lg = (w & 31) >> 2;
        q = lg & 3;
        s = 4 * (2 * n + (lg >> 2)) + t;
    }
}

// Stage the activations of the K range [256*kb0, 256*(kb0+nbl)) as
// B fragments (see b_slot) plus, for Q4_K and Q5_K, per block the two min
// steps (16: high terms, 17: low terms): lane (g, q) holds (X_2q, X_2q+1)
// of column g's term and zeros for K positions 8..15, X_j being the
// sub-block sum of 32 activations, split hi + lo so that the min term keeps
// 22 bits (dmin*m*X may nearly cancel d*sc*q*x).  Each
// (column, block) is scaled by its own power of two 2^sh (largest |x| of
// the block into [2^14, 2^15)) and its sums by 2^(sh-5); `bscale` gets
// (2^-sh, 2^(5-sh)) per block and column.  Only the ncol_real columns are
// staged: a column's products never mix with another column's, so the
// entries of the padding columns (whose outputs are not stored) are left as
// they are.
// One warp per (column, block) item, two float4 per lane, U items' loads in
// flight.  PRO: with the prologue a.pro, its second operand
// (gamma, or u) loaded beside x; for RMSNorm each item's sum of squares of
// the raw x (block_sq) goes to part[col][kb0 + bl] (a.nb per column), and
// with `publish` (a cluster) each storing lane also releases it at cluster
// scope.
template <int FMT, int NT, bool PRO, int U>
__device__ void stage_xb(const GemvArgs& a, uint32_t xb, float* bscale, int cw, int nwarps, int lane, int bar,
                         int kb0, int nbl, uint32_t part, bool publish) {
    constexpr int NC = 8 * NT;
    const float* xg = a.x + static_cast<int64_t>(kb0) * 256;
    const int kr = a.ncol_real;
    const int items = kr * nbl;
    const bool rms = PRO && a.pro == 1;
    for (int base = cw; base < items; base += nwarps * U) {
        float4 v[U][2], w[U][2];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int it = base + nwarps * u;
            const int col = it / nbl, bl = it - col * nbl;
            v[u][0] = v[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            if constexpr (PRO) w[u][0] = w[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (it < items && col < kr) {
                const float* xc = xg + col * a.ldx + 256 * bl + 4 * lane;
                if ((reinterpret_cast<uintptr_t>(xc) & 15u) == 0) {
                    v[u][0] = *reinterpret_cast<const float4*>(xc);
                    v[u][1] = *reinterpret_cast<const float4*>(xc + 128);
                } else {
                    v[u][0] = make_float4(xc[0], xc[1], xc[2], xc[3]);
                    v[u][1] = make_float4(xc[128], xc[129], xc[130], xc[131]);
                }
                if constexpr (PRO) {
                    const float* sc = rms ? a.gamma + static_cast<int64_t>(kb0 + bl) * 256 + 4 * lane : xc + a.K;
                    w[u][0] = ld_f4(sc);
                    w[u][1] = ld_f4(sc + 128);
                }
            }
        }
        if constexpr (PRO) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int it = base + nwarps * u;
                const int col = it / nbl, bl = it - col * nbl;
                if (it >= items || col >= kr) continue;  // warp-uniform
                if (rms) {
                    const float sq = block_sq(v[u][0], v[u][1]);
                    if (lane == 0) {
                        st_s32f(part + 4u * (col * a.nb + kb0 + bl), sq);
                        if (publish) fence_acq_rel_cluster();
                    }
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float4 t = v[u][h], m = w[u][h];
                    v[u][h] = rms ? make_float4(t.x * m.x, t.y * m.y, t.z * m.z, t.w * m.w)
                                  : make_float4(silu_gate(t.x, m.x), silu_gate(t.y, m.y), silu_gate(t.z, m.z),
                                                silu_gate(t.w, m.w));
                }
            }
        }
        // items advance two at a time in lockstep (a pair past the end is
        // skipped; an item past the end inside a pair stores nothing), so
        // that their shuffle latencies overlap
#pragma unroll
        for (int c = 0; c < U; c += 2) {
            if (base + nwarps * c >= items) break;  // warp-uniform
            float m[2];
#pragma unroll
            for (int u2 = 0; u2 < 2; ++u2) {
                m[u2] = 0.f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float4 t = v[c + u2][h];
                    m[u2] = fmaxf(m[u2], fmaxf(fmaxf(fabsf(t.x), fabsf(t.y)), fmaxf(fabsf(t.z), fabsf(t.w))));
                }
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
#pragma unroll
                for (int u2 = 0; u2 < 2; ++u2) m[u2] = fmaxf(m[u2], __shfl_xor_sync(0xffffffffu, m[u2], off));
            float X[2][2];
#pragma unroll
            for (int u2 = 0; u2 < 2; ++u2) {
                const int it = base + nwarps * (c + u2);
                const bool valid = it < items;  // warp-uniform
                const int col = it / nbl, bl = it - col * nbl;
                const int sh = col_shift(__float_as_uint(m[u2]));
                const float sc = pow2f(sh);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float4 t = make_float4(v[c + u2][h].x * sc, v[c + u2][h].y * sc, v[c + u2][h].z * sc,
                                                 v[c + u2][h].w * sc);
                    int st, sq;
                    b_slot<FMT>(128 * h + 4 * lane, st, sq);
                    if (valid) store_b_entry<FMT, NT>(xb, bl, st, sq, col, t);
                    if constexpr (FMT == 5) {
                        // Q3_K's code offset (-4 per weight) is a min step: its
                        // sums take the same fp16 activations as the quant steps
                        // (scaled by 2^sh), so that for a code of 4 (weight 0)
                        // the two terms cancel exactly
                        auto hr = [](float f) { return __half2float(__float2half_rn(f)); };
                        X[u2][h] = (hr(t.x) + hr(t.y)) + (hr(t.z) + hr(t.w));
                    } else {
                        X[u2][h] = (v[c + u2][h].x + v[c + u2][h].y) + (v[c + u2][h].z + v[c + u2][h].w);
                    }
                }
                if (valid && lane == 0) {
                    bscale[2 * (bl * NC + col)] = pow2f(-sh);
                    bscale[2 * (bl * NC + col) + 1] = pow2f(5 - sh);
                }
            }
            if constexpr (FMT == 2 || FMT == 6) continue;
            if constexpr (FMT == 4 || FMT == 5) {
                // 16-weight group 8h + lane/4: the 4 lanes of its group, fixed
                // order; K position g of the two min steps (m16n8k16: lane
                // (column, (g%8)/2), register g/8, half g%2)
#pragma unroll
                for (int off = 1; off <= 2; off <<= 1)
#pragma unroll
                    for (int u2 = 0; u2 < 2; ++u2)
#pragma unroll
                        for (int h = 0; h < 2; ++h) X[u2][h] += __shfl_xor_sync(0xffffffffu, X[u2][h], off);
#pragma unroll
                for (int u2 = 0; u2 < 2; ++u2) {
                    const int it = base + nwarps * (c + u2);
                    if (it >= items || (lane & 3) != 0) continue;
                    const int col = it / nbl, bl = it - col * nbl;
                    // (Q3_K's sums are of the scaled activations already)
                    const float scm = FMT == 5 ? 0.03125f : pow2f(col_shift(__float_as_uint(m[u2])) - 5);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int g16 = 8 * h + (lane >> 2);
                        const float Xs = X[u2][h] * scm;
                        const __half xh = __float2half_rn(Xs);
                        const __half xl = __float2half_rn(Xs - __half2float(xh));
                        const int nt = col >> 3, gc = col & 7, q = (g16 & 7) >> 1;
                        const uint32_t step =
                            xb + static_cast<uint32_t>(bl * xb_block_bytes<FMT>(NT)) + 16u * 256u * NT + 8u * nt;
                        const uint32_t eh = step + 8u * NT * (4 * gc + q) + 4u * (g16 >> 3) + 2u * (g16 & 1);
                        st_s16u(eh, __half_as_ushort(xh));
                        st_s16u(eh + 256u * NT, __half_as_ushort(xl));
                    }
                }
                continue;
            }
            // sub-block 4h + lane/8: the 8 lanes of its group, fixed order
#pragma unroll
            for (int off = 1; off <= 4; off <<= 1)
#pragma unroll
                for (int u2 = 0; u2 < 2; ++u2)
#pragma unroll
                    for (int h = 0; h < 2; ++h) X[u2][h] += __shfl_xor_sync(0xffffffffu, X[u2][h], off);
#pragma unroll
            for (int u2 = 0; u2 < 2; ++u2) {
                const int it = base + nwarps * (c + u2);
                if (it >= items || (lane & 7) != 0) continue;
                const int col = it / nbl, bl = it - col * nbl;
                const float scm = pow2f(col_shift(__float_as_uint(m[u2])) - 5);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int j = 4 * h + (lane >> 3);
                    const float Xs = X[u2][h] * scm;
                    const __half xh = __float2half_rn(Xs);
                    const __half xl = __float2half_rn(Xs - __half2float(xh));
                    const int nt = col >> 3, gc = col & 7, q = j >> 1;
                    // the min steps after the block's 16 quant steps: high terms, then low
                    const uint32_t step =
                        xb + static_cast<uint32_t>(bl * xb_block_bytes<FMT>(NT)) + 16u * 256u * NT + 4u * nt;
                    const uint32_t eh = step + 4u * NT * (4 * gc + q), el = eh + 128u * NT;
                    st_s16u(eh + 2 * (j & 1), __half_as_ushort(xh));
                    st_s16u(el + 2 * (j & 1), __half_as_ushort(xl));
                }
            }
        }
    }
    named_bar_sync(bar, 32 * nwarps);
}

// One Q4_K K-step in a single PTX block, so that the A quad and B pair are
// born in the registers the mma reads (separate statements left the
// compiler copying operands into place around every mma).  xg / xg8: quant
// words of rows g and g+8; xsg / xsg8: the same shifted right by 8 (bytes 1
// and 3 in the low halves); MASK picks the nibble (0x000F000F low,
// 0x00F000F0 high); (m, a): the fp16 FMA that turns 1024 + n (or 1024 + 16n)
// into sc*n; baddr: this lane's B entry (NT pairs of registers).
template <int NT, uint32_t MASK>
__device__ __forceinline__ void q4k_step(float (&d)[NT][4], uint32_t xg, uint32_t xg8, uint32_t xsg, uint32_t xsg8,
                                         uint32_t mg, uint32_t ag, uint32_t mg8, uint32_t ag8, uint32_t baddr) {
    if constexpr (NT == 1) {
        asm volatile(
            "{\n\t.reg .b32 t0, t1, t2, t3, a0, a1, a2, a3, b0, b1;\n\t"
            "lop3.b32 t0, %4, %13, 0x64006400, 0xEA;\n\t"
            "lop3.b32 t1, %5, %13, 0x64006400, 0xEA;\n\t"
            "lop3.b32 t2, %6, %13, 0x64006400, 0xEA;\n\t"
            "lop3.b32 t3, %7, %13, 0x64006400, 0xEA;\n\t"
            "fma.rn.f16x2 a0, t0, %8, %9;\n\t"
            "fma.rn.f16x2 a1, t1, %10, %11;\n\t"
            "fma.rn.f16x2 a2, t2, %8, %9;\n\t"
            "fma.rn.f16x2 a3, t3, %10, %11;\n\t"
            "ld.shared.v2.b32 {b0, b1}, [%12];\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {a0, a1, a2, a3}, {b0, b1}, "
            "{%0, %1, %2, %3};\n\t}"
            : "+f"(d[0][0]), "+f"(d[0][1]), "+f"(d[0][2]), "+f"(d[0][3])
            : "r"(xg), "r"(xg8), "r"(xsg), "r"(xsg8), "r"(mg), "r"(ag), "r"(mg8), "r"(ag8), "r"(baddr), "n"(MASK));
    } else {
        asm volatile(
            "{\n\t.reg .b32 t0, t1, t2, t3, a0, a1, a2, a3, b0, b1, b2, b3;\n\t"
            "lop3.b32 t0, %8, %17, 0x64006400, 0xEA;\n\t"
            "lop3.b32 t1, %9, %17, 0x64006400, 0xEA;\n\t"
            "lop3.b32 t2, %10, %17, 0x64006400, 0xEA;\n\t"
            "lop3.b32 t3, %11, %17, 0x64006400, 0xEA;\n\t"
            "fma.rn.f16x2 a0, t0, %12, %13;\n\t"
            "fma.rn.f16x2 a1, t1, %14, %15;\n\t"
            "fma.rn.f16x2 a2, t2, %12, %13;\n\t"
            "fma.rn.f16x2 a3, t3, %14, %15;\n\t"
            "ld.shared.v4.b32 {b0, b1, b2, b3}, [%16];\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {a0, a1, a2, a3}, {b0, b1}, "
            "{%0, %1, %2, %3};\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%4, %5, %6, %7}, {a0, a1, a2, a3}, {b2, b3}, "
            "{%4, %5, %6, %7};\n\t}"
            : "+f"(d[0][0]), "+f"(d[0][1]), "+f"(d[0][2]), "+f"(d[0][3]), "+f"(d[1][0]), "+f"(d[1][1]),
              "+f"(d[1][2]), "+f"(d[1][3])
            : "r"(xg), "r"(xg8), "r"(xsg), "r"(xsg8), "r"(mg), "r"(ag), "r"(mg8), "r"(ag8), "r"(baddr), "n"(MASK));
    }
}

// ------------------------------------------------------ one super-block

// Rows g and g+8 of the stage (smem rows rg, rg8), super-block b, this
// lane's K positions (q = lane%4); B fragments of the block at `xbl` (this
// lane's entry of step 0).  Adds d*S and dmin*M into ys / ym for the lane's
// columns 8n + 2q and 8n + 2q + 1 (at [2n] and [2n + 1]).
template <int NT>
__device__ __forceinline__ void q4k_mma_block(uint32_t rg, uint32_t rg8, int b, uint32_t xbl, uint32_t xml,
                                              uint32_t bsc, uint32_t sel, uint32_t msel, int q,
                                              float (&ys)[2][2 * NT], float (&ym)[2][2 * NT]) {
    const uint32_t o = static_cast<uint32_t>(b) * kQ4Bytes;
    const uint4 hg = ld_s128(rg + o), hg8 = ld_s128(rg8 + o);
    uint4 w[2][2];  // [row][chunk q / q+4]
    w[0][0] = ld_s128(rg + o + 16 + 16 * q);
    w[0][1] = ld_s128(rg + o + 80 + 16 * q);
    w[1][0] = ld_s128(rg8 + o + 16 + 16 * q);
    w[1][1] = ld_s128(rg8 + o + 80 + 16 * q);
    // per row and chunk: (scale of the low-nibble sub-block, of the high)
    uint32_t mlo[2][2], alo[2][2], mhi[2][2], ahi[2][2], mins[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint4 h = r ? hg8 : hg;
        uint32_t sc0, m0, sc1, m1;
        q4k_half_scales(h.y, h.z, h.w, 0, sc0, m0);
        q4k_half_scales(h.y, h.z, h.w, 1, sc1, m1);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const __half2 S = u2h2(byte_pair_h2(c ? sc1 : sc0, sel));
            const __half2 slo = __low2half2(S), shi = __high2half2(S);
            mlo[r][c] = h22u(slo);
            alo[r][c] = h22u(__hmul2(slo, u2h2(kH2_m1024)));
            mhi[r][c] = h22u(__hmul2(shi, u2h2(kH2_1_16)));
            ahi[r][c] = h22u(__hmul2(shi, u2h2(kH2_m64)));
        }
        mins[r] = byte_pair_h2(q < 2 ? m0 : m1, msel);
    }
    float acc[NT][4], accm[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[n][i] = accm[n][i] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int c = j >> 2;
        const uint32_t x0 = u4w(w[0][c], j & 3), x1 = u4w(w[1][c], j & 3);
        const uint32_t s_lo = xbl + 8u * NT * 32 * (2 * j), s_hi = s_lo + 8u * NT * 32;  // steps 2j, 2j+1
        q4k_step<NT, 0x000F000Fu>(acc, x0, x1, x0 >> 8, x1 >> 8, mlo[0][c], alo[0][c], mlo[1][c], alo[1][c], s_lo);
        q4k_step<NT, 0x00F000F0u>(acc, x0, x1, x0 >> 8, x1 >> 8, mhi[0][c], ahi[0][c], mhi[1][c], ahi[1][c], s_hi);
    }
    {
        // the min steps (high terms, then low): this lane's entries at xml
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            mma1688(accm[n], mins[0], mins[1], ld_s32(xml + 4 * n));
            mma1688(accm[n], mins[0], mins[1], ld_s32(xml + 128u * NT + 4 * n));
        }
    }
    const float d0 = __half2float(__ushort_as_half(static_cast<unsigned short>(hg.x & 0xFFFFu)));
    const float m0 = __half2float(__ushort_as_half(static_cast<unsigned short>(hg.x >> 16)));
    const float d1 = __half2float(__ushort_as_half(static_cast<unsigned short>(hg8.x & 0xFFFFu)));
    const float m1 = __half2float(__ushort_as_half(static_cast<unsigned short>(hg8.x >> 16)));
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        // this lane's columns 8n + 2q and 8n + 2q + 1: (2^-sh, 2^(5-sh)) each
        const float4 f = ld_s128f(bsc + 8u * (8 * n + 2 * q));
        ys[0][2 * n] = fmaf(d0 * f.x, acc[n][0], ys[0][2 * n]);
        ys[0][2 * n + 1] = fmaf(d0 * f.z, acc[n][1], ys[0][2 * n + 1]);
        ys[1][2 * n] = fmaf(d1 * f.x, acc[n][2], ys[1][2 * n]);
        ys[1][2 * n + 1] = fmaf(d1 * f.z, acc[n][3], ys[1][2 * n + 1]);
        ym[0][2 * n] = fmaf(m0 * f.y, accm[n][0], ym[0][2 * n]);
        ym[0][2 * n + 1] = fmaf(m0 * f.w, accm[n][1], ym[0][2 * n + 1]);
        ym[1][2 * n] = fmaf(m1 * f.y, accm[n][2], ym[1][2 * n]);
        ym[1][2 * n + 1] = fmaf(m1 * f.w, accm[n][3], ym[1][2 * n + 1]);
    }
}

// Q5_K K-step: as q4k_step, with each code's 5th bit merged in.  hc0..hc3
// replace the exponent constant of the four fp16 pairs: 0x6400 in each half
// with the 5th bit at bit 4 (low nibble: 1024 + q) or bit 8 (high nibble:
// 1024 + 16q) of the half; the scale operands are Q4_K's.
template <int NT, uint32_t MASK>
__device__ __forceinline__ void q5k_step(float (&d)[NT][4], uint32_t xg, uint32_t xg8, uint32_t xsg, uint32_t xsg8,
                                         uint32_t mg, uint32_t ag, uint32_t mg8, uint32_t ag8, uint32_t baddr,
                                         uint32_t hc0, uint32_t hc1, uint32_t hc2, uint32_t hc3) {
    if constexpr (NT == 1) {
        asm volatile(
            "{\n\t.reg .b32 t0, t1, t2, t3, a0, a1, a2, a3, b0, b1;\n\t"
            "lop3.b32 t0, %4, %13, %14, 0xEA;\n\t"
            "lop3.b32 t1, %5, %13, %15, 0xEA;\n\t"
            "lop3.b32 t2, %6, %13, %16, 0xEA;\n\t"
            "lop3.b32 t3, %7, %13, %17, 0xEA;\n\t"
            "fma.rn.f16x2 a0, t0, %8, %9;\n\t"
            "fma.rn.f16x2 a1, t1, %10, %11;\n\t"
            "fma.rn.f16x2 a2, t2, %8, %9;\n\t"
            "fma.rn.f16x2 a3, t3, %10, %11;\n\t"
            "ld.shared.v2.b32 {b0, b1}, [%12];\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {a0, a1, a2, a3}, {b0, b1}, "
            "{%0, %1, %2, %3};\n\t}"
            : "+f"(d[0][0]), "+f"(d[0][1]), "+f"(d[0][2]), "+f"(d[0][3])
            : "r"(xg), "r"(xg8), "r"(xsg), "r"(xsg8), "r"(mg), "r"(ag), "r"(mg8), "r"(ag8), "r"(baddr), "n"(MASK),
              "r"(hc0), "r"(hc1), "r"(hc2), "r"(hc3));
    } else {
        asm volatile(
            "{\n\t.reg .b32 t0, t1, t2, t3, a0, a1, a2, a3, b0, b1, b2, b3;\n\t"
            "lop3.b32 t0, %8, %17, %18, 0xEA;\n\t"
            "lop3.b32 t1, %9, %17, %19, 0xEA;\n\t"
            "lop3.b32 t2, %10, %17, %20, 0xEA;\n\t"
            "lop3.b32 t3, %11, %17, %21, 0xEA;\n\t"
            "fma.rn.f16x2 a0, t0, %12, %13;\n\t"
            "fma.rn.f16x2 a1, t1, %14, %15;\n\t"
            "fma.rn.f16x2 a2, t2, %12, %13;\n\t"
            "fma.rn.f16x2 a3, t3, %14, %15;\n\t"
            "ld.shared.v4.b32 {b0, b1, b2, b3}, [%16];\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {a0, a1, a2, a3}, {b0, b1}, "
            "{%0, %1, %2, %3};\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%4, %5, %6, %7}, {a0, a1, a2, a3}, {b2, b3}, "
            "{%4, %5, %6, %7};\n\t}"
            : "+f"(d[0][0]), "+f"(d[0][1]), "+f"(d[0][2]), "+f"(d[0][3]), "+f"(d[1][0]), "+f"(d[1][1]),
              "+f"(d[1][2]), "+f"(d[1][3])
            : "r"(xg), "r"(xg8), "r"(xsg), "r"(xsg8), "r"(mg), "r"(ag), "r"(mg8), "r"(ag8), "r"(baddr), "n"(MASK),
              "r"(hc0), "r"(hc1), "r"(hc2), "r"(hc3));
    }
}

// Q5_K super-block b of rows g and g+8: q4k_mma_block on the Q5_K byte
// offsets (quants at 48, qh at 16), the lane's 5th bits from qh bytes
// l = 16(q%2) .. 16(q%2)+15, which serve both of its chunks q/2 and q/2 + 2.
template <int NT>
__device__ __forceinline__ void q5k_mma_block(uint32_t rg, uint32_t rg8, int b, uint32_t xbl, uint32_t xml,
                                              uint32_t bsc, uint32_t sel, uint32_t msel, int q,
                                              float (&ys)[2][2 * NT], float (&ym)[2][2 * NT]) {
    const uint32_t o = static_cast<uint32_t>(b) * kQ5Bytes;
    const uint4 hg = ld_s128(rg + o), hg8 = ld_s128(rg8 + o);
    uint4 w[2][2];  // [row][chunk q / q+4 (16-byte segments)]
    w[0][0] = ld_s128(rg + o + 48 + 16 * q);
    w[0][1] = ld_s128(rg + o + 112 + 16 * q);
    w[1][0] = ld_s128(rg8 + o + 48 + 16 * q);
    w[1][1] = ld_s128(rg8 + o + 112 + 16 * q);
    const uint4 e[2] = {ld_s128(rg + o + 16 + 16 * (q & 1)), ld_s128(rg8 + o + 16 + 16 * (q & 1))};
    uint32_t mlo[2][2], alo[2][2], mhi[2][2], ahi[2][2], mins[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint4 h = r ? hg8 : hg;
        uint32_t sc0, m0, sc1, m1;
        q4k_half_scales(h.y, h.z, h.w, 0, sc0, m0);
        q4k_half_scales(h.y, h.z, h.w, 1, sc1, m1);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const __half2 S = u2h2(byte_pair_h2(c ? sc1 : sc0, sel));
            const __half2 slo = __low2half2(S), shi = __high2half2(S);
            mlo[r][c] = h22u(slo);
            alo[r][c] = h22u(__hmul2(slo, u2h2(kH2_m1024)));
            mhi[r][c] = h22u(__hmul2(shi, u2h2(kH2_1_16)));
            ahi[r][c] = h22u(__hmul2(shi, u2h2(kH2_m64)));
        }
        mins[r] = byte_pair_h2(q < 2 ? m0 : m1, msel);
    }
    float acc[NT][4], accm[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[n][i] = accm[n][i] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int c = j >> 2;
        const int sh = 2 * ((q >> 1) + 2 * c);  // bit of the low-nibble codes (chunk q/2 + 2c)
        const uint32_t x0 = u4w(w[0][c], j & 3), x1 = u4w(w[1][c], j & 3);
        const uint32_t e0 = u4w(e[0], j & 3), e1 = u4w(e[1], j & 3);
        const uint32_t bl0 = (e0 >> sh) & 0x01010101u, bl1 = (e1 >> sh) & 0x01010101u;
        const uint32_t bh0 = (e0 >> (sh + 1)) & 0x01010101u, bh1 = (e1 >> (sh + 1)) & 0x01010101u;
        // low nibbles: bytes 0, 2 keep bit 4 of their halves; bytes 1, 3 via >> 8
        const uint32_t l0 = ((bl0 << 4) & 0x00100010u) | 0x64006400u, l1 = ((bl1 << 4) & 0x00100010u) | 0x64006400u;
        const uint32_t l2 = ((bl0 >> 4) & 0x00100010u) | 0x64006400u, l3 = ((bl1 >> 4) & 0x00100010u) | 0x64006400u;
        // high nibbles (16n): the 5th bit is worth 256, bit 8 of the half
        const uint32_t h0 = ((bh0 << 8) & 0x01000100u) | 0x64006400u, h1 = ((bh1 << 8) & 0x01000100u) | 0x64006400u;
        const uint32_t h2 = (bh0 & 0x01000100u) | 0x64006400u, h3 = (bh1 & 0x01000100u) | 0x64006400u;
        const uint32_t s_lo = xbl + 8u * NT * 32 * (2 * j), s_hi = s_lo + 8u * NT * 32;  // steps 2j, 2j+1
        q5k_step<NT, 0x000F000Fu>(acc, x0, x1, x0 >> 8, x1 >> 8, mlo[0][c], alo[0][c], mlo[1][c], alo[1][c], s_lo,
                                  l0, l1, l2, l3);
        q5k_step<NT, 0x00F000F0u>(acc, x0, x1, x0 >> 8, x1 >> 8, mhi[0][c], ahi[0][c], mhi[1][c], ahi[1][c], s_hi,
                                  h0, h1, h2, h3);
    }
    {
        // the min steps (high terms, then low): this lane's entries at xml
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            mma1688(accm[n], mins[0], mins[1], ld_s32(xml + 4 * n));
            mma1688(accm[n], mins[0], mins[1], ld_s32(xml + 128u * NT + 4 * n));
        }
    }
    const float d0 = __half2float(__ushort_as_half(static_cast<unsigned short>(hg.x & 0xFFFFu)));
    const float m0 = __half2float(__ushort_as_half(static_cast<unsigned short>(hg.x >> 16)));
    const float d1 = __half2float(__ushort_as_half(static_cast<unsigned short>(hg8.x & 0xFFFFu)));
    const float m1 = __half2float(__ushort_as_half(static_cast<unsigned short>(hg8.x >> 16)));
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        // this lane's columns 8n + 2q and 8n + 2q + 1: (2^-sh, 2^(5-sh)) each
        const float4 f = ld_s128f(bsc + 8u * (8 * n + 2 * q));
        ys[0][2 * n] = fmaf(d0 * f.x, acc[n][0], ys[0][2 * n]);
        ys[0][2 * n + 1] = fmaf(d0 * f.z, acc[n][1], ys[0][2 * n + 1]);
        ys[1][2 * n] = fmaf(d1 * f.x, acc[n][2], ys[1][2 * n]);
        ys[1][2 * n + 1] = fmaf(d1 * f.z, acc[n][3], ys[1][2 * n + 1]);
        ym[0][2 * n] = fmaf(m0 * f.y, accm[n][0], ym[0][2 * n]);
        ym[0][2 * n + 1] = fmaf(m0 * f.w, accm[n][1], ym[0][2 * n + 1]);
        ym[1][2 * n] = fmaf(m1 * f.y, accm[n][2], ym[1][2 * n]);
        ym[1][2 * n + 1] = fmaf(m1 * f.w, accm[n][3], ym[1][2 * n + 1]);
    }
}

// Q6_K: rows g and g+8, super-block b (starting 2 bytes past a 4-byte
// boundary when ODD), this lane's quant groups (see b_slot).
// A = sc*(q-32): q in the mantissa of 1024 by byte permute, minus 1056,
// times the group's int8 scale (exact while |sc| <= 64; otherwise rounded
// to fp16, within 2^-11 of that weight).  Adds 2^-sh * d * S into ys.
template <int NT, bool ODD>
__device__ __forceinline__ void q6k_mma_block(uint32_t rg, uint32_t rg8, int b, uint32_t xbl, uint32_t bsc, int q,
                                              float (&ys)[2][2 * NT]) {
    uint32_t A[2][4], B[2][4], H[2][4];
    __half2 S[2][4][2];  // [row][combination][t/2]: scales of quarters (t even, t odd)
    float dsc[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint32_t bw = (r ? rg8 : rg) + static_cast<uint32_t>(b) * kQ6Bytes - (ODD ? 2u : 0u);
        auto ldw = [&](int i) -> uint32_t {
            if constexpr (ODD) return __byte_perm(ld_s32(bw + 4 * i), ld_s32(bw + 4 * i + 4), 0x5432);
            else return ld_s32(bw + 4 * i);
        };
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int n = c >> 1, lg = q + 4 * (c & 1);
            A[r][c] = ldw(16 * n + lg);
            B[r][c] = ldw(16 * n + 8 + lg);
            H[r][c] = ldw(32 + 8 * n + lg);
        }
        // int8 scale s as fp16: byte s^0x80 = s+128 in the mantissa of 1024,
        // minus 1152.  Combination c uses scales 8n + c%2 + 2t (t = 0..3):
        // bytes c%2 and c%2+2 of scale words 2n and 2n+1.
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const uint32_t w0 = ldw(48 + 2 * n) ^ 0x80808080u, w1 = ldw(49 + 2 * n) ^ 0x80808080u;
#pragma unroll
            for (int h4 = 0; h4 < 2; ++h4) {
                const uint32_t sel = 0x4040u | static_cast<uint32_t>(h4) | (static_cast<uint32_t>(h4 + 2) << 8);
                S[r][2 * n + h4][0] = __hadd2(u2h2(__byte_perm(w0, 0x64646464u, sel)), u2h2(0xE480E480u));
                S[r][2 * n + h4][1] = __hadd2(u2h2(__byte_perm(w1, 0x64646464u, sel)), u2h2(0xE480E480u));
            }
        }
        const uint32_t dword = ODD ? (ld_s32(bw + 208) >> 16) : ld_s32(bw + 208);
        dsc[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(dword & 0xFFFFu)));
    }
    const __half2 m1056 = u2h2(0xE420E420u);  // (-1056, -1056)
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            uint32_t lo[2], hi[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t src = (t & 1) ? B[r][c] : A[r][c];
                const uint32_t low4 = (t & 2) ? ((src >> 4) & 0x0F0F0F0Fu) : (src & 0x0F0F0F0Fu);
                const uint32_t top2 = (t == 0 ? (H[r][c] << 4) : t == 1 ? (H[r][c] << 2) : t == 2 ? H[r][c]
                                                                                                : (H[r][c] >> 2)) &
                                      0x30303030u;
                const uint32_t qw = low4 | top2;
                const __half2 sc = (t & 1) ? __high2half2(S[r][c][t >> 1]) : __low2half2(S[r][c][t >> 1]);
                lo[r] = h22u(__hmul2(__hadd2(u2h2(__byte_perm(qw, 0x64646464u, 0x4240u)), m1056), sc));
                hi[r] = h22u(__hmul2(__hadd2(u2h2(__byte_perm(qw, 0x64646464u, 0x4341u)), m1056), sc));
            }
            const uint32_t sp = xbl + 8u * NT * 32 * (4 * c + t);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const uint2 bv = ld_s64u(sp + 8 * n);
                mma16816(acc[n], lo[0], lo[1], hi[0], hi[1], bv.x, bv.y);
            }
        }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const float4 f = ld_s128f(bsc + 8u * (8 * n + 2 * q));  // 2^-sh of columns 8n + 2q, 8n + 2q + 1
        ys[0][2 * n] = fmaf(dsc[0] * f.x, acc[n][0], ys[0][2 * n]);
        ys[0][2 * n + 1] = fmaf(dsc[0] * f.z, acc[n][1], ys[0][2 * n + 1]);
        ys[1][2 * n] = fmaf(dsc[1] * f.x, acc[n][2], ys[1][2 * n]);
        ys[1][2 * n + 1] = fmaf(dsc[1] * f.z, acc[n][3], ys[1][2 * n + 1]);
    }
}

// Q2_K / Q3_K K-step (see b_slot): the 2-bit (Q3_K: with its third bit)
// code fields of bytes 0, 2 (t, t8) and 1, 3 (ts, ts8: the words shifted
// right by 8) of rows g and g+8, already masked into the mantissa of 1024
// (1024 + v*4^q), times (sc/4^q) minus 1024*sc/4^q: sc*v exactly, one fp16
// FMA per two weights.
template <int NT>
__device__ __forceinline__ void q23_step(float (&d)[NT][4], uint32_t t, uint32_t t8, uint32_t ts, uint32_t ts8,
                                         uint32_t m, uint32_t a, uint32_t m8, uint32_t a8, uint32_t baddr) {
    const uint32_t a0 = hfma2u(t, m, a), a1 = hfma2u(t8, m8, a8);
    const uint32_t a2 = hfma2u(ts, m, a), a3 = hfma2u(ts8, m8, a8);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const uint2 bv = ld_s64u(baddr + 8 * n);
        mma16816(d[n], a0, a1, a2, a3, bv.x, bv.y);
    }
}

// (v0, v1) - off, exactly: bytes p0, p0 + 1 of `w` (each < 64 + off) as the
// fp16 pair 1024 + v by byte permute, minus 1024 + off.
__device__ __forceinline__ __half2 byte_pair_minus(uint32_t w, uint32_t sel, uint32_t off_h2) {
    return __hsub2(u2h2(__byte_perm(w, 0x64646464u, sel)), u2h2(off_h2));
}

// Q2_K (Q3 = false; 84-byte blocks: 16 scale bytes sc | m << 4, 64 quant
// bytes, d, dmin) and Q3_K (Q3 = true; 110-byte blocks: 32 high-bit bytes,
// 64 quant bytes, 12 bytes of 6-bit scales v, d; a Q3_K block at an odd
// index is 2 bytes off the 4-byte grid (ODD), its words rebuilt by a byte
// permute): rows g and g+8, super-block b, this lane's shift j = q (see
// b_slot).  A = sc*v exactly (Q2_K: sc 0..15, v 0..3; Q3_K: sc = v_g - 32,
// v = the 3-bit code 0..7); the code's offset (Q3_K: -4) and the mins
// (Q2_K) form the min steps: A = the 16 groups' m (Q2_K) or 4*(v_g - 32)
// (Q3_K), B = the groups' activation sums.  Adds d*S and dmin*M (Q3_K: d*M)
// into ys / ym as the Q4_K block does.
template <int NT, bool Q3, bool ODD>
__device__ __forceinline__ void q23_mma_block(uint32_t rg, uint32_t rg8, int b, uint32_t xbl, uint32_t bsc, int q,
                                              float (&ys)[2][2 * NT], float (&ym)[2][2 * NT]) {
    constexpr uint32_t BS = Q3 ? kQ3Bytes : kQ2Bytes;
    constexpr int QW = Q3 ? 8 : 4;  // first quant word of the block
    const uint32_t mq = 0x00030003u << (2 * q);  // bits 2q, 2q+1 of bytes 0 and 2
    const uint32_t hq = 0x00040004u << (2 * q);  // bit 2q + 2 of either half (Q3_K's third bit)
    const uint32_t sel = 0x4040u | (2u * (q & 1)) | ((2u * (q & 1) + 1u) << 8);  // bytes 2(q%2), +1
    const __half2 pw = u2h2(q == 0 ? 0x3C003C00u : q == 1 ? 0x34003400u : q == 2 ? 0x2C002C00u : 0x24002400u);
    uint32_t bw[2];
    uint32_t mh[2][2][2], ah[2][2][2], mins[2][2];  // [row][n][h]; mins [row][n]: K positions 2q(+1) (+8)
    float dd[2], dm[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        bw[r] = (r ? rg8 : rg) + static_cast<uint32_t>(b) * BS - (ODD ? 2u : 0u);
        auto ldw = [&](int i) -> uint32_t {
            if constexpr (ODD) return __byte_perm(ld_s32(bw[r] + 4 * i), ld_s32(bw[r] + 4 * i + 4), 0x5432u);
            else return ld_s32(bw[r] + 4 * i);
        };
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            __half2 sv;  // (sc of group 8n + 2q, of 8n + 2q + 1)
            if constexpr (!Q3) {
                const uint32_t w = ldw(2 * n + (q >> 1));  // scale bytes 8n + 4(q/2) .. +3
                sv = byte_pair_minus(w & 0x0F0F0F0Fu, sel, 0x64006400u);
                mins[r][n] = h22u(byte_pair_minus((w >> 4) & 0x0F0F0F0Fu, sel, 0x64006400u));
            } else {
                // v_g: low 4 bits from byte g (g < 8) or the high nibble of
                // byte g - 8, top 2 bits from bits 2(g/4) of byte 8 + g%4
                const uint32_t lo = ldw(24 + (q >> 1)), hi = ldw(26);
                const uint32_t lo4 = (n ? lo >> 4 : lo) & 0x0F0F0F0Fu;
                const uint32_t hi2 = (hi >> (2 * (2 * n + (q >> 1)))) & 0x03030303u;
                sv = byte_pair_minus(lo4 | (hi2 << 4), sel, 0x64206420u);  // v - 32
                mins[r][n] = h22u(__hmul2(sv, u2h2(0x44004400u)));          // 4*(v - 32)
            }
            const __half2 svq = __hmul2(sv, pw);  // sc / 4^q
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __half2 m = h ? __high2half2(svq) : __low2half2(svq);
                mh[r][n][h] = h22u(m);
                ah[r][n][h] = h22u(__hmul2(m, u2h2(kH2_m1024)));
            }
        }
        const uint32_t dw = Q3 ? ldw(27) : ldw(20);
        dd[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(dw & 0xFFFFu)));
        dm[r] = Q3 ? dd[r] : __half2float(__ushort_as_half(static_cast<unsigned short>(dw >> 16)));
    }
    float acc[NT][4], accm[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[n][i] = accm[n][i] = 0.f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int n = u >> 3, h = (u >> 2) & 1;
        uint32_t t[2], ts[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint32_t bwr = bw[r];
            auto ldw = [&](int i) -> uint32_t {
                if constexpr (ODD) return __byte_perm(ld_s32(bwr + 4 * i), ld_s32(bwr + 4 * i + 4), 0x5432u);
                else return ld_s32(bwr + 4 * i);
            };
            const uint32_t x = ldw(QW + u);
            t[r] = (x & mq) | 0x64006400u;
            ts[r] = ((x >> 8) & mq) | 0x64006400u;
            if constexpr (Q3) {
                // bit 4n + q of each high-bit byte (weights l..l+3) to bit
                // 2q + 2 of its half (bytes 1 and 3 first moved down by 8, so
                // that no bit leaves the word)
                const uint32_t hw = ldw(u & 7);
                auto place = [&](uint32_t v) -> uint32_t {
                    return n == 0 ? v << (q + 2) : q >= 2 ? v << (q - 2) : v >> (2 - q);
                };
                t[r] |= place(hw) & hq;
                ts[r] |= place(hw >> 8) & hq;
            }
        }
        q23_step<NT>(acc, t[0], t[1], ts[0], ts[1], mh[0][n][h], ah[0][n][h], mh[1][n][h], ah[1][n][h],
                     xbl + 8u * NT * 32 * u);
    }
    {
        // the min steps (high terms, then low): K = the 16 groups
        const uint32_t s_m = xbl + 8u * NT * 32 * 16;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const uint2 bh = ld_s64u(s_m + 8 * n), bl = ld_s64u(s_m + 8u * NT * 32 + 8 * n);
            mma16816(accm[n], mins[0][0], mins[1][0], mins[0][1], mins[1][1], bh.x, bh.y);
            mma16816(accm[n], mins[0][0], mins[1][0], mins[0][1], mins[1][1], bl.x, bl.y);
        }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const float4 f = ld_s128f(bsc + 8u * (8 * n + 2 * q));  // (2^-sh, 2^(5-sh)) of columns 8n + 2q, +1
        ys[0][2 * n] = fmaf(dd[0] * f.x, acc[n][0], ys[0][2 * n]);
        ys[0][2 * n + 1] = fmaf(dd[0] * f.z, acc[n][1], ys[0][2 * n + 1]);
        ys[1][2 * n] = fmaf(dd[1] * f.x, acc[n][2], ys[1][2 * n]);
        ys[1][2 * n + 1] = fmaf(dd[1] * f.z, acc[n][3], ys[1][2 * n + 1]);
        ym[0][2 * n] = fmaf(dm[0] * f.y, accm[n][0], ym[0][2 * n]);
        ym[0][2 * n + 1] = fmaf(dm[0] * f.w, accm[n][1], ym[0][2 * n + 1]);
        ym[1][2 * n] = fmaf(dm[1] * f.y, accm[n][2], ym[1][2 * n]);
        ym[1][2 * n + 1] = fmaf(dm[1] * f.w, accm[n][3], ym[1][2 * n + 1]);
    }
}

// Q8_0: rows g and g+8, unit b (8 blocks of 34 bytes), this lane's quant
// words q and 4 + q of each block.  A = q exactly (byte ^ 0x80 = q + 128
// in the mantissa of 1024 by byte permute, minus 1152); a block's two
// K-steps sum into their own accumulator, which is scaled by the block's d
// in fp32.  Blocks at even j have their quants 2 bytes past a 4-byte
// boundary (words rebuilt from two loaded words), odd j aligned ones.  Adds
// 2^-sh * sum_j d_j S_j into ys.
template <int NT>
__device__ __forceinline__ void q80_mma_block(uint32_t rg, uint32_t rg8, int b, uint32_t xbl, uint32_t bsc, int q,
                                              float (&ys)[2][2 * NT]) {
    const uint32_t o = static_cast<uint32_t>(b) * kQ80Bytes;
    const __half2 m1152 = u2h2(0xE480E480u);  // (-1152, -1152)
    float yb[2][2 * NT];  // sum over the unit's blocks of d * S, rows g and g+8
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int n = 0; n < 2 * NT; ++n) yb[r][n] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t w[2][2];
        float d[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint32_t base = (r ? rg8 : rg) + o + 34u * j;  // block j: d, then the quants
            if (j & 1) {  // quants on a 4-byte boundary, d in the upper half of the word below
                w[r][0] = ld_s32(base + 2 + 4 * q);
                w[r][1] = ld_s32(base + 18 + 4 * q);
                d[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(ld_s32(base - 2) >> 16)));
            } else {
                w[r][0] = __byte_perm(ld_s32(base + 4 * q), ld_s32(base + 4 + 4 * q), 0x5432u);
                w[r][1] = __byte_perm(ld_s32(base + 16 + 4 * q), ld_s32(base + 20 + 4 * q), 0x5432u);
                d[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(ld_s32(base) & 0xFFFFu)));
            }
        }
        float acc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t lo[2], hi[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t t = w[r][h] ^ 0x80808080u;
                lo[r] = h22u(__hadd2(u2h2(__byte_perm(t, 0x64646464u, 0x4240u)), m1152));
                hi[r] = h22u(__hadd2(u2h2(__byte_perm(t, 0x64646464u, 0x4341u)), m1152));
            }
            const uint32_t sp = xbl + 8u * NT * 32 * (2 * j + h);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const uint2 bv = ld_s64u(sp + 8 * n);
                mma16816(acc[n], lo[0], lo[1], hi[0], hi[1], bv.x, bv.y);
            }
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            yb[0][2 * n] = fmaf(d[0], acc[n][0], yb[0][2 * n]);
            yb[0][2 * n + 1] = fmaf(d[0], acc[n][1], yb[0][2 * n + 1]);
            yb[1][2 * n] = fmaf(d[1], acc[n][2], yb[1][2 * n]);
            yb[1][2 * n + 1] = fmaf(d[1], acc[n][3], yb[1][2 * n + 1]);
        }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const float4 f = ld_s128f(bsc + 8u * (8 * n + 2 * q));  // 2^-sh of columns 8n + 2q, 8n + 2q + 1
        ys[0][2 * n] = fmaf(f.x, yb[0][2 * n], ys[0][2 * n]);
        ys[0][2 * n + 1] = fmaf(f.z, yb[0][2 * n + 1], ys[0][2 * n + 1]);
        ys[1][2 * n] = fmaf(f.x, yb[1][2 * n], ys[1][2 * n]);
        ys[1][2 * n + 1] = fmaf(f.z, yb[1][2 * n + 1], ys[1][2 * n + 1]);
    }
}

// ------------------------------------------------------------ the kernel

// Split K inside a cluster (a.cluster): the ksplit CTAs of a cluster share
// one row range, CTA r covering K range r (and staging only that range's
// activations).  Each stage's partial sums of CTAs 1..S-1 go into rank 0's
// shared memory (two buffers, by stage parity) with a remote arrive per
// value on rank 0's `recv` barrier; rank 0 adds them in rank order, writes
// y and releases the buffer to each sender through its `sent` barrier
// (skipped for the last two stages, which no sender waits for).  A cluster
// barrier at the start (barriers initialised) and at the end (no CTA leaves
// while another may still address its shared memory) brackets it all.
template <int FMT, int NT, int NG, bool PRO>
__global__ void __launch_bounds__(32 + NG * kConsumers, 1) mma_kernel(const __grid_constant__ GemvArgs a) {
    constexpr int NC = 8 * NT;
    constexpr int NRED = 16 * NC;  // values of one stage's partial sums
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 2 * kMaxStages * 8);
    uint64_t* recv = reinterpret_cast<uint64_t*>(smem + 2 * kMaxStages * 8 + 8);  // [2], rank 0
    uint64_t* sent = recv + 2;                                                    // [2], ranks > 0
    uint64_t* pready = sent + 2;  // RMSNorm in a cluster: the other ranks' partial sums are in place
    float* bscale = reinterpret_cast<float*>(smem + a.xscale_offset);  // [block][column] (2^-sh, 2^(5-sh))
    uint8_t* sbuf = smem + a.sbuf_offset;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ns = a.nstage;
    const int S = a.ksplit;
    const bool cl = a.cluster != 0;
    if (tid == 0) {
        for (int s = 0; s < ns; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        if (cl)
            for (int i = 0; i < 2; ++i) {
                mbar_init(&recv[i], static_cast<uint32_t>((S - 1) * NRED));
                mbar_init(&sent[i], 1);
            }
        if (PRO && cl) mbar_init(pready, static_cast<uint32_t>(S - 1));
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (cl) cluster_sync();

    const int64_t rps = (a.N + 1) / 2;
    const int ks = static_cast<int>(blockIdx.x) % S;  // = the rank within the cluster
    const int64_t rc = blockIdx.x / S, G = gridDim.x / S;
    const int64_t rp_begin = rps * rc / G;
    const int64_t rp_end = rps * (rc + 1) / G;
    const int total = static_cast<int>((rp_end - rp_begin + kMmaRowPairs - 1) / kMmaRowPairs);
    constexpr int BS = block_bytes_of<FMT>();
    const int kb0 = ks * a.nbs;
    const int nbl = a.nb - kb0 < a.nbs ? a.nb - kb0 : a.nbs;
    const uint32_t rem = static_cast<uint32_t>(kb0 * BS) & 15u;  // Q6_K ranges may start off a 16-byte boundary

    if (warp == 0) {
        if (lane == 0) {
            prefetch_activations(a, kb0, nbl);
            produce_stages<BS>(a, full, empty, abort_flag, sbuf, rp_begin, rp_end, rps, ns, kb0, nbl, a.sp, false);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ consumers
        // NG groups of 8 warps take alternate stages (group g: stages with
        // index = g mod NG), hiding each other's latencies
        const int ct_all = tid - 32;
        const int g_id = NG == 2 ? (ct_all >> 8) : 0;
        const int ct = ct_all & (kConsumers - 1);
        const int cw = ct >> 5;
        const int g = lane >> 2, q = lane & 3;
        const uint32_t xb_s = smem_u32(smem + a.xs_offset);
        const uint32_t wp_s = smem_u32(smem + a.wp_offset);
        const uint32_t red_s = smem_u32(smem + a.red_offset);
        const uint32_t sbuf_s = smem_u32(sbuf);
        pdl_wait();
        pdl_launch_dependents();
        // RMSNorm scratch: partial sums of squares [column][super-block], then
        // the columns' 1/rms
        const uint32_t pro_s = smem_u32(smem + a.pro_offset), pro_inv = pro_s + 4u * 8 * a.nb;
        stage_xb<FMT, NT, PRO, (PRO || NG == 2) ? 4 : 8>(a, xb_s, bscale, ct_all >> 5, NG * kConsumerWarps, lane, 3, kb0, nbl, pro_s, cl);
        if constexpr (PRO) {
            if (a.pro == 1) {
                // each CTA of a cluster has its own blocks' sums: tell the
                // other ranks they are in place, wait for theirs, and read
                // them from their shared memory
                if (cl && ct_all == 0)
                    for (int r = 0; r < S; ++r)
                        if (r != ks) mbar_arrive_remote(map_rank(smem_u32(pready), static_cast<uint32_t>(r)));
                if (cl && (ct_all >> 5) < a.ncol_real && !mbar_wait_cluster_bounded(pready, 0, abort_flag))
                    raise_fault(a, abort_flag, 6);
                rms_finish(static_cast<float>(a.K), a.eps, pro_s, a.nb, a.nb, pro_inv, a.ncol_real, ct_all >> 5, lane,
                           3, NG * kConsumers, cl ? a.nbs : 0);
            }
        }
        // RMSNorm: this thread's outputs are all of column ct % NC (NC
        // divides the group's thread count), so its 1/rms is read once
        float rinv = 1.f;
        if (PRO && a.pro == 1) rinv = ld_s32f(pro_inv + 4u * (ct % NC));

        // byte selectors: scales of chunk q (half 0) / q+4 (half 1) sit at
        // bytes 2*(q/2), 2*(q/2)+1 of either half; mins 2q, 2q+1 at bytes
        // 2*(q%2), +1
        const uint32_t p0 = 2u * static_cast<uint32_t>(q >> 1), pm = 2u * static_cast<uint32_t>(q & 1);
        const uint32_t sel = 0x4040u | p0 | ((p0 + 1) << 8);
        const uint32_t msel = 0x4040u | pm | ((pm + 1) << 8);
        const uint32_t xlane = xb_s + 8u * NT * lane;            // this lane's quant-step entries
        const uint32_t xmlane = xb_s + 16u * 256u * NT + 4u * NT * lane;  // and min-step entries
        const uint32_t bsc_s = smem_u32(bscale);

        StageIter it(rp_begin, rp_end, rps, a.N, kMmaRowPairs, ns);
        Stage st;
        while (it.next(st)) {
            const int slot = it.slot;
            const int si = it.count - 1;  // this stage's index in the CTA's sequence
            if (NG == 2 && (si & 1) != g_id) continue;
            // with an odd ring depth, first the other group's release of the
            // slot's previous stage (see gemv_kernel)
            if (NG == 2 && (ns & 1) && si >= ns && !mbar_wait_bounded(&empty[slot], it.phase ^ 1u, abort_flag))
                raise_fault(a, abort_flag, 6);
            if (!mbar_wait_bounded(&full[slot], it.phase, abort_flag)) raise_fault(a, abort_flag, 6);
            float ys[2][2 * NT], ym[2][2 * NT];  // rows g, g+8; columns 8n + 2q + c at [2n + c]
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int n = 0; n < 2 * NT; ++n) ys[r][n] = ym[r][n] = 0.f;
            if (!*abort_flag) {
                // the K range starts `rem` bytes into each smem row (see produce_stages)
                const uint32_t rg = sbuf_s + slot * a.stage_bytes + g * a.sp + rem;
                const uint32_t rg8 = rg + 8 * a.sp;
                for (int b = cw; b < nbl; b += kConsumerWarps) {
                    const uint32_t xbo = static_cast<uint32_t>(xb_block_bytes<FMT>(NT) * b);
                    const uint32_t xbl = xlane + xbo, xml = xmlane + xbo, bsc = bsc_s + 8u * NC * b;
                    if constexpr (FMT == 1) q4k_mma_block<NT>(rg, rg8, b, xbl, xml, bsc, sel, msel, q, ys, ym);
                    else if constexpr (FMT == 3) q5k_mma_block<NT>(rg, rg8, b, xbl, xml, bsc, sel, msel, q, ys, ym);
                    else if constexpr (FMT == 6) q80_mma_block<NT>(rg, rg8, b, xbl, bsc, q, ys);
                    else if constexpr (FMT == 4) q23_mma_block<NT, false, false>(rg, rg8, b, xbl, bsc, q, ys, ym);
                    else if constexpr (FMT == 5) {
                        if (((rem >> 1) + b) & 1) q23_mma_block<NT, true, true>(rg, rg8, b, xbl, bsc, q, ys, ym);
                        else q23_mma_block<NT, true, false>(rg, rg8, b, xbl, bsc, q, ys, ym);
                    }
                    else if (((rem >> 1) + b) & 1) q6k_mma_block<NT, true>(rg, rg8, b, xbl, bsc, q, ys);
                    else q6k_mma_block<NT, false>(rg, rg8, b, xbl, bsc, q, ys);
                }
            }
            const int p = si & 1;  // reduction buffer (with two groups: the group's own)
            const uint32_t wb =
                wp_s + 4u * ((2 * g_id + ((si / NG) & 1)) * (kConsumerWarps * 16 * NC));
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        st_s32f(wb + 4u * ((cw * 16 + g + 8 * r) * NC + 8 * n + 2 * q + c),
                                ys[r][2 * n + c] - ym[r][2 * n + c]);
            const bool stop = named_bar_or(1 + g_id, kConsumers, *abort_flag != 0);
            if (lane == 0) mbar_arrive(&empty[slot]);
            if (stop) break;
            if (!cl) {
                for (int t = ct; t < st.nrows * NC; t += kConsumers) {
                    const int row = t / NC, j = t - row * NC;
                    if (j >= a.ncol_real) continue;
                    float v = 0.f;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) v += ld_s32f(wb + 4u * ((w * 16 + row) * NC + j));
                    if constexpr (PRO) v *= rinv;
                    if (S == 1) a.y[j * a.ldy + st.row0 + row] = v;
                    else a.partial[(static_cast<int64_t>(ks) * a.ncol_real + j) * a.N + st.row0 + row] = v;
                }
                continue;
            }
            // cluster reduction: thread ct < NRED owns (row, column) ct
            if (ct < NRED) {
                const int row = ct / NC, j = ct - row * NC;
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) v += ld_s32f(wb + 4u * ((w * 16 + row) * NC + j));
                if (ks == 0) {
                    if (!mbar_wait_cluster_bounded(&recv[p], (si >> 1) & 1, abort_flag)) raise_fault(a, abort_flag, 6);
                    for (int r = 1; r < S; ++r) v += ld_s32f(red_s + 4u * ((p * (S - 1) + r - 1) * NRED + ct));
                    if constexpr (PRO) v *= rinv;
                    if (row < st.nrows && j < a.ncol_real) a.y[j * a.ldy + st.row0 + row] = v;
                    named_bar_sync(4 + g_id, NRED);  // every value of buffer p read
                    if (ct < S - 1 && si + 2 < total) mbar_arrive_remote(map_rank(smem_u32(&sent[p]), ct + 1));
                } else {
                    if (si >= 2 && !mbar_wait_cluster_bounded(&sent[p], ((si >> 1) - 1) & 1, abort_flag))
                        raise_fault(a, abort_flag, 6);
                    st_cluster_f32(map_rank(red_s + 4u * ((p * (S - 1) + ks - 1) * NRED + ct), 0), v);
                    mbar_arrive_remote(map_rank(smem_u32(&recv[p]), 0));
                }
            }
        }
    }
    __syncwarp();
    if (cl) cluster_sync();
}

template <int FMT, int NT, int NG>
cudaError_t launch_mma(const GemvArgs& a, const LaunchPlan& p, cudaStream_t stream) {
    auto kern = a.pro ? mma_kernel<FMT, NT, NG, true> : mma_kernel<FMT, NT, NG, false>;
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void*>(kern), p.smem_bytes);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(32 + NG * kConsumers);
    cfg.dynamicSmemBytes = p.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = p.pdl ? 1 : 0;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = p.cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.cluster > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

// Clusters of `cluster` CTAs of this kernel (the prologue instantiation if
// `pro`) with `smem_bytes` each that fit on the device at once (0 if none).
template <int FMT, int NT, int NG>
cudaError_t mma_active_clusters(int cluster, size_t smem_bytes, bool pro, int* out) {
    auto kern = pro ? mma_kernel<FMT, NT, NG, true> : mma_kernel<FMT, NT, NG, false>;
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem_bytes);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster);
    cfg.blockDim = dim3(32 + NG * kConsumers);
    cfg.dynamicSmemBytes = smem_bytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaOccupancyMaxActiveClusters(out, kern, &cfg);
}

}  // namespace kq
