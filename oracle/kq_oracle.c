/*
 * kq_oracle — plain, slow, obviously correct CPU reference for the K-quant
 * dequant-GEMV.  TEST INFRASTRUCTURE ONLY: tests, the smoke check and the
 * benchmark's CPU-baseline leg use it; the product (libkq) never links,
 * loads or calls it, and it shares no code, header or table with libkq.
 *
 * What it computes (the method's definition, written out):
 *   y_r = sum_i w_{r,i} * x_i       (double precision, natural index order)
 *   s_r = sum_i |w_{r,i} * x_i|     (for the per-output tolerance)
 * where w is obtained by dequantising every super-block of row r to double
 * by its block formula.  Sources:
 *  - "Out-of-core LLM inference engine written from scratch in Rust",
 *    Approach: quantised weights are dequantised inside the fused matmul
 *    kernels; Results: Llama-3.3-70B Q4_K_M.
 *  - "Kortex: Streaming 70B Models on Consumer GPUs", Key components item 3:
 *    weights are dequantised only in GPU registers (so the product equals the
 *    plain matvec over dequantised weights, up to rounding).
 *  - "RunNburn - Run a 295B MoE ...": native K-quant kernels Q2_K..Q6_K.
 *  The pages name the formats (GGUF K-quants, "Q4_K_M") but print no bit
 *  layout; the layout below is the public GGUF one, restated:
 *   Q4_K (144 B, 256 weights = 8 sub-blocks of 32):
 *     w = d*sc_j*q - dmin*m_j for weight in sub-block j.
 *   Q5_K (176 B, 256 weights = 8 sub-blocks of 32):
 *     w = d*sc_j*q - dmin*m_j as Q4_K, with q a 5-bit quant (0..31).
 *   Q6_K (210 B, 256 weights = 16 groups of 16):
 *     w = d*s_g*(q - 32) for weight in group g, s_g a signed byte.
 *   Q2_K (84 B, 16 groups of 16): w = d*sc_g*q - dmin*m_g, q in 0..3,
 *     sc_g and m_g 4-bit.
 *   Q3_K (110 B, 16 groups of 16): w = d*(v_g - 32)*q, q in -4..3, v_g a
 *     6-bit scale.
 *   Q8_0 (34 B per block of 32: fp16 d, then 32 int8 quants): w = d*q.  A
 *     row of K weights is K/32 consecutive blocks; here taken 8 blocks (256
 *     weights, 272 B) at a time, like the K-quant super-blocks.
 *
 * Every step is a literal loop; no blocking, fusion or reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { KQO_Q4_K = 1, KQO_Q6_K = 2, KQO_Q5_K = 3, KQO_Q2_K = 4, KQO_Q3_K = 5, KQO_Q8_0 = 6 };

/* IEEE binary16 -> double (exact), including subnormals, inf and NaN. */
double kqo_f16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int mant = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)mant, -24);                 /* subnormal / zero */
    else if (e == 31) v = mant ? NAN : INFINITY;
    else v = ldexp((double)(1024 + mant), e - 25);            /* (1 + mant/1024) * 2^(e-15) */
    return sign ? -v : v;
}

static uint16_t rd16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* Q4_K super-block -> logical fields.
 * Header: d (fp16), dmin (fp16), 12 bytes of packed 6-bit scales and mins.
 * For j < 4 the scale and min are the low 6 bits of bytes j and j+4.
 * For j >= 4 the low 4 bits come from byte j+4 (scale: low nibble, min:
 * high nibble) and the top 2 bits from bits 6..7 of byte j-4 (scale) and
 * byte j (min).
 * Quants: 4 chunks of 32 bytes; byte l of chunk c holds weight 64c+l in its
 * low nibble and weight 64c+32+l in its high nibble. */
void kqo_q4k_unpack(const uint8_t* blk, uint8_t q[256], uint8_t sc[8], uint8_t m[8],
                    double* d, double* dmin) {
    const uint8_t* s = blk + 4;
    const uint8_t* qs = blk + 16;
    *d = kqo_f16(rd16(blk));
    *dmin = kqo_f16(rd16(blk + 2));
    for (int j = 0; j < 8; ++j) {
        if (j < 4) {
            sc[j] = s[j] & 63;
            m[j] = s[j + 4] & 63;
        } else {
            sc[j] = (uint8_t)((s[j + 4] & 15) | ((s[j - 4] >> 6) << 4));
            m[j] = (uint8_t)((s[j + 4] >> 4) | ((s[j] >> 6) << 4));
        }
    }
    for (int i = 0; i < 256; ++i) {
        int c = i / 64;           /* 32-byte chunk */
        int within = i % 64;      /* 0..31 low nibbles, 32..63 high nibbles */
        uint8_t byte = qs[32 * c + (within % 32)];
        q[i] = within < 32 ? (byte & 15) : (byte >> 4);
    }
}

/* Q5_K super-block -> logical fields.
 * Header as Q4_K (d, dmin, the same 12 packed scale/min bytes), then 32
 * bytes qh, then 128 quant bytes qs.  Weight i lies in 32-byte chunk
 * c = i/64 of qs at byte l = i%32: its low 4 bits are the low nibble of that
 * byte when i%64 < 32 and the high nibble otherwise; its 5th bit is bit
 * 2c (low-nibble weights) or 2c+1 (high-nibble weights) of qh[l]. */
void kqo_q5k_unpack(const uint8_t* blk, uint8_t q[256], uint8_t sc[8], uint8_t m[8],
                    double* d, double* dmin) {
    const uint8_t* s = blk + 4;
    const uint8_t* qh = blk + 16;
    const uint8_t* qs = blk + 48;
    *d = kqo_f16(rd16(blk));
    *dmin = kqo_f16(rd16(blk + 2));
    for (int j = 0; j < 8; ++j) {
        if (j < 4) {
            sc[j] = s[j] & 63;
            m[j] = s[j + 4] & 63;
        } else {
            sc[j] = (uint8_t)((s[j + 4] & 15) | ((s[j - 4] >> 6) << 4));
            m[j] = (uint8_t)((s[j + 4] >> 4) | ((s[j] >> 6) << 4));
        }
    }
    for (int i = 0; i < 256; ++i) {
        int c = i / 64;
        int within = i % 64;
        int l = within % 32;
        int upper = within >= 32;
        uint8_t byte = qs[32 * c + l];
        int lo4 = upper ? (byte >> 4) : (byte & 15);
        int bit5 = (qh[l] >> (2 * c + upper)) & 1;
        q[i] = (uint8_t)(lo4 | (bit5 << 4));
    }
}

/* Q2_K super-block -> logical fields.
 * Bytes 0..15: one byte per 16-weight group g, scale in the low nibble, min
 * in the high nibble.  Bytes 16..79: quants; weight 128n + 32j + l (n < 2,
 * j < 4, l < 32) is bits 2j..2j+1 of byte 16 + 32n + l.  Then d, dmin. */
void kqo_q2k_unpack(const uint8_t* blk, uint8_t q[256], uint8_t sc[16], uint8_t m[16], double* d, double* dmin) {
    for (int g = 0; g < 16; ++g) {
        sc[g] = blk[g] & 15;
        m[g] = blk[g] >> 4;
    }
    for (int i = 0; i < 256; ++i) {
        int n = i / 128, j = (i % 128) / 32, l = i % 32;
        q[i] = (uint8_t)((blk[16 + 32 * n + l] >> (2 * j)) & 3);
    }
    *d = kqo_f16(rd16(blk + 80));
    *dmin = kqo_f16(rd16(blk + 82));
}

/* Q3_K super-block -> logical fields.
 * Bytes 0..31 hmask, 32..95 quants, 96..107 scales, then d.  Weight
 * 128n + 32j + l: low 2 bits = bits 2j..2j+1 of byte 32 + 32n + l; third bit
 * = bit 4n + j of hmask[l]; value = (low | third << 2) - 4.  Group g's 6-bit
 * scale: low 4 bits from the low nibble of scale byte g (g < 8) or the high
 * nibble of byte g - 8 (g >= 8); top 2 bits from bits 2(g/4)..2(g/4)+1 of
 * scale byte 8 + g%4.  The group multiplies by (v - 32). */
void kqo_q3k_unpack(const uint8_t* blk, int8_t q[256], uint8_t v[16], double* d) {
    const uint8_t* hm = blk;
    const uint8_t* qs = blk + 32;
    const uint8_t* sb = blk + 96;
    for (int i = 0; i < 256; ++i) {
        int n = i / 128, j = (i % 128) / 32, l = i % 32;
        int low = (qs[32 * n + l] >> (2 * j)) & 3;
        int third = (hm[l] >> (4 * n + j)) & 1;
        q[i] = (int8_t)((low | (third << 2)) - 4);
    }
    for (int g = 0; g < 16; ++g) {
        int lo = g < 8 ? (sb[g] & 15) : (sb[g - 8] >> 4);
        int hi = (sb[8 + g % 4] >> (2 * (g / 4))) & 3;
        v[g] = (uint8_t)(lo | (hi << 4));
    }
    *d = kqo_f16(rd16(blk + 108));
}

/* Q6_K super-block -> logical fields.
 * Layout: ql[128] (low 4 bits), qh[64] (top 2 bits), 16 signed scales, d.
 * Weight i = 128h + 32t + l (h<2, t<4, l<32): low bits from
 * ql[64h + l + 32*(t%2)] (low nibble for t<2, high nibble for t>=2), top
 * bits from bits 2t..2t+1 of qh[32h + l]; its scale is scales[i/16]. */
void kqo_q6k_unpack(const uint8_t* blk, uint8_t q[256], int8_t s[16], double* d) {
    const uint8_t* ql = blk;
    const uint8_t* qh = blk + 128;
    for (int i = 0; i < 256; ++i) {
        int h = i / 128, t = (i % 128) / 32, l = i % 32;
        uint8_t lb = ql[64 * h + l + 32 * (t % 2)];
        int lo = t < 2 ? (lb & 15) : (lb >> 4);
        int hi = (qh[32 * h + l] >> (2 * t)) & 3;
        q[i] = (uint8_t)(lo | (hi << 4));
    }
    for (int g = 0; g < 16; ++g) s[g] = (int8_t)blk[192 + g];
    *d = kqo_f16(rd16(blk + 208));
}

/* Q8_0, eight blocks (256 weights) -> logical fields: block j at byte 34j
 * holds d_j (fp16) and then the int8 quants of weights 32j..32j+31. */
void kqo_q80_unpack(const uint8_t* unit, int8_t q[256], double d[8]) {
    for (int j = 0; j < 8; ++j) {
        const uint8_t* blk = unit + 34 * j;
        d[j] = kqo_f16(rd16(blk));
        for (int i = 0; i < 32; ++i) q[32 * j + i] = (int8_t)blk[2 + i];
    }
}

/* Bytes per 256 weights. */
static int64_t block_bytes(int fmt) {
    return fmt == KQO_Q4_K ? 144 : fmt == KQO_Q6_K ? 210 : fmt == KQO_Q5_K ? 176 : fmt == KQO_Q2_K ? 84
         : fmt == KQO_Q3_K ? 110 : fmt == KQO_Q8_0 ? 272 : -1;
}

/* Dequantise one row of K weights (K/256 consecutive super-blocks). */
int kqo_dequant_row(int fmt, const uint8_t* row, int64_t K, double* w) {
    int64_t bb = block_bytes(fmt);
    if (bb < 0 || K % 256 != 0) return -1;
    for (int64_t b = 0; b < K / 256; ++b) {
        const uint8_t* blk = row + b * bb;
        uint8_t q[256];
        double* wb = w + 256 * b;
        if (fmt == KQO_Q4_K || fmt == KQO_Q5_K) {
            uint8_t sc[8], m[8];
            double d, dmin;
            if (fmt == KQO_Q4_K) kqo_q4k_unpack(blk, q, sc, m, &d, &dmin);
            else kqo_q5k_unpack(blk, q, sc, m, &d, &dmin);
            for (int i = 0; i < 256; ++i) {
                int j = i / 32;
                wb[i] = d * sc[j] * q[i] - dmin * m[j];
            }
        } else if (fmt == KQO_Q2_K) {
            uint8_t sc[16], m[16];
            double d, dmin;
            kqo_q2k_unpack(blk, q, sc, m, &d, &dmin);
            for (int i = 0; i < 256; ++i) {
                int g = i / 16;
                wb[i] = d * sc[g] * q[i] - dmin * m[g];
            }
        } else if (fmt == KQO_Q3_K) {
            int8_t qq[256];
            uint8_t v[16];
            double d;
            kqo_q3k_unpack(blk, qq, v, &d);
            for (int i = 0; i < 256; ++i) {
                int g = i / 16;
                wb[i] = d * ((int)v[g] - 32) * qq[i];
            }
        } else if (fmt == KQO_Q8_0) {
            int8_t qq[256];
            double d[8];
            kqo_q80_unpack(blk, qq, d);
            for (int i = 0; i < 256; ++i) wb[i] = d[i / 32] * qq[i];
        } else {
            int8_t s[16];
            double d;
            kqo_q6k_unpack(blk, q, s, &d);
            for (int i = 0; i < 256; ++i) {
                int g = i / 16;
                wb[i] = d * s[g] * ((int)q[i] - 32);
            }
        }
    }
    return 0;
}

/* y and s for the listed rows of W (row r starts at W + r*row_bytes). */
int kqo_gemv_rows(int fmt, const uint8_t* W, int64_t K, const int64_t* rows, int64_t nrows,
                  const float* x, double* y, double* sabs, int nthreads) {
    int64_t bb = block_bytes(fmt);
    if (bb < 0 || K % 256 != 0) return -1;
    int64_t row_bytes = K / 256 * bb;
    int bad = 0;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel num_threads(nthreads)
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)K);
        if (!w) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(static)
        for (int64_t t = 0; t < nrows; ++t) {
            if (!w) continue;
            kqo_dequant_row(fmt, W + rows[t] * row_bytes, K, w);
            double acc = 0.0, acc_abs = 0.0;
            for (int64_t i = 0; i < K; ++i) {
                double p = w[i] * (double)x[i];
                acc += p;
                acc_abs += fabs(p);
            }
            y[t] = acc;
            if (sabs) sabs[t] = acc_abs;
        }
        free(w);
    }
    return bad ? -2 : 0;
}

/* Full matvec: all N rows. */
int kqo_gemv(int fmt, const uint8_t* W, int64_t N, int64_t K, const float* x, double* y,
             double* sabs, int nthreads) {
    int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)(N > 0 ? N : 1));
    if (!rows) return -2;
    for (int64_t r = 0; r < N; ++r) rows[r] = r;
    int rc = kqo_gemv_rows(fmt, W, K, rows, N, x, y, sabs, nthreads);
    free(rows);
    return rc;
}

/* ---------------------------------------------------------------------
 * Activation prologues (the step in front of a layer's matmuls).  The
 * pages do not define them; these are the textbook RMSNorm and SiLU-gated
 * unit of the Llama/Qwen decoder layers whose decode the pages benchmark:
 *   rmsnorm: out_i = x_i * gamma_i / sqrt( (1/K) sum_j x_j^2 + eps )
 *   swiglu:  out_i = silu(g_i) * u_i,  silu(g) = g / (1 + exp(-g)),
 *            with gu = [g_0..g_{K-1}, u_0..u_{K-1}].
 * Computed in double from the fp32 inputs. */
void kqo_rmsnorm(const float* x, const float* gamma, int64_t K, double eps, double* out) {
    double ss = 0.0;
    for (int64_t i = 0; i < K; ++i) ss += (double)x[i] * (double)x[i];
    const double inv = 1.0 / sqrt(ss / (double)K + eps);
    for (int64_t i = 0; i < K; ++i) out[i] = (double)x[i] * (double)gamma[i] * inv;
}

void kqo_swiglu(const float* gu, int64_t K, double* out) {
    for (int64_t i = 0; i < K; ++i) {
        const double g = (double)gu[i];
        out[i] = g / (1.0 + exp(-g)) * (double)gu[K + i];
    }
}

/* kqo_gemv with double activations (the output of a prologue). */
int kqo_gemv_x64(int fmt, const uint8_t* W, int64_t N, int64_t K, const double* x, double* y, double* sabs,
                 int nthreads) {
    int64_t bb = block_bytes(fmt);
    if (bb < 0 || K % 256 != 0) return -1;
    int64_t row_bytes = K / 256 * bb;
    int bad = 0;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel num_threads(nthreads)
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)K);
        if (!w) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(static)
        for (int64_t r = 0; r < N; ++r) {
            if (!w) continue;
            kqo_dequant_row(fmt, W + r * row_bytes, K, w);
            double acc = 0.0, acc_abs = 0.0;
            for (int64_t i = 0; i < K; ++i) {
                double p = w[i] * x[i];
                acc += p;
                acc_abs += fabs(p);
            }
            y[r] = acc;
            if (sabs) sabs[r] = acc_abs;
        }
        free(w);
    }
    return bad ? -2 : 0;
}

/* Logical fields of `nblocks` consecutive super-blocks, in the layout the
 * bit-exact unpack check compares:
 *   q[256*b + i]      quant of weight i (Q4_K 0..15, Q5_K 0..31, Q6_K 0..63,
 *                     before -32)
 *   sc[16*b + j]      Q4_K, Q5_K: sc_0..7 then m_0..7; Q6_K: the 16 signed
 *                     scales as two's-complement bytes
 *                     Q2_K: the 16 raw scale bytes (scale | min << 4);
 *                     Q3_K: the 16 6-bit scales v (before -32);
 *                     Q8_0: the 8 blocks' fp16 scales, raw (little-endian)
 *                     (Q2_K quants 0..3; Q3_K values -4..3 and Q8_0 quants
 *                     as two's-complement bytes)
 *   d[2*b], d[2*b+1]  Q4_K, Q5_K, Q2_K: d, dmin; Q6_K, Q3_K: d, 0 (fp16
 *                     widened exactly); Q8_0: 0, 0
 * (For Q8_0, b counts units of eight 34-byte blocks, 256 weights.) */
int kqo_unpack(int fmt, const uint8_t* W, int64_t nblocks, uint8_t* q, uint8_t* sc, float* d) {
    int64_t bb = block_bytes(fmt);
    if (bb < 0) return -1;
    for (int64_t b = 0; b < nblocks; ++b) {
        const uint8_t* blk = W + b * bb;
        if (fmt == KQO_Q4_K || fmt == KQO_Q5_K) {
            double dd, dm;
            if (fmt == KQO_Q4_K) kqo_q4k_unpack(blk, q + 256 * b, sc + 16 * b, sc + 16 * b + 8, &dd, &dm);
            else kqo_q5k_unpack(blk, q + 256 * b, sc + 16 * b, sc + 16 * b + 8, &dd, &dm);
            d[2 * b] = (float)dd;
            d[2 * b + 1] = (float)dm;
        } else if (fmt == KQO_Q2_K) {
            uint8_t s2[16], m2[16];
            double dd, dm;
            kqo_q2k_unpack(blk, q + 256 * b, s2, m2, &dd, &dm);
            for (int g = 0; g < 16; ++g) sc[16 * b + g] = (uint8_t)(s2[g] | (m2[g] << 4));
            d[2 * b] = (float)dd;
            d[2 * b + 1] = (float)dm;
        } else if (fmt == KQO_Q3_K) {
            double dd;
            kqo_q3k_unpack(blk, (int8_t*)(q + 256 * b), sc + 16 * b, &dd);
            d[2 * b] = (float)dd;
            d[2 * b + 1] = 0.0f;
        } else if (fmt == KQO_Q8_0) {
            double dd[8];
            kqo_q80_unpack(blk, (int8_t*)(q + 256 * b), dd);
            for (int j = 0; j < 8; ++j) {  /* the raw fp16 scale bits */
                sc[16 * b + 2 * j] = blk[34 * j];
                sc[16 * b + 2 * j + 1] = blk[34 * j + 1];
            }
            d[2 * b] = 0.0f;
            d[2 * b + 1] = 0.0f;
        } else {
            double dd;
            kqo_q6k_unpack(blk, q + 256 * b, (int8_t*)(sc + 16 * b), &dd);
            d[2 * b] = (float)dd;
            d[2 * b + 1] = 0.0f;
        }
    }
    return 0;
}
