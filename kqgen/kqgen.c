/*
 * kqgen — seeded synthetic inputs for the K-quant GEMV workloads.
 *
 * This module only DRAWS logical values (quants, 6-bit scales/mins, int8
 * scales, fp16 block scales, fp32 activations, expert ids) and ENCODES them
 * into the GGUF K-quant super-block byte layout.  It holds none of the
 * method's arithmetic: no dequantisation, no dot product.  Both the CPU
 * oracle and the CUDA path consume its bytes; neither depends on the other.
 *
 * Randomness: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014), used counter-style: draw i of stream
 * `key` is the output of a SplitMix64 generator seeded with `key` after i+1
 * steps, i.e. mix(key + (i+1)*gamma).  That makes every super-block
 * independently addressable, so large tensors fill in parallel and give the
 * same bytes for any thread count.
 * Normals: Box-Muller in double precision, then rounded (fp32 for x, fp16
 * round-to-nearest-even for block scales).
 *
 * Block layouts (GGUF K-quants; the Q4_K fill is the one the workload
 * specification gives: quants uniform 0..15, scales/mins uniform 0..63,
 * d and dmin = |N(0,1)|*1e-3 rounded to fp16; Q6_K "seeded the same way":
 * quants uniform over the 6-bit range 0..63, scales uniform -64..63):
 *
 *   Q4_K, 144 B: [0,2) d fp16 | [2,4) dmin fp16 | [4,16) 12 scale bytes |
 *                [16,144) 128 quant bytes.
 *     Scale bytes: for j<4, byte j low 6 bits = sc_j, byte j+4 low 6 bits =
 *     m_j.  For j>=4, byte j+4 holds sc_j's low 4 bits (low nibble) and m_j's
 *     low 4 bits (high nibble); sc_j's top 2 bits sit in bits 6-7 of byte j-4,
 *     m_j's top 2 bits in bits 6-7 of byte j.
 *     Quant bytes: chunk c (0..3) of 32 bytes; byte 32c+l carries weight
 *     64c+l in its low nibble and weight 64c+32+l in its high nibble.
 *   Q5_K, 176 B: [0,2) d fp16 | [2,4) dmin fp16 | [4,16) 12 scale bytes
 *                (packed as Q4_K) | [16,48) qh | [48,176) 128 quant bytes.
 *     Weight 64c+l (l<32, c<4) has its low 4 bits in the low nibble of quant
 *     byte 32c+l and its 5th bit in bit 2c of qh[l]; weight 64c+32+l has its
 *     low 4 bits in the high nibble of the same byte and its 5th bit in bit
 *     2c+1 of qh[l].  The fill draws quants uniform over 0..31, the rest as
 *     Q4_K.
 *   Q2_K, 84 B: [0,16) scale bytes | [16,80) 64 quant bytes | [80,82) d fp16 |
 *                [82,84) dmin fp16.
 *     Scale byte j (j<16, the 16-weight sub-block j): low nibble scale,
 *     high nibble min.  Weight 128n+32j+l (n<2, j<4, l<32) is bits 2j..2j+1
 *     of quant byte 32n+l.  The fill draws quants uniform over 0..3, scales
 *     and mins over 0..15, d and dmin as Q4_K.
 *   Q3_K, 110 B: [0,32) hmask | [32,96) 64 quant bytes | [96,108) 12 scale
 *                bytes | [108,110) d fp16.
 *     Weight 128n+32j+l has its low 2 bits at bits 2j..2j+1 of quant byte
 *     32n+l and its third bit at bit 4n+j of hmask[l]; its value is
 *     (low | third << 2) - 4, in -4..3.  Sub-block j (16 weights) has a
 *     6-bit scale v_j, used as v_j - 32: its low 4 bits are the low nibble
 *     of scale byte j (j<8) or the high nibble of byte j-8 (j>=8), its top
 *     2 bits are bits 2(j/4)..2(j/4)+1 of byte 8 + j%4.  The fill draws the
 *     values uniform over -4..3, v_j over 0..63, d as Q4_K.
 *   Q8_0, 34 B per 32 weights: [0,2) d fp16 | [2,34) 32 int8 quants;
 *     w = d*q.  Handled in units of 8 blocks (256 weights, 272 B), like the
 *     super-blocks of the K-quants.  The fill draws quants uniform over the
 *     whole int8 range -128..127 and d as Q4_K.
 *   Q6_K, 210 B: [0,128) ql | [128,192) qh | [192,208) int8 scales |
 *                [208,210) d fp16.
 *     Half h (0..1) covers weights 128h..128h+127.  For l<32 and t<4, weight
 *     128h+32t+l has low 4 bits in ql[64h+l+32*(t&1)] (low nibble if t<2,
 *     high nibble otherwise) and top 2 bits in bits 2t..2t+1 of qh[32h+l].
 *     Weight i uses scale byte i/16.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define KQG_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t kqg_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Draw number `ctr` (0-based) of the SplitMix64 stream seeded with `key`. */
static inline uint64_t kqg_draw(uint64_t key, uint64_t ctr) {
    return kqg_mix(key + (ctr + 1) * KQG_GAMMA);
}

uint64_t kqg_splitmix64(uint64_t key, uint64_t ctr) { return kqg_draw(key, ctr); }

/* Seed of one tensor of a workload: mixes the workload seed, the layer and
 * the matrix id, so every tensor gets an independent stream. */
uint64_t kqg_tensor_seed(uint64_t base, uint64_t layer, uint64_t matrix) {
    return kqg_mix(base ^ (layer * 1000003ULL) ^ (matrix * 0x100000001B3ULL));
}

/* Uniform in (0,1] and [0,1) with 53 random bits. */
static inline double kqg_u01_open0(uint64_t r) { return ((double)(r >> 11) + 1.0) * 0x1.0p-53; }
static inline double kqg_u01(uint64_t r) { return (double)(r >> 11) * 0x1.0p-53; }

static void kqg_box_muller(uint64_t key, uint64_t ctr, double* z0, double* z1) {
    const double two_pi = 6.283185307179586476925286766559;
    double u1 = kqg_u01_open0(kqg_draw(key, ctr));
    double u2 = kqg_u01(kqg_draw(key, ctr + 1));
    double r = sqrt(-2.0 * log(u1));
    *z0 = r * cos(two_pi * u2);
    *z1 = r * sin(two_pi * u2);
}

/* IEEE binary16 encoding of a double, round to nearest, ties to even.
 * Overflow gives +-inf, NaN gives a quiet NaN, subnormals are kept. */
uint16_t kqg_f16_bits(double v) {
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v)) return 0x7E00;
    if (a >= 65520.0) return sign | 0x7C00;              /* rounds past 65504 */
    if (a < 0x1.0p-14) {                                  /* subnormal or zero */
        double m = nearbyint(a * 0x1.0p24);               /* units of 2^-24 */
        return sign | (uint16_t)m;                        /* m==1024 is 0x0400 */
    }
    int ex;
    frexp(a, &ex);                                        /* a = f*2^ex, f in [0.5,1) */
    int e = ex - 1;                                       /* a in [2^e, 2^(e+1)) */
    double mant = nearbyint((ldexp(a, -e) - 1.0) * 1024.0);
    if (mant >= 1024.0) { mant = 0.0; e += 1; }
    if (e + 15 >= 31) return sign | 0x7C00;
    return sign | (uint16_t)(((e + 15) << 10) | (int)mant);
}

/* ---------------------------------------------------------------- Q4_K */

/* Logical values of super-block `b` of stream `key`. */
static void kqg_q4k_draw_block(uint64_t key, uint64_t b, uint8_t q[256], uint8_t sc[8],
                               uint8_t m[8], uint16_t* d, uint16_t* dmin) {
    const uint64_t base = b * 32;
    for (int k = 0; k < 16; ++k) {
        uint64_t r = kqg_draw(key, base + k);
        for (int i = 0; i < 16; ++i) q[16 * k + i] = (uint8_t)((r >> (4 * i)) & 15);
    }
    uint64_t rs = kqg_draw(key, base + 16), rm = kqg_draw(key, base + 17);
    for (int j = 0; j < 8; ++j) {
        sc[j] = (uint8_t)((rs >> (6 * j)) & 63);
        m[j] = (uint8_t)((rm >> (6 * j)) & 63);
    }
    double z0, z1;
    kqg_box_muller(key, base + 18, &z0, &z1);
    *d = kqg_f16_bits(fabs(z0) * 1e-3);
    *dmin = kqg_f16_bits(fabs(z1) * 1e-3);
}

static void kqg_q4k_pack_block(const uint8_t q[256], const uint8_t sc[8], const uint8_t m[8],
                               uint16_t d, uint16_t dmin, uint8_t* out) {
    out[0] = (uint8_t)(d & 0xFF);
    out[1] = (uint8_t)(d >> 8);
    out[2] = (uint8_t)(dmin & 0xFF);
    out[3] = (uint8_t)(dmin >> 8);
    uint8_t* s = out + 4;
    for (int j = 0; j < 4; ++j) {
        s[j] = (uint8_t)((sc[j] & 63) | (((sc[j + 4] >> 4) & 3) << 6));
        s[j + 4] = (uint8_t)((m[j] & 63) | (((m[j + 4] >> 4) & 3) << 6));
        s[j + 8] = (uint8_t)((sc[j + 4] & 15) | ((m[j + 4] & 15) << 4));
    }
    uint8_t* qs = out + 16;
    for (int c = 0; c < 4; ++c)
        for (int l = 0; l < 32; ++l)
            qs[32 * c + l] = (uint8_t)((q[64 * c + l] & 15) | ((q[64 * c + 32 + l] & 15) << 4));
}

/* Draw logical values for `nblocks` super-blocks (for tests and pins). */
void kqg_q4k_draw(uint64_t key, int64_t nblocks, uint8_t* q, uint8_t* sc, uint8_t* m,
                  uint16_t* d, uint16_t* dmin) {
    for (int64_t b = 0; b < nblocks; ++b)
        kqg_q4k_draw_block(key, (uint64_t)b, q + 256 * b, sc + 8 * b, m + 8 * b, d + b, dmin + b);
}

/* Encode logical values into 144-byte super-blocks. */
void kqg_q4k_pack(int64_t nblocks, const uint8_t* q, const uint8_t* sc, const uint8_t* m,
                  const uint16_t* d, const uint16_t* dmin, uint8_t* out) {
    for (int64_t b = 0; b < nblocks; ++b)
        kqg_q4k_pack_block(q + 256 * b, sc + 8 * b, m + 8 * b, d[b], dmin[b], out + 144 * b);
}

/* Draw and encode blocks [b0, b0+nblocks) of stream `key` straight into
 * `out` (nblocks*144 bytes), in parallel over blocks. */
void kqg_q4k_fill(uint64_t key, int64_t b0, int64_t nblocks, uint8_t* out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        uint8_t q[256], sc[8], m[8];
        uint16_t d, dmin;
        kqg_q4k_draw_block(key, (uint64_t)(b0 + b), q, sc, m, &d, &dmin);
        kqg_q4k_pack_block(q, sc, m, d, dmin, out + 144 * b);
    }
}

/* ---------------------------------------------------------------- Q5_K */

/* Logical values of super-block `b` of stream `key`: 5-bit quants, then the
 * scales, mins and block scales drawn as for Q4_K. */
static void kqg_q5k_draw_block(uint64_t key, uint64_t b, uint8_t q[256], uint8_t sc[8],
                               uint8_t m[8], uint16_t* d, uint16_t* dmin) {
    const uint64_t base = b * 32;
    for (int i = 0; i < 256; ++i) {
        uint64_t r = kqg_draw(key, base + (uint64_t)(i / 12));
        q[i] = (uint8_t)((r >> (5 * (i % 12))) & 31);
    }
    uint64_t rs = kqg_draw(key, base + 22), rm = kqg_draw(key, base + 23);
    for (int j = 0; j < 8; ++j) {
        sc[j] = (uint8_t)((rs >> (6 * j)) & 63);
        m[j] = (uint8_t)((rm >> (6 * j)) & 63);
    }
    double z0, z1;
    kqg_box_muller(key, base + 24, &z0, &z1);
    *d = kqg_f16_bits(fabs(z0) * 1e-3);
    *dmin = kqg_f16_bits(fabs(z1) * 1e-3);
}

static void kqg_q5k_pack_block(const uint8_t q[256], const uint8_t sc[8], const uint8_t m[8],
                               uint16_t d, uint16_t dmin, uint8_t* out) {
    out[0] = (uint8_t)(d & 0xFF);
    out[1] = (uint8_t)(d >> 8);
    out[2] = (uint8_t)(dmin & 0xFF);
    out[3] = (uint8_t)(dmin >> 8);
    uint8_t* s = out + 4;
    for (int j = 0; j < 4; ++j) {
        s[j] = (uint8_t)((sc[j] & 63) | (((sc[j + 4] >> 4) & 3) << 6));
        s[j + 4] = (uint8_t)((m[j] & 63) | (((m[j + 4] >> 4) & 3) << 6));
        s[j + 8] = (uint8_t)((sc[j + 4] & 15) | ((m[j + 4] & 15) << 4));
    }
    uint8_t* qh = out + 16;
    uint8_t* qs = out + 48;
    memset(qh, 0, 32);
    for (int c = 0; c < 4; ++c)
        for (int l = 0; l < 32; ++l) {
            const uint8_t lo = q[64 * c + l] & 31, hi = q[64 * c + 32 + l] & 31;
            qs[32 * c + l] = (uint8_t)((lo & 15) | ((hi & 15) << 4));
            qh[l] |= (uint8_t)(((lo >> 4) << (2 * c)) | ((hi >> 4) << (2 * c + 1)));
        }
}

void kqg_q5k_draw(uint64_t key, int64_t nblocks, uint8_t* q, uint8_t* sc, uint8_t* m,
                  uint16_t* d, uint16_t* dmin) {
    for (int64_t b = 0; b < nblocks; ++b)
        kqg_q5k_draw_block(key, (uint64_t)b, q + 256 * b, sc + 8 * b, m + 8 * b, d + b, dmin + b);
}

void kqg_q5k_pack(int64_t nblocks, const uint8_t* q, const uint8_t* sc, const uint8_t* m,
                  const uint16_t* d, const uint16_t* dmin, uint8_t* out) {
    for (int64_t b = 0; b < nblocks; ++b)
        kqg_q5k_pack_block(q + 256 * b, sc + 8 * b, m + 8 * b, d[b], dmin[b], out + 176 * b);
}

void kqg_q5k_fill(uint64_t key, int64_t b0, int64_t nblocks, uint8_t* out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        uint8_t q[256], sc[8], m[8];
        uint16_t d, dmin;
        kqg_q5k_draw_block(key, (uint64_t)(b0 + b), q, sc, m, &d, &dmin);
        kqg_q5k_pack_block(q, sc, m, d, dmin, out + 176 * b);
    }
}

/* ---------------------------------------------------------------- Q2_K */

static void kqg_q2k_draw_block(uint64_t key, uint64_t b, uint8_t q[256], uint8_t sc[16], uint8_t m[16],
                               uint16_t* d, uint16_t* dmin) {
    const uint64_t base = b * 32;
    for (int k = 0; k < 8; ++k) {
        uint64_t r = kqg_draw(key, base + k);
        for (int i = 0; i < 32; ++i) q[32 * k + i] = (uint8_t)((r >> (2 * i)) & 3);
    }
    uint64_t r = kqg_draw(key, base + 8);
    for (int j = 0; j < 16; ++j) {
        sc[j] = (uint8_t)((r >> (4 * j)) & 15);
    }
    r = kqg_draw(key, base + 9);
    for (int j = 0; j < 16; ++j) m[j] = (uint8_t)((r >> (4 * j)) & 15);
    double z0, z1;
    kqg_box_muller(key, base + 10, &z0, &z1);
    *d = kqg_f16_bits(fabs(z0) * 1e-3);
    *dmin = kqg_f16_bits(fabs(z1) * 1e-3);
}

static void kqg_q2k_pack_block(const uint8_t q[256], const uint8_t sc[16], const uint8_t m[16], uint16_t d,
                               uint16_t dmin, uint8_t* out) {
    for (int j = 0; j < 16; ++j) out[j] = (uint8_t)((sc[j] & 15) | ((m[j] & 15) << 4));
    uint8_t* qs = out + 16;
    memset(qs, 0, 64);
    for (int n = 0; n < 2; ++n)
        for (int j = 0; j < 4; ++j)
            for (int l = 0; l < 32; ++l) qs[32 * n + l] |= (uint8_t)((q[128 * n + 32 * j + l] & 3) << (2 * j));
    out[80] = (uint8_t)(d & 0xFF);
    out[81] = (uint8_t)(d >> 8);
    out[82] = (uint8_t)(dmin & 0xFF);
    out[83] = (uint8_t)(dmin >> 8);
}

void kqg_q2k_draw(uint64_t key, int64_t nblocks, uint8_t* q, uint8_t* sc, uint8_t* m, uint16_t* d,
                  uint16_t* dmin) {
    for (int64_t b = 0; b < nblocks; ++b)
        kqg_q2k_draw_block(key, (uint64_t)b, q + 256 * b, sc + 16 * b, m + 16 * b, d + b, dmin + b);
}

void kqg_q2k_pack(int64_t nblocks, const uint8_t* q, const uint8_t* sc, const uint8_t* m, const uint16_t* d,
                  const uint16_t* dmin, uint8_t* out) {
    for (int64_t b = 0; b < nblocks; ++b)
        kqg_q2k_pack_block(q + 256 * b, sc + 16 * b, m + 16 * b, d[b], dmin[b], out + 84 * b);
}

void kqg_q2k_fill(uint64_t key, int64_t b0, int64_t nblocks, uint8_t* out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        uint8_t q[256], sc[16], m[16];
        uint16_t d, dmin;
        kqg_q2k_draw_block(key, (uint64_t)(b0 + b), q, sc, m, &d, &dmin);
        kqg_q2k_pack_block(q, sc, m, d, dmin, out + 84 * b);
    }
}

/* ---------------------------------------------------------------- Q3_K */

/* q: the signed values -4..3; v: the 6-bit scales 0..63 (used as v - 32). */
static void kqg_q3k_draw_block(uint64_t key, uint64_t b, int8_t q[256], uint8_t v[16], uint16_t* d) {
    const uint64_t base = b * 32;
    for (int i = 0; i < 256; ++i) {
        uint64_t r = kqg_draw(key, base + (uint64_t)(i / 21));
        q[i] = (int8_t)((int)((r >> (3 * (i % 21))) & 7) - 4);
    }
    uint64_t r0 = kqg_draw(key, base + 13), r1 = kqg_draw(key, base + 14);
    for (int j = 0; j < 16; ++j) {
        uint64_t r = j < 10 ? r0 : r1;
        v[j] = (uint8_t)((r >> (6 * (j < 10 ? j : j - 10))) & 63);
    }
    double z0, z1;
    kqg_box_muller(key, base + 15, &z0, &z1);
    *d = kqg_f16_bits(fabs(z0) * 1e-3);
}

static void kqg_q3k_pack_block(const int8_t q[256], const uint8_t v[16], uint16_t d, uint8_t* out) {
    uint8_t* hm = out;
    uint8_t* qs = out + 32;
    uint8_t* sb = out + 96;
    memset(out, 0, 108);
    for (int n = 0; n < 2; ++n)
        for (int j = 0; j < 4; ++j)
            for (int l = 0; l < 32; ++l) {
                const int u = q[128 * n + 32 * j + l] + 4;  /* 0..7 */
                qs[32 * n + l] |= (uint8_t)((u & 3) << (2 * j));
                hm[l] |= (uint8_t)(((u >> 2) & 1) << (4 * n + j));
            }
    for (int j = 0; j < 16; ++j) {
        const int lo = v[j] & 15, hi = (v[j] >> 4) & 3;
        if (j < 8) sb[j] |= (uint8_t)lo;
        else sb[j - 8] |= (uint8_t)(lo << 4);
        sb[8 + (j % 4)] |= (uint8_t)(hi << (2 * (j / 4)));
    }
    out[108] = (uint8_t)(d & 0xFF);
    out[109] = (uint8_t)(d >> 8);
}

void kqg_q3k_draw(uint64_t key, int64_t nblocks, int8_t* q, uint8_t* v, uint16_t* d) {
    for (int64_t b = 0; b < nblocks; ++b) kqg_q3k_draw_block(key, (uint64_t)b, q + 256 * b, v + 16 * b, d + b);
}

void kqg_q3k_pack(int64_t nblocks, const int8_t* q, const uint8_t* v, const uint16_t* d, uint8_t* out) {
    for (int64_t b = 0; b < nblocks; ++b) kqg_q3k_pack_block(q + 256 * b, v + 16 * b, d[b], out + 110 * b);
}

void kqg_q3k_fill(uint64_t key, int64_t b0, int64_t nblocks, uint8_t* out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        int8_t q[256];
        uint8_t v[16];
        uint16_t d;
        kqg_q3k_draw_block(key, (uint64_t)(b0 + b), q, v, &d);
        kqg_q3k_pack_block(q, v, d, out + 110 * b);
    }
}

/* ---------------------------------------------------------------- Q6_K */

static void kqg_q6k_draw_block(uint64_t key, uint64_t b, uint8_t q[256], int8_t s[16], uint16_t* d) {
    const uint64_t base = b * 32;
    for (int i = 0; i < 256; ++i) {
        uint64_t r = kqg_draw(key, base + (uint64_t)(i / 10));
        q[i] = (uint8_t)((r >> (6 * (i % 10))) & 63);
    }
    uint64_t r0 = kqg_draw(key, base + 26), r1 = kqg_draw(key, base + 27);
    for (int g = 0; g < 16; ++g) {
        uint64_t r = g < 9 ? r0 : r1;
        int sh = 7 * (g < 9 ? g : g - 9);
        s[g] = (int8_t)((int)((r >> sh) & 127) - 64);
    }
    double z0, z1;
    kqg_box_muller(key, base + 28, &z0, &z1);
    *d = kqg_f16_bits(fabs(z0) * 1e-3);
}

static void kqg_q6k_pack_block(const uint8_t q[256], const int8_t s[16], uint16_t d, uint8_t* out) {
    uint8_t* ql = out;
    uint8_t* qh = out + 128;
    memset(out, 0, 192);
    for (int h = 0; h < 2; ++h)
        for (int t = 0; t < 4; ++t)
            for (int l = 0; l < 32; ++l) {
                uint8_t v = q[128 * h + 32 * t + l] & 63;
                int li = 64 * h + l + 32 * (t & 1);
                if (t < 2) ql[li] |= (uint8_t)(v & 15);
                else ql[li] |= (uint8_t)((v & 15) << 4);
                qh[32 * h + l] |= (uint8_t)((v >> 4) << (2 * t));
            }
    for (int g = 0; g < 16; ++g) out[192 + g] = (uint8_t)s[g];
    out[208] = (uint8_t)(d & 0xFF);
    out[209] = (uint8_t)(d >> 8);
}

void kqg_q6k_draw(uint64_t key, int64_t nblocks, uint8_t* q, int8_t* s, uint16_t* d) {
    for (int64_t b = 0; b < nblocks; ++b)
        kqg_q6k_draw_block(key, (uint64_t)b, q + 256 * b, s + 16 * b, d + b);
}

void kqg_q6k_pack(int64_t nblocks, const uint8_t* q, const int8_t* s, const uint16_t* d, uint8_t* out) {
    for (int64_t b = 0; b < nblocks; ++b) kqg_q6k_pack_block(q + 256 * b, s + 16 * b, d[b], out + 210 * b);
}

void kqg_q6k_fill(uint64_t key, int64_t b0, int64_t nblocks, uint8_t* out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        uint8_t q[256];
        int8_t s[16];
        uint16_t d;
        kqg_q6k_draw_block(key, (uint64_t)(b0 + b), q, s, &d);
        kqg_q6k_pack_block(q, s, d, out + 210 * b);
    }
}

/* ---------------------------------------------------------------- Q8_0 */

/* One unit of 8 blocks: q the 256 int8 quants, d the 8 fp16 block scales. */
static void kqg_q80_draw_unit(uint64_t key, uint64_t u, int8_t q[256], uint16_t d[8]) {
    const uint64_t base = u * 40;
    for (int k = 0; k < 32; ++k) {
        uint64_t r = kqg_draw(key, base + k);
        for (int i = 0; i < 8; ++i) q[8 * k + i] = (int8_t)(uint8_t)((r >> (8 * i)) & 0xFF);
    }
    for (int j = 0; j < 8; j += 2) {
        double z0, z1;
        kqg_box_muller(key, base + 32 + j, &z0, &z1);
        d[j] = kqg_f16_bits(fabs(z0) * 1e-3);
        d[j + 1] = kqg_f16_bits(fabs(z1) * 1e-3);
    }
}

static void kqg_q80_pack_unit(const int8_t q[256], const uint16_t d[8], uint8_t* out) {
    for (int j = 0; j < 8; ++j) {
        uint8_t* blk = out + 34 * j;
        blk[0] = (uint8_t)(d[j] & 0xFF);
        blk[1] = (uint8_t)(d[j] >> 8);
        for (int i = 0; i < 32; ++i) blk[2 + i] = (uint8_t)q[32 * j + i];
    }
}

void kqg_q80_draw(uint64_t key, int64_t nunits, int8_t* q, uint16_t* d) {
    for (int64_t u = 0; u < nunits; ++u) kqg_q80_draw_unit(key, (uint64_t)u, q + 256 * u, d + 8 * u);
}

void kqg_q80_pack(int64_t nunits, const int8_t* q, const uint16_t* d, uint8_t* out) {
    for (int64_t u = 0; u < nunits; ++u) kqg_q80_pack_unit(q + 256 * u, d + 8 * u, out + 272 * u);
}

void kqg_q80_fill(uint64_t key, int64_t u0, int64_t nunits, uint8_t* out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t u = 0; u < nunits; ++u) {
        int8_t q[256];
        uint16_t d[8];
        kqg_q80_draw_unit(key, (uint64_t)(u0 + u), q, d);
        kqg_q80_pack_unit(q, d, out + 272 * u);
    }
}

/* ---------------------------------------------------------- activations */

/* x[i] ~ N(0,1) rounded to fp32; element i uses the Box-Muller pair i/2. */
void kqg_normal_f32(uint64_t key, int64_t n, float* out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t p = 0; p < (n + 1) / 2; ++p) {
        double z0, z1;
        kqg_box_muller(key, 2 * (uint64_t)p, &z0, &z1);
        out[2 * p] = (float)z0;
        if (2 * p + 1 < n) out[2 * p + 1] = (float)z1;
    }
}

/* ------------------------------------------------------------ routing */

/* `k` distinct expert ids drawn uniformly from 0..E-1 without replacement
 * (partial Fisher-Yates; index pick by the 64x64->128 multiply-shift map). */
int kqg_topk_ids(uint64_t key, int E, int k, int32_t* out) {
    if (E <= 0 || k < 0 || k > E || E > 4096) return -1;
    int32_t perm[4096];
    for (int i = 0; i < E; ++i) perm[i] = i;
    for (int i = 0; i < k; ++i) {
        uint64_t r = kqg_draw(key, (uint64_t)i);
        uint64_t span = (uint64_t)(E - i);
        int j = i + (int)(((unsigned __int128)r * span) >> 64);
        int32_t t = perm[i];
        perm[i] = perm[j];
        perm[j] = t;
        out[i] = perm[i];
    }
    return 0;
}
