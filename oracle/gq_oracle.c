/*
 * gq_oracle.c -- plain, slow, scalar CPU oracle.  TEST INFRASTRUCTURE ONLY:
 * the CUDA library never includes, links or calls it, and it includes nothing
 * of the CUDA library.  Built by gcc with -O2 -fno-fast-math
 * -ffp-contract=off, so every fp32 operation below is one IEEE operation in
 * round-to-nearest-even, in the order written.
 *
 * Citations name the page and the section (see gq_oracle.h for the list):
 *   [Q40] the Q4_0 chapter, [KQ] the K-quants super-block post.
 */
#include "gq_oracle.h"

#include <math.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 from the standard's definition (not from any library).  */
/* ------------------------------------------------------------------------ */

static uint32_t bits_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float float_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* Round the integer m / 2^s to nearest, ties to even (s >= 1). */
static uint32_t shift_rne(uint32_t m, int s) {
    if (s >= 32) return 0;  /* m < 2^24, so the quotient is below one half */
    uint32_t q = m >> s;
    uint32_t rem = m & ((1u << s) - 1u);
    uint32_t half = 1u << (s - 1);
    if (rem > half || (rem == half && (q & 1u))) q += 1u;
    return q;
}

uint16_t orc_f32_to_f16(float f) {
    uint32_t u = bits_of(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t e = (u >> 23) & 0xFFu;
    uint32_t frac = u & 0x7FFFFFu;
    if (e == 0xFFu) {                        /* infinity or NaN */
        if (frac == 0) return sign | 0x7C00u;
        return (uint16_t)(sign | 0x7E00u | (frac >> 13));  /* quiet NaN */
    }
    if (e == 0) return sign;                 /* |f| < 2^-126: rounds to zero */
    uint32_t m = frac | 0x800000u;           /* value = m * 2^(e-150)        */
    int ue = (int)e - 127;                   /* unbiased exponent of f       */
    if (ue > 15) return sign | 0x7C00u;      /* at least 2^16: overflow      */
    if (ue >= -14) {
        /* normal binary16 range: keep 11 significant bits (drop 13).  A carry
         * out of the significand bumps the exponent, and from 2^15 * 2047/1024
         * upward into infinity, by plain integer addition. */
        uint32_t r = shift_rne(m, 13);       /* r in [1024, 2048]            */
        return (uint16_t)(sign | (((uint32_t)(ue + 14) << 10) + r));
    }
    /* subnormal binary16: value = r * 2^-24, r in [0, 1024] */
    uint32_t r = shift_rne(m, 126 - (int)e);
    return (uint16_t)(sign | r);
}

float orc_f16_to_f32(uint16_t h) {
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1Fu;
    uint32_t frac = h & 0x3FFu;
    if (e == 0x1Fu)                          /* infinity / NaN */
        return float_of(sign | 0x7F800000u | (frac << 13));
    if (e == 0) {                            /* zero or subnormal: frac*2^-24 */
        float v = (float)frac * float_of(0x33800000u);  /* 2^-24, exact */
        return float_of(bits_of(v) | sign);
    }
    return float_of(sign | ((e + 112u) << 23) | (frac << 13));
}

uint16_t orc_f32_to_bf16(float f) {
    uint32_t u = bits_of(f);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x7FFFFFu))
        return (uint16_t)((u >> 16) | 0x40u);            /* quiet NaN */
    uint32_t r = shift_rne(u & 0x7FFFFFFFu, 16);         /* carries are fine */
    return (uint16_t)(((u >> 16) & 0x8000u) | r);
}

float orc_bf16_to_f32(uint16_t h) { return float_of((uint32_t)h << 16); }

void orc_f32_to_f16_array(const float* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_f16(x[i]);
}
void orc_f16_to_f32_array(const uint16_t* h, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f16_to_f32(h[i]);
}

/* ------------------------------------------------------------------------ */
/* Sizes: [Q40] 4.1.2 -- 2-byte FP16 scale + 16 bytes of nibbles per 32      */
/* weights; [KQ] bits table -- 16-bit super-scale + 8 x 8-bit sub-scales +   */
/* 256 x 4-bit codes = 2 + 8 + 128 bytes per 256 weights.                    */
/* ------------------------------------------------------------------------ */

#define Q40_BLOCK 32
#define Q40_BYTES 18
#define KSB_BLOCK 256
#define KSB_BYTES 138

int64_t orc_q4_0_bytes(int64_t n) {
    if (n < 0 || n % Q40_BLOCK) return 0;
    return n / Q40_BLOCK * Q40_BYTES;
}
int64_t orc_ksb_bytes(int64_t n) {
    if (n < 0 || n % KSB_BLOCK) return 0;
    return n / KSB_BLOCK * KSB_BYTES;
}

static void put_u16le(uint8_t* p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static uint16_t get_u16le(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* One 4-bit code under the build's rule: clamp(rint(x/scale) + 8, 0, 15),
 * with the quotient rounded to fp32 first and rint rounding half to even.
 * A zero scale gives code 8 (zero). */
static int code_of(float x, float scale) {
    if (scale == 0.0f) return 8;
    float t = x / scale;
    if (!(fabsf(t) < 1e9f)) return 8;        /* non-finite input: flagged */
    int c = (int)rintf(t) + 8;
    if (c < 0) c = 0;
    if (c > 15) c = 15;
    return c;
}

/* Pack 32 codes: byte j carries code j in its low nibble and code j+16 in its
 * high nibble ([Q40] 4.2.1, the "lo-hi split", not even/odd). */
static void pack_32(const int c[32], uint8_t qs[16]) {
    for (int j = 0; j < 16; ++j)
        qs[j] = (uint8_t)(c[j] | (c[j + 16] << 4));
}

/* ------------------------------------------------------------------------ */
/* Q4_0 quantization                                                          */
/* ------------------------------------------------------------------------ */

static int quant_block_absmax7(const float* x, uint8_t* out) {
    int flags = ORC_OK;
    float a = 0.0f;
    for (int i = 0; i < Q40_BLOCK; ++i) {
        if (!isfinite(x[i])) flags |= ORC_NONFINITE;
        float v = fabsf(x[i]);
        if (v > a) a = v;
    }
    /* d = absmax / 7, fp32 quotient, then rounded to FP16 (build rule) */
    uint16_t d16 = orc_f32_to_f16(a / 7.0f);
    if ((d16 & 0x7FFFu) == 0x7C00u) flags |= ORC_RANGE;
    float d = orc_f16_to_f32(d16);
    int c[32];
    for (int i = 0; i < Q40_BLOCK; ++i) c[i] = code_of(x[i], d);
    put_u16le(out, d16);
    pack_32(c, out + 2);
    return flags;
}

/* The element of largest magnitude, with its sign; among equal magnitudes
 * the one seen first ([Q40] 4.4: the scan keeps its candidate unless a later
 * value is strictly larger in magnitude).  A block of zeros gives +0. */
static float signed_absmax_first(const float* x, int n) {
    float best = 0.0f;
    for (int i = 0; i < n; ++i)
        if (fabsf(x[i]) > fabsf(best)) best = x[i];
    return best;
}

/* One 4-bit code under the page's reference rule ([Q40] 4.4): the value is
 * multiplied by the inverse scale, shifted by 8.5 and truncated toward zero,
 * each operation rounded to fp32; the result is capped at 15.  Below zero
 * (only reachable through rounding) the code is 0. */
static int code_ref_rule(float x, float inv_d) {
    float shifted = x * inv_d;
    shifted = shifted + 8.5f;
    if (!(shifted >= 0.0f) || !(shifted < 1e9f)) return 0;
    int c = (int)shifted;
    return c > 15 ? 15 : c;
}

/* Block quantizer of the page's reference rule ([Q40] 4.4, demonstrated on
 * the outlier block of 4.5): the scale is d = vmax / -8 for the signed value
 * vmax of largest magnitude, so vmax itself lands on code 0; the inverse
 * scale is 1/d, or 0 for a zero scale (every code then 8). */
static int quant_block_llama(const float* x, uint8_t* out) {
    int flags = ORC_OK;
    for (int i = 0; i < Q40_BLOCK; ++i)
        if (!isfinite(x[i])) flags |= ORC_NONFINITE;
    const float d = signed_absmax_first(x, Q40_BLOCK) / -8.0f;
    const float inv_d = (d == 0.0f) ? 0.0f : 1.0f / d;
    const uint16_t d16 = orc_f32_to_f16(d);
    if ((d16 & 0x7FFFu) == 0x7C00u) flags |= ORC_RANGE;
    int c[32];
    for (int i = 0; i < Q40_BLOCK; ++i) c[i] = code_ref_rule(x[i], inv_d);
    put_u16le(out, d16);
    pack_32(c, out + 2);
    return flags;
}

int orc_quantize_q4_0(const float* x, int64_t n, uint8_t* out, int rule) {
    if (n < 0 || n % Q40_BLOCK) return -1;
    int64_t nb = n / Q40_BLOCK;
    int flags = ORC_OK;
#pragma omp parallel for reduction(| : flags) schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        const float* xb = x + b * Q40_BLOCK;
        uint8_t* ob = out + b * Q40_BYTES;
        flags |= (rule == ORC_RULE_LLAMA) ? quant_block_llama(xb, ob)
                                          : quant_block_absmax7(xb, ob);
    }
    return flags;
}

/* ------------------------------------------------------------------------ */
/* Super-block K-quant ([KQ] "套娃")                                          */
/* ------------------------------------------------------------------------ */

/* The eight FP16 sub-scales are themselves treated as weights: the symmetric
 * range [-max, max] is split into the INT8 buckets -127..127, so the
 * super-scale is S = (max - (-max)) / (127 - (-127)) = max / 127 (same real
 * number, hence the same correctly rounded fp32 quotient), stored as FP16;
 * each sub-scale becomes round(s / S).  Sub-scales are >= 0, so codes lie in
 * 0..127; the clamp only catches FP16 rounding of S downward. */
void orc_ksb_scale_step(const uint16_t d16[8], uint16_t* S16, int8_t q[8]) {
    float m = 0.0f;
    for (int j = 0; j < 8; ++j) {
        float dj = orc_f16_to_f32(d16[j]);
        if (dj > m) m = dj;
    }
    uint16_t s16 = orc_f32_to_f16(m / 127.0f);
    float S = orc_f16_to_f32(s16);
    for (int j = 0; j < 8; ++j) {
        float dj = orc_f16_to_f32(d16[j]);
        int v = 0;
        if (S != 0.0f && S < INFINITY) {
            float t = dj / S;
            v = (int)rintf(t);
            if (v < 0) v = 0;
            if (v > 127) v = 127;
        }
        q[j] = (int8_t)v;
    }
    *S16 = s16;
}

static int quant_superblock(const float* x, uint8_t* out) {
    int flags = ORC_OK;
    uint16_t d16[8];
    for (int j = 0; j < 8; ++j) {
        float a = 0.0f;
        for (int i = 0; i < 32; ++i) {
            float v = x[32 * j + i];
            if (!isfinite(v)) flags |= ORC_NONFINITE;
            if (fabsf(v) > a) a = fabsf(v);
        }
        /* each sub-block's own scale, FP16, by the build rule */
        d16[j] = orc_f32_to_f16(a / 7.0f);
        if ((d16[j] & 0x7FFFu) == 0x7C00u) flags |= ORC_RANGE;
    }
    uint16_t S16;
    int8_t q[8];
    orc_ksb_scale_step(d16, &S16, q);
    float S = orc_f16_to_f32(S16);
    put_u16le(out, S16);
    for (int j = 0; j < 8; ++j) out[2 + j] = (uint8_t)q[j];
    for (int j = 0; j < 8; ++j) {
        /* codes are taken against the scale the decoder will rebuild,
         * s~_j = S * q_j (an exact fp32 product), so stored codes and
         * stored scales agree */
        float st = S * (float)q[j];
        int c[32];
        for (int i = 0; i < 32; ++i) c[i] = code_of(x[32 * j + i], st);
        pack_32(c, out + 10 + 16 * j);
    }
    return flags;
}

int orc_quantize_ksb(const float* x, int64_t n, uint8_t* out) {
    if (n < 0 || n % KSB_BLOCK) return -1;
    int64_t nb = n / KSB_BLOCK;
    int flags = ORC_OK;
#pragma omp parallel for reduction(| : flags) schedule(static)
    for (int64_t b = 0; b < nb; ++b)
        flags |= quant_superblock(x + b * KSB_BLOCK, out + b * KSB_BYTES);
    return flags;
}

/* ------------------------------------------------------------------------ */
/* Dequantization                                                             */
/* ------------------------------------------------------------------------ */

/* [Q40] 4.3: y[j] = d * (lo(qs[j]) - 8), y[j+16] = d * (hi(qs[j]) - 8). */
static void dequant_q40_block(const uint8_t* blk, float* y) {
    float d = orc_f16_to_f32(get_u16le(blk));
    const uint8_t* qs = blk + 2;
    for (int j = 0; j < 16; ++j) {
        int lo = qs[j] & 0x0F;
        int hi = (qs[j] >> 4) & 0x0F;
        y[j] = d * (float)(lo - 8);
        y[j + 16] = d * (float)(hi - 8);
    }
}

/* [KQ]: the INT8 sub-scale times the super-scale rebuilds s~_j; each weight
 * is then s~_j * (code - 8) as in Q4_0.  Both products are exact in fp32. */
static void dequant_ksb_block(const uint8_t* blk, float* y) {
    float S = orc_f16_to_f32(get_u16le(blk));
    for (int j = 0; j < 8; ++j) {
        float st = S * (float)(int8_t)blk[2 + j];
        const uint8_t* qs = blk + 10 + 16 * j;
        for (int i = 0; i < 16; ++i) {
            int lo = qs[i] & 0x0F;
            int hi = (qs[i] >> 4) & 0x0F;
            y[32 * j + i] = st * (float)(lo - 8);
            y[32 * j + i + 16] = st * (float)(hi - 8);
        }
    }
}

void orc_dequantize_q4_0(const uint8_t* q, int64_t n, float* out) {
    int64_t nb = n / Q40_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b)
        dequant_q40_block(q + b * Q40_BYTES, out + b * Q40_BLOCK);
}

void orc_dequantize_ksb(const uint8_t* q, int64_t n, float* out) {
    int64_t nb = n / KSB_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b)
        dequant_ksb_block(q + b * KSB_BYTES, out + b * KSB_BLOCK);
}

/* ------------------------------------------------------------------------ */
/* Tiled storage: a byte permutation (layout in gq_oracle.h)                  */
/* ------------------------------------------------------------------------ */

static int64_t row_bytes(int fmt, int64_t K) {
    return fmt == ORC_FMT_KSB ? K / KSB_BLOCK * KSB_BYTES : K / Q40_BLOCK * Q40_BYTES;
}

int64_t orc_tiled_bytes(int fmt, int64_t M, int64_t K) {
    if (M < 0 || K < 0 || K % (fmt == ORC_FMT_KSB ? 256 : 64)) return -1;
    return (M + 15) / 16 * 16 * row_bytes(fmt, K);
}

/* Visit every canonical byte once: call f(tiled offset, canonical offset)
 * for each byte of each row group (rows past M give canonical offset -1). */
typedef void (*visit_fn)(int64_t tiled, int64_t canon, const uint8_t* src, uint8_t* dst);

static void visit_tiles(int fmt, int64_t M, int64_t K, visit_fn f, const uint8_t* src,
                        uint8_t* dst) {
    const int64_t rb = row_bytes(fmt, K);
    const int64_t groups = (M + 15) / 16;
    if (fmt == ORC_FMT_Q4_0) {
        const int64_t nblk = K / 32;
        for (int64_t g = 0; g < groups; ++g)
            for (int64_t c0 = 0; c0 < nblk; c0 += 64) {
                const int64_t nb = (nblk - c0 < 64) ? nblk - c0 : 64;
                const int64_t tile = g * 16 * rb + c0 * 16 * 18;
                for (int64_t u = 0; u < nb / 2; ++u) {
                    for (int l = 0; l < 32; ++l) {
                        const int gg = l / 4, t = l % 4;
                        const int64_t rows[4] = {16 * g + gg, 16 * g + gg + 8, 16 * g + gg,
                                                 16 * g + gg + 8};
                        const int64_t blks[4] = {c0 + 2 * u, c0 + 2 * u, c0 + 2 * u + 1,
                                                 c0 + 2 * u + 1};
                        for (int w = 0; w < 4; ++w)
                            for (int b = 0; b < 4; ++b) {
                                const int64_t canon = rows[w] < M
                                    ? rows[w] * rb + blks[w] * 18 + 2 + 4 * t + b : -1;
                                f(tile + 512 * u + 16 * l + 4 * w + b, canon, src, dst);
                            }
                    }
                    for (int r = 0; r < 16; ++r)
                        for (int h = 0; h < 2; ++h)
                            for (int b = 0; b < 2; ++b) {
                                const int64_t row = 16 * g + r;
                                const int64_t canon = row < M
                                    ? row * rb + (c0 + 2 * u + h) * 18 + b : -1;
                                f(tile + 256 * nb + 64 * u + 4 * r + 2 * h + b, canon, src, dst);
                            }
                }
            }
    } else {
        const int64_t nsb = K / 256;
        for (int64_t g = 0; g < groups; ++g)
            for (int64_t c0 = 0; c0 < nsb; c0 += 8) {
                const int64_t ns = (nsb - c0 < 8) ? nsb - c0 : 8;
                const int64_t tile = g * 16 * rb + c0 * 16 * 138;
                for (int64_t u = 0; u < 2 * ns; ++u) {
                    const int64_t sb = c0 + u / 2;
                    for (int l = 0; l < 32; ++l) {
                        const int gg = l / 4, t = l % 4;
                        for (int h = 0; h < 4; ++h) {
                            const int64_t j = 4 * (u % 2) + h;
                            for (int w = 0; w < 2; ++w) {
                                const int64_t row = 16 * g + gg + 8 * w;
                                for (int b = 0; b < 4; ++b) {
                                    const int64_t canon = row < M
                                        ? row * rb + sb * 138 + 10 + 16 * j + 4 * t + b : -1;
                                    f(tile + 1024 * u + 32 * l + 8 * h + 4 * w + b, canon, src, dst);
                                }
                            }
                        }
                    }
                    for (int r = 0; r < 16; ++r)
                        for (int h = 0; h < 4; ++h) {
                            const int64_t row = 16 * g + r;
                            const int64_t canon = row < M
                                ? row * rb + sb * 138 + 2 + 4 * (u % 2) + h : -1;
                            f(tile + 2048 * ns + 64 * u + 4 * r + h, canon, src, dst);
                        }
                }
                for (int64_t s = 0; s < ns; ++s)
                    for (int r = 0; r < 16; ++r)
                        for (int b = 0; b < 2; ++b) {
                            const int64_t row = 16 * g + r;
                            const int64_t canon = row < M ? row * rb + (c0 + s) * 138 + b : -1;
                            f(tile + 2176 * ns + 32 * s + 2 * r + b, canon, src, dst);
                        }
            }
    }
}

static void put_tiled(int64_t tiled, int64_t canon, const uint8_t* src, uint8_t* dst) {
    dst[tiled] = canon >= 0 ? src[canon] : 0;
}
static void get_tiled(int64_t tiled, int64_t canon, const uint8_t* src, uint8_t* dst) {
    if (canon >= 0) dst[canon] = src[tiled];
}

int orc_repack(int fmt, const uint8_t* W, int64_t M, int64_t K, uint8_t* out) {
    if (orc_tiled_bytes(fmt, M, K) < 0) return -1;
    visit_tiles(fmt, M, K, put_tiled, W, out);
    return 0;
}

int orc_unrepack(int fmt, const uint8_t* T, int64_t M, int64_t K, uint8_t* out) {
    if (orc_tiled_bytes(fmt, M, K) < 0) return -1;
    visit_tiles(fmt, M, K, get_tiled, T, out);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Matrix products over the dequantized weights, fp64                        */
/* ------------------------------------------------------------------------ */

static double widen(const void* X, int xt, int64_t i) {
    switch (xt) {
    case ORC_F16:  return (double)orc_f16_to_f32(((const uint16_t*)X)[i]);
    case ORC_BF16: return (double)orc_bf16_to_f32(((const uint16_t*)X)[i]);
    default:       return (double)((const float*)X)[i];
    }
}

static void dequant_row(int fmt, const uint8_t* W, int64_t K, int64_t m, float* w) {
    if (fmt == ORC_FMT_KSB) {
        const uint8_t* row = W + m * (K / KSB_BLOCK) * KSB_BYTES;
        for (int64_t b = 0; b < K / KSB_BLOCK; ++b)
            dequant_ksb_block(row + b * KSB_BYTES, w + b * KSB_BLOCK);
    } else {
        const uint8_t* row = W + m * (K / Q40_BLOCK) * Q40_BYTES;
        for (int64_t b = 0; b < K / Q40_BLOCK; ++b)
            dequant_q40_block(row + b * Q40_BYTES, w + b * Q40_BLOCK);
    }
}

#include <stdlib.h>

void orc_gemm_rows(int fmt, const uint8_t* W, int64_t M, int64_t K,
                   const void* X, int xt, int64_t B,
                   const int64_t* rows, int64_t nrows,
                   double* Y, double* bound) {
    (void)M;
    double* xd = (double*)malloc(sizeof(double) * (size_t)(B * K));
    for (int64_t i = 0; i < B * K; ++i) xd[i] = widen(X, xt, i);
#pragma omp parallel
    {
        float* w = (float*)malloc(sizeof(float) * (size_t)K);
#pragma omp for schedule(static)
        for (int64_t i = 0; i < nrows; ++i) {
            dequant_row(fmt, W, K, rows[i], w);
            for (int64_t b = 0; b < B; ++b) {
                const double* xb = xd + b * K;
                double s = 0.0, a = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double p = (double)w[k] * xb[k];   /* exact in fp64 */
                    s += p;
                    a += fabs(p);
                }
                if (Y) Y[b * nrows + i] = s;
                if (bound) bound[b * nrows + i] = a;
            }
        }
        free(w);
    }
    free(xd);
}

void orc_gemm(int fmt, const uint8_t* W, int64_t M, int64_t K,
              const void* X, int xt, int64_t B,
              double* Y, double* bound) {
    int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)(M > 0 ? M : 1));
    for (int64_t m = 0; m < M; ++m) rows[m] = m;
    orc_gemm_rows(fmt, W, M, K, X, xt, B, rows, M, Y, bound);
    free(rows);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the parallel loops that follow (timing runs only; results do
 * not depend on it: every output is one thread's fp64 loop). */
void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
