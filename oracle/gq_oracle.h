/*
 * gq_oracle.h -- plain CPU oracle for the Q4_0 and super-block K-quant
 * ("ksb") formats and their dequantize-fused matrix products.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path includes, links or
 * calls this code; only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no source with the CUDA library.
 *
 * Sources (web pages, by title and section):
 *   [Q40]  "GGUF 量化内幕 第4章：Q4_0 块量化格式解析" (sxkj888.cn), sections
 *          4.1.2 (18-byte block), 4.2.1 (lo/hi nibble split), 4.2.2 (q-8),
 *          4.3 (dequantization), 4.4 (the llama.cpp reference quantizer),
 *          4.5 (outlier demo).
 *   [KQ]   "GGUF K-quants" (hugo-blog, 2025/gguf-k-quants), sections
 *          "套娃" (super-block, INT8 sub-scales against an FP16 super-scale,
 *          worked 8-scale table) and the 4 + 80/256 bits-per-weight table.
 * Where the pages leave a rounding rule open, the rule fixed for this build is
 * used: d = FP16(absmax/7) with an IEEE fp32 quotient, and
 * code = clamp(rint(x/d) + 8, 0, 15) with round-half-to-even.
 */
#ifndef GQ_ORACLE_H
#define GQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status flags ORed together by the quantizers. */
#define ORC_OK        0
#define ORC_NONFINITE 1  /* a NaN or an infinity was seen in the block      */
#define ORC_RANGE     2  /* a scale overflowed FP16 (absmax/7 >= 65520)     */

/* Formats */
#define ORC_FMT_Q4_0 0
#define ORC_FMT_KSB  1

/* Element types of activations */
#define ORC_F32  0
#define ORC_F16  1
#define ORC_BF16 2

/* Q4_0 rounding rules.  ORC_RULE_ABSMAX7 is the rule fixed for this build;
 * ORC_RULE_LLAMA is the signed max/-8 rule of the page's reference quantizer
 * ([Q40] 4.4), kept for the format-compatibility checks. */
#define ORC_RULE_ABSMAX7 0
#define ORC_RULE_LLAMA   1

/* IEEE 754 binary16 <-> binary32, round to nearest even, subnormals kept. */
uint16_t orc_f32_to_f16(float f);
float    orc_f16_to_f32(uint16_t h);
/* bfloat16 <-> binary32 (RNE on the way down). */
uint16_t orc_f32_to_bf16(float f);
float    orc_bf16_to_f32(uint16_t h);
/* Bulk versions, used to pin the converters against other implementations. */
void orc_f32_to_f16_array(const float* x, int64_t n, uint16_t* out);
void orc_f16_to_f32_array(const uint16_t* h, int64_t n, float* out);

/* Bytes of n weights in each format; 0 if n is not a whole number of blocks. */
int64_t orc_q4_0_bytes(int64_t n);
int64_t orc_ksb_bytes(int64_t n);

/* Quantize n fp32 values (n a multiple of 32 / 256).  Returns ORed flags. */
int orc_quantize_q4_0(const float* x, int64_t n, uint8_t* out, int rule);
int orc_quantize_ksb(const float* x, int64_t n, uint8_t* out);

/* The super-scale step of [KQ] on its own: eight FP16 sub-scales in, the FP16
 * super-scale and the eight INT8 codes out. */
void orc_ksb_scale_step(const uint16_t d16[8], uint16_t* S16, int8_t q[8]);

/* Dequantize n values. */
void orc_dequantize_q4_0(const uint8_t* q, int64_t n, float* out);
void orc_dequantize_ksb(const uint8_t* q, int64_t n, float* out);

/* Y[b][m] = sum_k What[m][k] * X[b][k] in fp64 over the dequantized weights.
 * W holds M rows of K weights, each row quantized along K and stored
 * contiguously.  X holds B rows of K activations of element type xt (raw
 * bits: float, binary16 or bfloat16).  bound[b][m] = sum_k |What||X|.
 * Either output may be NULL. */
void orc_gemm(int fmt, const uint8_t* W, int64_t M, int64_t K,
              const void* X, int xt, int64_t B,
              double* Y, double* bound);

/* Same product restricted to the listed rows (for sampled checks of large
 * matrices): Y[b][i] and bound[b][i] refer to row rows[i]. */
void orc_gemm_rows(int fmt, const uint8_t* W, int64_t M, int64_t K,
                   const void* X, int xt, int64_t B,
                   const int64_t* rows, int64_t nrows,
                   double* Y, double* bound);

/* Tiled storage (this library's own device layout; the pages have no
 * counterpart): a permutation of the canonical bytes in which every tile of
 * 16 rows x 64 Q4_0 blocks (16 rows x 8 super-blocks for ksb) is contiguous
 * and arranged by the lanes that multiply it.  Rows are taken 16 at a time
 * (rows past M are zero); tile (g, c) of row group g and K-tile c starts at
 * byte g * 16 * rowbytes + c * 18432 (Q4_0) or c * 17664 (ksb); the last
 * K-tile of a row holds the remaining blocks.  For lane l = 4 * gg + t
 * (gg = 0..7, t = 0..3), "word t" of a block is its code bytes qs[4t..4t+3].
 *   Q4_0 tile of nb blocks: unit u = blocks 2u, 2u+1.
 *     codes at 512 u + 16 l: word t of block 2u of rows gg, gg+8, then of
 *       block 2u+1 of rows gg, gg+8 (4 bytes each);
 *     scales at 256 nb + 64 u + 4 r: d of blocks 2u, 2u+1 of row r.
 *   ksb tile of ns super-blocks: unit u = half u % 2 of super-block u / 2
 *     (sub-blocks j = 4 (u % 2) + h, h = 0..3).
 *     codes at 1024 u + 32 l + 8 h: word t of sub-block j of rows gg, gg+8;
 *     sub-scales at 2048 ns + 64 u + 4 r + h: q_j of row r;
 *     super-scales at 2176 ns + 32 (u / 2) + 2 r: S of row r.
 * Returns -1 when K is not a whole number of units (K % 64 for Q4_0,
 * K % 256 for ksb). */
int64_t orc_tiled_bytes(int fmt, int64_t M, int64_t K);
int orc_repack(int fmt, const uint8_t* W, int64_t M, int64_t K, uint8_t* out);
int orc_unrepack(int fmt, const uint8_t* T, int64_t M, int64_t K, uint8_t* out);

/* Number of threads the parallel loops above use. */
int orc_num_threads(void);
void orc_set_threads(int n);

#ifdef __cplusplus
}
#endif
#endif
