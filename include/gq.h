/*
 * gq.h -- C ABI of libgq: GGUF-style 4-bit block weight quantization and the
 * dequantize-fused matrix-vector / small-batch matrix products that stream
 * those weights, as hand-written CUDA for sm_100a (NVIDIA B200).
 *
 * Formats (byte layouts are normative):
 *
 *   Q4_0 -- "GGUF 量化内幕 第4章：Q4_0 块量化格式解析", sections 4.1.2 and 4.2.1.
 *     32 weights in 18 bytes: bytes 0-1 the FP16 scale d (little-endian bit
 *     pattern), bytes 2-17 qs[0..15]; qs[j] holds the 4-bit code of weight j
 *     in its low nibble and of weight j+16 in its high nibble.  4.5 bits per
 *     weight.  Decoding (section 4.2.2 / 4.3): w = d * (code - 8).
 *
 *   KSB (super-block K-quant) -- "GGUF K-quants" (hugo-blog), section "套娃"
 *     and its bits table.  256 weights in 138 bytes: bytes 0-1 the FP16
 *     super-scale S, bytes 2-9 the INT8 sub-scales q_0..q_7, then 8 x 16 bytes
 *     of codes; sub-block j (weights 32j..32j+31) has its 16 code bytes at
 *     offset 10+16j with the Q4_0 low/high nibble split.  4.3125 bits per
 *     weight.  Decoding: w = (S * q_j) * (code - 8); both products are exact
 *     in fp32, so decoded values are bit-exact whatever the evaluation order.
 *
 *   Matrices: W has M rows of K weights; each row is quantized along K and its
 *   blocks are stored contiguously, rows one after another (row m starts at
 *   byte m * gq_q4_0_bytes(K) or m * gq_ksb_bytes(K)).
 *
 * Quantization rule (the pages leave the rounding open; this library fixes
 * it): d = FP16(absmax / 7) with an IEEE fp32 quotient rounded to nearest even
 * in FP16; code = clamp(rint(x / d) + 8, 0, 15) with an IEEE fp32 quotient and
 * rint rounding half to even; d == 0 gives code 8.  For KSB each sub-block's
 * d_j is formed this way, then S = FP16(max_j d_j / 127) (the post's
 * (max - (-max)) / (127 - (-127))), q_j = clamp(rint(d_j / S), 0, 127)
 * (0 when S == 0), and the codes are taken against the rebuilt scale S * q_j.
 *
 * Conventions shared by every entry point:
 *   - All data pointers are device (or managed) memory owned by the caller;
 *     the library allocates nothing and keeps no pointer after returning.
 *   - `stream` is a cudaStream_t passed as void* (NULL: the legacy default
 *     stream).  Every call is asynchronous on that stream; a returned GQ_OK
 *     means the arguments were valid and the launch was accepted.
 *   - Argument checks are synchronous and happen before any launch: on any
 *     error nothing is launched and nothing is written.
 *   - Data-dependent problems are reported through the optional device word
 *     `dev_status` (int*, may be NULL): the kernels atomically OR GQ_DEV_*
 *     bits into it; the caller zeroes it beforehand and reads it after the
 *     stream is synchronized (gq_status_from_dev() maps it to a gq_status).
 *     No kernel traps or asserts.
 *   - Base pointers must be 16-byte aligned (GQ_ERR_ALIGNMENT otherwise).
 *     Packed weights are read in whole 16-byte granules: bytes after the end
 *     of a packed buffer, up to the next 16-byte boundary, may be read and are
 *     ignored (such a granule never crosses a page, so this cannot fault).
 *   - Sizes of 0 are valid and launch nothing (a K of 0 writes y = 0).
 */
#ifndef GQ_H
#define GQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GQ_API __attribute__((visibility("default")))
#else
#define GQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define GQ_ABI_VERSION 1

typedef enum gq_status {
    GQ_OK = 0,
    GQ_ERR_INVALID_ARG = 1,  /* NULL pointer, negative size, bad enum      */
    GQ_ERR_SHAPE = 2,        /* size not a whole number of blocks, B range  */
    GQ_ERR_ALIGNMENT = 3,    /* pointer not 16-byte aligned                 */
    GQ_ERR_DTYPE = 4,        /* unsupported element type                    */
    GQ_ERR_NONFINITE = 5,    /* (device) NaN or infinity in quantizer input */
    GQ_ERR_RANGE = 6,        /* (device) a scale overflowed FP16            */
    GQ_ERR_TIMEOUT = 7,      /* (device) a bounded wait in a kernel gave up */
    GQ_ERR_CUDA = 8,         /* a CUDA launch or runtime call failed        */
    GQ_ERR_WORKSPACE = 9     /* workspace missing or too small              */
} gq_status;

typedef enum gq_dtype { GQ_F32 = 0, GQ_F16 = 1, GQ_BF16 = 2 } gq_dtype;
typedef enum gq_format { GQ_FMT_Q4_0 = 0, GQ_FMT_KSB = 1 } gq_format;

/* Bits ORed into *dev_status by the kernels. */
#define GQ_DEV_NONFINITE 1
#define GQ_DEV_RANGE     2
#define GQ_DEV_TIMEOUT   4

/* gq_gemv_* flags.
 * GQ_GEMV_PDL: launch with programmatic dependent launch.  The kernel may be
 *   scheduled while the previous kernel on the stream is still running; it
 *   streams W at once and waits for that kernel to finish before it reads x
 *   or writes y.  Use it only when W is not written by work still in flight
 *   on the stream (the usual case in decode, where weights are static). */
#define GQ_GEMV_PDL 1u

GQ_API int gq_abi_version(void);
GQ_API const char* gq_status_string(int status);
/* First error among the GQ_DEV_* bits of a device status word (GQ_OK if 0). */
GQ_API gq_status gq_status_from_dev(int dev_flags);

/* Packed bytes of n weights; 0 when n < 0 or n is not a whole number of
 * blocks (32 for Q4_0, 256 for KSB).  Q4_0 chapter 4.1.2: 18 bytes / 32;
 * K-quants bits table: 138 bytes / 256. */
GQ_API size_t gq_q4_0_bytes(int64_t n);
GQ_API size_t gq_ksb_bytes(int64_t n);

/* Quantize n fp32 values into Q4_0 blocks (Q4_0 chapter 4.4 for the shape of
 * the step, with this library's rounding rule above).
 *   x:   n floats, 16-byte aligned.  n % 32 == 0 (GQ_ERR_SHAPE otherwise).
 *   out: gq_q4_0_bytes(n) bytes, 16-byte aligned.
 *   dev_status: optional; GQ_DEV_NONFINITE if any input is NaN/inf (that
 *     block's bytes are then unspecified), GQ_DEV_RANGE if absmax/7 rounds to
 *     an FP16 infinity (the block then stores d = inf and codes 8). */
GQ_API gq_status gq_quantize_q4_0(const float* x, int64_t n, void* out,
                                  int* dev_status, void* stream);

/* gq_quantize_q4_0 with a choice of rule.  flags: 0 (the rule above, the same
 * as gq_quantize_q4_0) or GQ_QUANT_REF_RULE, the page's own reference
 * quantizer (Q4_0 chapter 4.4, the printed quantizer, and its outlier demo in
 * 4.5): the signed value of largest magnitude (the first on ties; +0 for a
 * block of zeros) sets d = max / -8, and with id = 1/d (0 when d is 0) each
 * code is min(15, trunc(x * id + 8.5)), the product and the sum each rounded
 * to fp32.  The stored scale is FP16(d).  Other flag bits give
 * GQ_ERR_INVALID_ARG.  Arguments and status as for gq_quantize_q4_0
 * (GQ_DEV_RANGE when FP16(d) is infinite). */
#define GQ_QUANT_REF_RULE 1u
GQ_API gq_status gq_quantize_q4_0_ex(const float* x, int64_t n, void* out, unsigned flags,
                                     int* dev_status, void* stream);

/* Quantize n fp32 values into KSB super-blocks (K-quants post, "套娃": the
 * eight sub-block scales are quantized to INT8 against an FP16 super-scale).
 *   n % 256 == 0; out holds gq_ksb_bytes(n) bytes.  dev_status as above. */
GQ_API gq_status gq_quantize_ksb(const float* x, int64_t n, void* out,
                                 int* dev_status, void* stream);

/* Decode n weights to fp32 (Q4_0 chapter 4.3: y = d * (code - 8); K-quants
 * post step 5: the INT8 sub-scale times S rebuilds the scale).  Output values
 * are exact, hence identical on every implementation.
 *   q: packed bytes (16-byte aligned); out: n floats (16-byte aligned). */
GQ_API gq_status gq_dequantize_q4_0(const void* q, int64_t n, float* out, void* stream);
GQ_API gq_status gq_dequantize_ksb(const void* q, int64_t n, float* out, void* stream);

/* Dequantize-fused matrix-vector product for decode, y = W_hat * x, for a
 * batch of 1..8 activation vectors (the matrix multiply that consumes the
 * decoded weights: Q4_0 chapter 4.3; the memory-bound decode step: the
 * TurboQuant W4A8 post, section 2.3).
 *   W: M x K packed (row layout above), 16-byte aligned.  K % 32 == 0 (Q4_0)
 *      or K % 256 == 0 (KSB).  M <= 2^31 - 1, K <= 2^24.
 *   x: [B][K] of x_dtype (GQ_F16, GQ_BF16 or GQ_F32), row-major.
 *   y: [B][M] of y_dtype (GQ_F16, GQ_BF16 or GQ_F32), row-major.
 *   B: 1..8 (0 launches nothing).
 * Arithmetic: products of the exact decoded weights with the exact inputs
 * (fp32 x is split exactly into three bfloat16 terms), accumulated in fp32,
 * rounded once to y_dtype.  When the B activation rows do not fit in one
 * SM's shared memory beside the weight pipeline (e.g. B >= 6 at K = 11008
 * with fp16 x), K is split over a thread-block cluster of 2..8 CTAs, each
 * holding its slice of x; their fp32 partial sums are added in rank order,
 * so results still do not depend on scheduling.
 * workspace / ws_bytes: optional caller-owned device scratch of at least
 *   gq_gemv_workspace_bytes(...) bytes (a size that does not depend on M or
 *   K), 256-byte aligned, all zero before its first use.  When that size is
 *   nonzero and a workspace is given, the call takes the batch-1 integer
 *   tensor-core path: x is split exactly into six signed 7-bit digit columns
 *   (every fp16 value is an integer multiple of 2^-24 below 2^16), the codes
 *   are multiplied as unsigned bytes with exact int32 sums, and only the fp32
 *   accumulation rounds.  The work is split evenly over the SMs; rows shared
 *   by two SMs are combined in a fixed order, so results do not depend on
 *   scheduling.  A successful call leaves the workspace ready for the next
 *   call (of any shape); after a call that fails or reports GQ_DEV_TIMEOUT,
 *   zero it again.  Calls that may run at the same time need separate
 *   workspaces.  NULL (or a size of 0) selects the path above.  A NaN or
 *   infinite x element makes every output of that path NaN (and sets
 *   GQ_DEV_NONFINITE).
 * flags: 0 or GQ_GEMV_PDL.  dev_status: optional, receives GQ_DEV_TIMEOUT if
 * a pipeline wait ever gives up. */
GQ_API size_t gq_gemv_workspace_bytes(int fmt, int64_t M, int64_t K, int64_t B, int x_dtype);
GQ_API gq_status gq_gemv_q4_0(const void* W, int64_t M, int64_t K,
                              const void* x, int x_dtype, int64_t B,
                              void* y, int y_dtype, void* workspace, size_t ws_bytes,
                              unsigned flags, int* dev_status, void* stream);
GQ_API gq_status gq_gemv_ksb(const void* W, int64_t M, int64_t K,
                             const void* x, int x_dtype, int64_t B,
                             void* y, int y_dtype, void* workspace, size_t ws_bytes,
                             unsigned flags, int* dev_status, void* stream);

/* Grouped dequantize-fused GEMV: several matrices that share K and the
 * activations, y_i[b][m] = sum_k W_hat_i[m][k] * x[b][k] for every descriptor
 * (the same operation as gq_gemv_q4_0 / gq_gemv_ksb, matrix by matrix).  It
 * serves a decode step that multiplies one activation vector by many weight
 * matrices: the whole-model stream, or the projections that read the same x.
 * The pages stream one matrix at a time; this entry point has no counterpart
 * on them.  One launch covers up to 256 matrices: its CTAs load x once and
 * stream the 16-row groups of all of them back to back, so there is no
 * launch gap and no repeated activation load between matrices.  Tables with
 * fewer than 8 row groups per SM give each output bit for bit what
 * gq_gemv_* gives; larger ones run a pipeline shaped for long streams whose
 * results differ from it only in the order of fp32 additions.
 *   mats:  count host descriptors {W, M, y} (read during the call only).  W as
 *          for gq_gemv_*, 16-byte aligned; y: [B][M] of y_dtype, 16-byte
 *          aligned.  M == 0 entries are skipped (W and y may then be NULL).
 *   K, x, x_dtype, B, y_dtype, flags, dev_status: as for gq_gemv_*, shared by
 *          all matrices (the integer path and its workspace do not apply).
 * Validation covers every descriptor before anything is launched; more than
 * 256 matrices are processed in several launches in stream order. */
typedef struct gq_gemv_desc {
    const void* W;
    int64_t M;
    void* y;
} gq_gemv_desc;
GQ_API gq_status gq_gemv_q4_0_grouped(const gq_gemv_desc* mats, int count, int64_t K,
                                      const void* x, int x_dtype, int64_t B, int y_dtype,
                                      unsigned flags, int* dev_status, void* stream);
GQ_API gq_status gq_gemv_ksb_grouped(const gq_gemv_desc* mats, int count, int64_t K,
                                     const void* x, int x_dtype, int64_t B, int y_dtype,
                                     unsigned flags, int* dev_status, void* stream);

/* Tiled storage (no counterpart on the pages: a device layout of this
 * library).  A byte permutation of the canonical rows in which every tile of
 * 16 rows x 64 Q4_0 blocks (16 rows x 8 super-blocks for KSB) is contiguous
 * and ordered by the lanes that multiply it, so that one bulk copy moves a
 * whole pipeline stage and each lane's code words are aligned 16-byte reads.
 * It holds the same bytes as the canonical rows (plus zero rows up to a
 * multiple of 16), and is made once, e.g. when a model is loaded.
 * Layout: rows are taken 16 at a time (row group g = rows 16g .. 16g+15, rows
 * past M stored as zeros); tile (g, c) covers the K-tile c of group g and
 * starts at byte g * 16 * R + c * 18432 (Q4_0) or c * 17664 (KSB), R the
 * canonical row bytes; the last tile of a row holds the remaining blocks.
 * For lane l = 4 gg + t (gg = 0..7, t = 0..3), "word t" of a block is its
 * code bytes qs[4t .. 4t+3].
 *   Q4_0 tile of nb blocks (nb even), unit u = blocks 2u, 2u+1:
 *     at 512 u + 16 l: word t of block 2u of rows gg and gg+8, then of block
 *       2u+1 of rows gg and gg+8 (4 bytes each);
 *     at 256 nb + 64 u + 4 r: the FP16 scales of blocks 2u and 2u+1, row r.
 *   KSB tile of ns super-blocks, unit u = sub-blocks j = 4 (u % 2) + h
 *   (h = 0..3) of super-block u / 2:
 *     at 1024 u + 32 l + 8 h: word t of sub-block j of rows gg and gg+8;
 *     at 2048 ns + 64 u + 4 r + h: the INT8 sub-scale q_j of row r;
 *     at 2176 ns + 32 (u / 2) + 2 r: the FP16 super-scale S of row r.
 * gq_tiled_bytes: bytes of the tiled storage of an M x K matrix; 0 unless K
 * is a multiple of 64 (Q4_0) or 256 (KSB).
 * gq_repack_*: canonical rows W (M x K, as for gq_gemv_*) -> tiled storage
 * `out` of gq_tiled_bytes(...) bytes; both 16-byte aligned, not overlapping.
 * Asynchronous on `stream`; bad shapes give GQ_ERR_SHAPE. */
GQ_API size_t gq_tiled_bytes(int fmt, int64_t M, int64_t K);
GQ_API gq_status gq_repack_q4_0(const void* W, int64_t M, int64_t K, void* out, void* stream);
GQ_API gq_status gq_repack_ksb(const void* W, int64_t M, int64_t K, void* out, void* stream);

/* Batch-1 GEMV on tiled storage, y[m] = sum_k W_hat[m][k] * x[k] (the same
 * product as gq_gemv_* with B = 1, computed from the tiled bytes): Q4_0
 * chapter 4.3 and the K-quants post's step 5 for the decoded weights, the
 * TurboQuant W4A8 post, section 2.3, for the memory-bound decode step.
 *   T: gq_tiled_bytes(fmt, M, K) bytes from gq_repack_* (16-byte aligned).
 *   K: a multiple of 64 (Q4_0) or 256 (KSB), at most 16384 (GQ_ERR_SHAPE).
 *   x: K fp16 values (x_dtype must be GQ_F16, GQ_ERR_DTYPE otherwise).
 *   y: M values of y_dtype (GQ_F16, GQ_BF16 or GQ_F32).
 * Arithmetic: each 4-bit code enters the tensor core exactly (as an fp16
 * subnormal c * 2^-24), the -8 offset enters as -8 * (block sum of x), and
 * the fp32 MMA accumulation, the fp32 block sums of x and the fp32 sum over
 * blocks round; the result is rounded once to y_dtype.  Non-finite
 * activations give non-finite outputs.
 * flags: 0 or GQ_GEMV_PDL (with PDL the kernel also stages its first tiles in
 * tensor memory while the preceding kernel runs).  dev_status: optional,
 * receives GQ_DEV_TIMEOUT if a pipeline wait ever gives up. */
GQ_API gq_status gq_gemv_q4_0_tiled(const void* T, int64_t M, int64_t K, const void* x,
                                    int x_dtype, void* y, int y_dtype, unsigned flags,
                                    int* dev_status, void* stream);
GQ_API gq_status gq_gemv_ksb_tiled(const void* T, int64_t M, int64_t K, const void* x, int x_dtype,
                                   void* y, int y_dtype, unsigned flags, int* dev_status,
                                   void* stream);

/* Grouped tiled GEMV (no counterpart on the pages: the GGUF GEMV of the format
 * pages applied to many tiled matrices that share one activation vector, e.g.
 * every projection of a decoder layer or of a whole model in one call).
 * y_i = W_i x for each descriptor, each output as gq_gemv_*_tiled computes it
 * (the same fp32 additions in the same order, so bit for bit the same).
 *   mats:  count host descriptors {W, M, y} (read during the call only); W is
 *          the TILED storage of an M x K matrix (gq_repack_*), y: [M] of
 *          y_dtype; both 16-byte aligned.  M == 0 entries are skipped (W and
 *          y may then be NULL).
 *   K, x, x_dtype, y_dtype, flags, dev_status: as for gq_gemv_*_tiled, shared
 *          by all matrices (B = 1, fp16 x).
 * Validation covers every descriptor before anything is launched; more than
 * 256 matrices are processed in several launches in stream order. */
GQ_API gq_status gq_gemv_q4_0_tiled_grouped(const gq_gemv_desc* mats, int count, int64_t K,
                                            const void* x, int x_dtype, int y_dtype,
                                            unsigned flags, int* dev_status, void* stream);
GQ_API gq_status gq_gemv_ksb_tiled_grouped(const gq_gemv_desc* mats, int count, int64_t K,
                                           const void* x, int x_dtype, int y_dtype,
                                           unsigned flags, int* dev_status, void* stream);

/* Allocation-free variant (no counterpart on the pages): the batch-1 integer
 * tensor-core path of gq_gemv_q4_0 (fp16 x, B = 1) with its scratch -- the
 * per-CTA counts and partial sums, 33 KB -- in a static device array of the
 * library instead of a caller workspace.  For callers that cannot give the
 * library device memory.  The counts are cleared with an asynchronous memset
 * on `stream` before each launch; the library allocates nothing.
 *   Arguments as for gq_gemv_q4_0 with x_dtype = GQ_F16, B = 1 and no
 *   workspace.  K must be a multiple of 256 and at most 14336
 *   (GQ_ERR_SHAPE otherwise); a launch wider than the scratch covers (more
 *   than 256 CTAs, which needs a GPU of more than 256 SMs) gives
 *   GQ_ERR_WORKSPACE.
 *   The scratch is one per device: calls that may overlap (other streams,
 *   other host threads) race on it and must be serialised by the caller.
 *   The first call in a CUDA context looks the scratch up with
 *   cudaGetSymbolAddress; make it before capturing work into a graph.  A
 *   context created later (e.g. after cudaDeviceReset) is looked up anew. */
GQ_API gq_status gq_gemv_q4_0_noalloc(const void* W, int64_t M, int64_t K, const void* x,
                                      void* y, int y_dtype, unsigned flags, int* dev_status,
                                      void* stream);

/* Self-test of the bounded waits (no counterpart on the pages): runs the
 * Q4_0 GEMV (fp16 x and y, batch 1) on the given buffers with a producer that
 * never fills its first pipeline stage and a ~1 ms wait budget.  The consumer
 * waits run out; the kernel ORs GQ_DEV_TIMEOUT into *dev_status (required),
 * lets the copies it did issue land and exits; y is unspecified.  Nothing
 * faults, traps or hangs, and the context stays usable.  Arguments as for
 * gq_gemv_q4_0. */
GQ_API gq_status gq_selftest_gemv_timeout(const void* W, int64_t M, int64_t K, const void* x,
                                          void* y, int* dev_status, void* stream);

/* Calibration (no counterpart on the pages): reads `bytes` bytes at p once
 * with 16-byte streaming loads and XORs every little-endian 32-bit word of
 * them into *sink (device memory; the caller zeroes it first, the fold is
 * applied with atomics).  One launch of this is the practical ceiling for a
 * kernel that reads that many bytes once, launch and drain included: the
 * reference the GEMV's streamed-weight rate is compared with beside the
 * long-copy peak.
 *   p: device pointer, 16-byte aligned (GQ_ERR_ALIGNMENT); bytes % 16 == 0
 *   (GQ_ERR_SHAPE); sink: 4-byte aligned device word.  bytes == 0 launches
 *   nothing.  Asynchronous on `stream`. */
GQ_API gq_status gq_stream_read(const void* p, size_t bytes, uint32_t* sink, void* stream);

/* Dequantize-fused batched product for batches that make a dense
 * contraction: Y = W_hat * X^T on the tcgen05 tensor cores (the matrix
 * multiply that consumes decoded blocks, Q4_0 chapter 4.3).
 *   W: M x K packed as for gq_gemv_*.  K % 32 == 0 (Q4_0) / K % 256 == 0 (KSB).
 *   X: [B][K] bfloat16 (x_dtype must be GQ_BF16), row-major, 16-byte aligned.
 *   Y: [B][M] of y_dtype (GQ_F32, GQ_F16 or GQ_BF16), row-major.
 *   B: 1..256 (0 launches nothing).
 * Batches of 1..16 run on the warp-MMA product of gq_gemv_* (each code
 * decoded once for all columns, two n8 MMA tiles; the workspace is checked
 * but not used): below about 16 columns a tcgen05 MMA would spend its fixed
 * cost mostly on empty columns.  Larger batches run on the tcgen05 kernel:
 * Arithmetic: each decoded weight (at most 14 significant bits) is split
 * exactly into two bfloat16 parts, both multiplied by X on the tensor core
 * into one fp32 accumulator, so every product is exact and only the fp32
 * accumulation rounds.  (The warp-MMA path multiplies the exact code - 8 in
 * bfloat16 and applies the FP16 scale in fp32: also exact products.)
 * Work split: the 128-row tiles x 64-wide k-steps are divided evenly over
 * the SMs (stream-K); a tile shared by two or three SMs is combined through
 * fp32 partial sums, in a fixed order, so results do not depend on
 * scheduling.
 * workspace / ws_bytes: caller-owned device scratch of at least
 * gq_gemm_workspace_bytes(...) bytes (GQ_ERR_WORKSPACE otherwise),
 * 256-byte aligned, all zero before its first use; a successful call leaves
 * it ready for the next call of the same or a smaller shape; after a call
 * that fails or reports GQ_DEV_TIMEOUT, zero it again.  Calls that may run
 * at the same time need separate workspaces.
 * dev_status: optional, receives GQ_DEV_TIMEOUT if a pipeline wait gives up. */
GQ_API size_t gq_gemm_workspace_bytes(int fmt, int64_t M, int64_t K, int64_t B);
GQ_API gq_status gq_gemm_q4_0(const void* W, int64_t M, int64_t K,
                              const void* X, int x_dtype, int64_t B,
                              void* Y, int y_dtype, void* workspace, size_t ws_bytes,
                              int* dev_status, void* stream);
GQ_API gq_status gq_gemm_ksb(const void* W, int64_t M, int64_t K,
                             const void* X, int x_dtype, int64_t B,
                             void* Y, int y_dtype, void* workspace, size_t ws_bytes,
                             int* dev_status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* GQ_H */
