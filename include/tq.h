/*
 * tq.h -- C ABI of libtq: ternary weight-only grouped linear layer on B200.
 *
 * The operations follow two pages:
 *   "precisit/pack-unpack-run" (codec.py description and payload-rate
 *   paragraph): per group of G input columns, a scale equal to the mean of
 *   |w| kept as binary16, trits by rounding w / scale half to even, base-3
 *   digits five to a byte, every group starting on a byte boundary with its
 *   unused digit slots holding the zero trit, byte values 243..255 invalid,
 *   a zero scale decoding to an all-zero group, and decoding to bf16.
 *   tiny-llm "Week 2 Day 3: Quantize the Model" ("Mathematical Formulation",
 *   "Computation Flow"): C = A B^T with B reconstructed per group and the
 *   products accumulated in float.
 *
 * Layout (all row-major, all buffers contiguous, no padding between rows):
 *   W, W_out  bf16   [N][K]                      weights, nn.Linear "out x in"
 *   codes     uint8  [N][K/G][B],  B = ceil(G/5) one byte-aligned run per group
 *   scales    fp16   [N][K/G]                    one binary16 scale per group
 *   X         bf16   [M][K]                      activations
 *   Y         fp32 or bf16 [M][N]                Y = X . What^T
 * Byte encoding: weight j of a group (0 <= j < G) is digit (j mod 5) of byte
 * floor(j/5); digit d = t + 1 for trit t in {-1, 0, +1}; byte = sum_i d_i 3^i,
 * the first weight being the least significant digit.  Positions j >= G in
 * the last byte hold the padding digit 1 (the zero trit).
 * Decoded weight: What = +0 if t == 0 or the scale is +0, else
 * t * RNE_bf16(scale).  A group with an invalid byte, a padding digit other
 * than 1, or a scale that is NaN, Inf or has its sign bit set, decodes to
 * bf16 NaN, so every output that touches it is NaN.
 *
 * Calling convention: every pointer except the sizes is a DEVICE pointer
 * owned by the caller; the library never allocates or frees device memory
 * and never synchronizes.  Work is enqueued on `stream` (NULL = legacy
 * default stream).  A call returns TQ_OK once its kernels are enqueued; a
 * synchronous error code means nothing was launched.  Data errors found by
 * the kernels are OR-ed into *d_err (a device word the caller zeroes; may be
 * NULL) using the TQ_DERR_* bits.  No exceptions cross this boundary and
 * there is no CPU fallback.  Calls are thread-safe.  One device per process:
 * the kernels' shared-memory size attributes are raised once per process, on
 * the device current at the first call that needs them, so launches on a
 * second device of the same process may fail with TQ_ERR_CUDA.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *tq_stream_t;

typedef enum {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1, /* null pointer, bad shape, G out of range, K % G != 0, overlap */
    TQ_ERR_ALIGNMENT = 2,   /* a pointer misses the alignment stated for it */
    TQ_ERR_UNSUPPORTED = 3, /* valid arguments this build cannot run (e.g. no sm_100 device) */
    TQ_ERR_CUDA = 4         /* a CUDA launch or attribute call failed */
} tq_status;

typedef enum { TQ_OUT_F32 = 0, TQ_OUT_BF16 = 1 } tq_out_dtype;

/* Asynchronous data-error bits written to *d_err. */
#define TQ_DERR_BYTE     1u  /* a code byte >= 243 (decode, matmul)               */
#define TQ_DERR_PADDING  2u  /* a padding digit other than 1 (decode, matmul)     */
#define TQ_DERR_WEIGHT   4u  /* a NaN or Inf weight (quantize): group stored as 0 */
#define TQ_DERR_SCALE    8u  /* a stored scale NaN, Inf or negative (decode, mm)  */
#define TQ_DERR_OVERFLOW 16u /* a group mean that overflows binary16 (quantize)   */
#define TQ_DERR_TIMEOUT  32u /* a bounded pipeline wait gave up (matmul)          */

/* Largest supported group size. */
#define TQ_MAX_G 4096

/* Bytes of the codes buffer: N * (K/G) * ceil(G/5).  0 for invalid shapes. */
TQ_API size_t tq_codes_bytes(int64_t N, int64_t K, int G);
/* Bytes of the scales buffer: N * (K/G) * 2.  0 for invalid shapes. */
TQ_API size_t tq_scales_bytes(int64_t N, int64_t K, int G);
/* Bytes of device scratch tq_gemv / tq_gemm need for these shapes.  Every
 * kernel of this build keeps its partial sums on chip (registers, shared
 * memory, distributed shared memory of a cluster, tensor memory), so this is
 * 0 for every shape and the workspace arguments below are accepted but not
 * read; callers that pass a buffer of this size stay correct if a later
 * build needs one. */
TQ_API size_t tq_workspace_bytes(int64_t M, int64_t N, int64_t K, int G);

/*
 * Quantize and pack ("precisit/pack-unpack-run", codec.py: per-group mean
 * |w| scale in fp16, round-half-even trits, base-3 packing).
 * W_bf16: [N][K] bf16, 16-byte aligned.  codes: tq_codes_bytes() bytes.
 * scales_f16: [N][K/G] binary16, 2-byte aligned.
 * Scale = RNE_binary16(exact mean of |w| over the group); trit =
 * clamp(round_half_even(w / scale), -1, 1), all zero when the scale is +0.
 * A group with a NaN/Inf weight or a mean >= 65520 is stored as a zero group
 * and flagged (TQ_DERR_WEIGHT / TQ_DERR_OVERFLOW).
 * Errors: TQ_ERR_INVALID_ARG for N < 0, K < 0, G < 1, G > TQ_MAX_G, K % G,
 * null pointers with nonzero sizes, or codes/scales overlapping W;
 * TQ_ERR_ALIGNMENT; TQ_ERR_CUDA.
 */
TQ_API tq_status tq_quantize_pack(const void *W_bf16, int64_t N, int64_t K, int G, uint8_t *codes,
                           void *scales_f16, uint32_t *d_err, tq_stream_t stream);

/*
 * Decode to bf16 ("precisit/pack-unpack-run", codec.py: decoding; bytes
 * 243..255 invalid; weights restored as bf16).
 * codes/scales as produced by tq_quantize_pack; W_bf16_out: [N][K] bf16,
 * 16-byte aligned.  Rejected groups are written as bf16 NaN and flagged
 * (TQ_DERR_BYTE, TQ_DERR_PADDING, TQ_DERR_SCALE).
 */
TQ_API tq_status tq_unpack_bf16(const uint8_t *codes, const void *scales_f16, int64_t N, int64_t K,
                         int G, void *W_bf16_out, uint32_t *d_err, tq_stream_t stream);

/*
 * Fused unpack-and-scale matmul for decode (tiny-llm "Week 2 Day 3",
 * "Computation Flow"; the scale is applied once per group as in its "SIMD
 * Matvec" stage): Y[m][n] = sum_g RNE_bf16(s[n][g]) * sum_{j in g} t[n][j] X[m][j],
 * accumulated in fp32, written as fp32 or RNE bf16.  Any M >= 1: CUDA-core
 * kernels up to 4 tokens, and up to 8 where the tensor path does not take
 * the shape (weights decoded on chip ahead of the activations when a
 * matrix's rows fit; otherwise lookup tables: one streaming launch per token
 * for 1 token, and for 2..4 tokens on matrices of at least 48 M weights,
 * with G in {64, 128} and K a multiple of 512 up to 4096), tensor-core
 * small-M kernels up to 64 tokens (K % 64 == 0, G % 64 == 0), a row kernel
 * beyond and for the shapes those do not cover.  X: [M][K] bf16, 16-byte aligned; Y: [M][N]
 * (fp32: 4-byte aligned, bf16: 2-byte aligned), must not overlap the inputs.
 * K == 0 is allowed: every output is an empty sum and Y is set to +0.
 * workspace: at least tq_workspace_bytes(M, N, K, G) bytes of device scratch
 * (NULL allowed when that is 0), 256-byte aligned.
 * Ordering: the kernels are launched as programmatic dependents of the work
 * before them on `stream`.  X is read only after that work has completed;
 * codes and scales (the weights) may be read while it is still finishing, so
 * they must not be written by the kernel launched immediately before this
 * call on the same stream (write them earlier, or on another stream and
 * join with an event).  The one exception is this library's own
 * tq_quantize_pack / tq2_quantize_pack: they never release their dependents
 * early and make their stores visible device-wide before their blocks exit,
 * so a matmul may directly follow them on the same buffers and stream.
 */
TQ_API tq_status tq_gemv(const void *X_bf16, int64_t M, const uint8_t *codes, const void *scales_f16,
                  int64_t N, int64_t K, int G, void *Y, tq_out_dtype y_dtype, void *workspace,
                  size_t ws_bytes, uint32_t *d_err, tq_stream_t stream);

/*
 * Fused unpack-and-scale matmul for prefill: same result definition as
 * tq_gemv, computed on the tensor cores (tcgen05, fp32 accumulators in
 * tensor memory) from bf16 weights decoded on chip: What = t * RNE_bf16(s).
 * Same arguments, alignment and ordering rules as tq_gemv (with M <= 64
 * the small-M kernels are launched as programmatic dependents too).
 */
TQ_API tq_status tq_gemm(const void *X_bf16, int64_t M, const uint8_t *codes, const void *scales_f16,
                  int64_t N, int64_t K, int G, void *Y, tq_out_dtype y_dtype, void *workspace,
                  size_t ws_bytes, uint32_t *d_err, tq_stream_t stream);

/*
 * The 2-bit ternary format ("Autoregressive Language Model on the 6502
 * Processor", summary: BitNet ternary weights packed four per byte).  Same
 * groups, binary16 scales and trits as the base-3 codec; code c = t + 1 in
 * two bits, weight j of a group in bits 2 (j % 4) of its byte j / 4, each
 * group ceil(G/4) bytes, padding codes 1, code 3 invalid (TQ_DERR_BYTE; a
 * padding code other than 1 or 3 sets TQ_DERR_PADDING).  Buffers:
 * codes [N][K/G][ceil(G/4)] (4-byte aligned), scales as for base-3.
 */
/* Bytes of the 2-bit codes buffer: N * (K/G) * ceil(G/4).  0 for invalid shapes. */
TQ_API size_t tq2_codes_bytes(int64_t N, int64_t K, int G);
/* Quantize and pack into the 2-bit format; arguments, errors and error bits as
 * tq_quantize_pack, plus TQ_ERR_ALIGNMENT for codes not 4-byte aligned. */
TQ_API tq_status tq2_quantize_pack(const void *W_bf16, int64_t N, int64_t K, int G, uint8_t *codes,
                            void *scales_f16, uint32_t *d_err, tq_stream_t stream);
/* Decode the 2-bit format to bf16; as tq_unpack_bf16 (rejected groups NaN). */
TQ_API tq_status tq2_unpack_bf16(const uint8_t *codes, const void *scales_f16, int64_t N, int64_t K,
                          int G, void *W_bf16_out, uint32_t *d_err, tq_stream_t stream);
/* Fused unpack-and-scale matmul on the 2-bit format for decode; result
 * definition, arguments, alignment and ordering rule as tq_gemv (X is read
 * after the preceding work has completed; codes and scales may be read
 * before, so the kernel launched immediately before on the same stream must
 * not write them).  1 token on matrices of at least 24 M weights (8 M at
 * K >= 2048), and 2..4 tokens from 48 M weights, with G in {64, 128}, K a
 * multiple of 512 up to 4096 and 8-byte-aligned codes, take the streaming
 * lookup-table kernel, one launch per token; 1..4 tokens (1..8 at G < 64)
 * with K % 512 == 0, G % 16 == 0, 4-byte-aligned codes and rows that fit
 * in shared memory the pre-decode kernel (weights decoded before the
 * activations are awaited); 3..64 tokens with K % 64 == 0
 * and G % 64 == 0 the tensor-core small-M kernels (2-bit codes decoded on
 * chip); otherwise the CUDA-core kernel, eight tokens per launch, which
 * covers G in {16, 32, 64, 128, 256} and K <= 49152; other shapes return
 * TQ_ERR_UNSUPPORTED. */
TQ_API tq_status tq2_gemv(const void *X_bf16, int64_t M, const uint8_t *codes, const void *scales_f16,
                   int64_t N, int64_t K, int G, void *Y, tq_out_dtype y_dtype, void *workspace,
                   size_t ws_bytes, uint32_t *d_err, tq_stream_t stream);
/* Fused unpack-and-scale matmul on the 2-bit format for prefill, on the
 * tensor cores (tcgen05, fp32 accumulators in tensor memory), What decoded on
 * chip from the 2-bit codes: the result definition, arguments and ordering
 * rule of tq_gemm.  Needs K % 64 == 0 and G % 64 == 0 (a 64-column stage is
 * 16 whole code bytes of one group), else TQ_ERR_UNSUPPORTED. */
TQ_API tq_status tq2_gemm(const void *X_bf16, int64_t M, const uint8_t *codes, const void *scales_f16,
                   int64_t N, int64_t K, int G, void *Y, tq_out_dtype y_dtype, void *workspace,
                   size_t ws_bytes, uint32_t *d_err, tq_stream_t stream);

/*
 * The W4A16 affine format (tiny-llm "Week 2 Day 3: Quantize the Model",
 * "Group-Wise Affine Quantization", "Reconstruct a Stored Group", "Packed
 * Storage Layout"), a second weight format next to the ternary codes:
 * unsigned 4-bit codes q, eight per 32-bit word, code j of a row in bits
 * 4 (j mod 8) .. 4 (j mod 8) + 3 of word j / 8 (first code in the low nibble);
 * per group of G columns (G a multiple of 8) a signed bf16 scale s and a
 * bf16 bias b; the weight is w = q * s + b.  Buffers: codes uint32 [N][K/8]
 * (4-byte aligned; 16-byte aligned for the fast kernel), scales and biases
 * bf16 [N][K/G] (2-byte aligned), X bf16 [M][K] (16-byte aligned), Y as for
 * tq_gemv.  There are no invalid codes and no data-error bits.
 */
/* Bytes of the W4 codes buffer: N * (K/8) * 4.  0 for invalid shapes or G % 8 != 0. */
TQ_API size_t tq_w4_codes_bytes(int64_t N, int64_t K, int G);
/* Decode matmul on the W4 format, CUDA cores, any M >= 1 (eight tokens per
 * launch): Y[m][n] = sum_g (s[n][g] * sum_{j in g} q[n][j] X[m][j] + b[n][g] *
 * sum_{j in g} X[m][j]) with fp32 accumulation ("Stage 2: SIMD Matvec" factors
 * the bias out of the group's dot product), written as fp32 or RNE bf16.
 * Ordering rule as tq_gemv.  G in {64, 128}, K a multiple of 256 up to
 * 2048, 8-byte-aligned codes and scales and biases aligned to 4 bytes
 * (G = 128) or 8 (G = 64) take the streaming lookup-table kernel (one
 * 256-column slice of tables per CTA, the slices of a row over a
 * thread-block cluster), one launch per token, for one token from 12 Mi
 * weights (6 Mi at K >= 2048) and for 2..4 tokens from 12 Mi weights at
 * K <= 512 or from 96 Mi weights at any K; 5..64 tokens with G % 64 == 0
 * and K % 64 == 0 the small-M tensor-core kernels (each weight as two bf16
 * terms, as tq_w4_gemm; above about 9,500 rows only with 16-byte-aligned
 * codes); other
 * shapes with G % 32 == 0, K % 32 == 0 and K <= 4096 the CUDA-core streaming
 * kernel, eight tokens per launch, and the rest a plain one-warp-per-row
 * kernel.
 * Errors: TQ_ERR_INVALID_ARG (shapes, G % 8, nulls, Y overlapping an input),
 * TQ_ERR_ALIGNMENT, TQ_ERR_CUDA. */
TQ_API tq_status tq_w4_gemv(const void *X_bf16, int64_t M, const uint32_t *codes, const void *scales_bf16,
                     const void *biases_bf16, int64_t N, int64_t K, int G, void *Y, tq_out_dtype y_dtype,
                     tq_stream_t stream);

/* Fused matmul on the W4 format for prefill, on the tensor cores (tcgen05,
 * fp32 accumulators in tensor memory): the same result definition as
 * tq_w4_gemv.  Each weight w = q * s + b is formed with one fp32 FMA and fed
 * to the MMA as two bf16 terms, RNE_bf16(w) and RNE_bf16 of the remainder,
 * so the products keep w to about 2^-17 relative.  Up to 64 tokens the
 * small-M kernels (the two terms stored in tensor memory as the MMA's A
 * operand; above about 9,500 rows only with 16-byte-aligned codes),
 * otherwise the prefill kernel.  Needs K % 64 == 0 and G % 64 == 0, else
 * TQ_ERR_UNSUPPORTED; other arguments as tq_w4_gemv. */
TQ_API tq_status tq_w4_gemm(const void *X_bf16, int64_t M, const uint32_t *codes, const void *scales_bf16,
                     const void *biases_bf16, int64_t N, int64_t K, int G, void *Y, tq_out_dtype y_dtype,
                     tq_stream_t stream);

/* Human-readable name of a status code (static string). */
TQ_API const char *tq_status_string(tq_status s);
/* Library version and build flags (static string). */
TQ_API const char *tq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
