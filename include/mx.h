/*
 * mx.h -- C ABI of libmx: the MX (microscaling) cast and the block-scaled
 * GEMM on NVIDIA B200 (sm_100a).
 *
 * The operations follow the pages:
 *  - "Microscaling Data Formats for Deep Learning" (summary page), section 2
 *    "Microscaling": an MX block holds k = 32 values as one shared E8M0 scale X
 *    and 32 narrow elements P_i, v_i = X * P_i; a NaN scale (code 0xFF) makes
 *    the whole block NaN; the storage layout is left to the implementation.
 *  - same page, section 3 "Scalar Float to MX Format Conversion" (Algorithm 1):
 *    X = 2^(floor(log2 amax) - emax_elem), P_i = quantize(V_i / X) with
 *    overflow clamped to the element format's largest normal, and FP32
 *    subnormal inputs set to zero; the block axis is a parameter because the
 *    cast does not commute with a transpose.
 *  - same page, section 4, compute flow: dot products consume MX operands and
 *    return scalar floats (here fp32 accumulation, fp32 or bf16 output).
 *  - "Format-Aware Fusion for Fast FP4 Pretraining" (abstract): stochastic
 *    rounding and a fixed-sign 32-point Hadamard before the FP4 cast of the
 *    weight-gradient operands.
 *
 * Conventions shared by every entry point
 *  - Pointers named x, codes, scales, y, c, a_*, b_* are DEVICE pointers
 *    (cudaMalloc'd or torch-allocated on the current device) unless the name
 *    says otherwise.  The caller owns all of them; the library never frees,
 *    retains or allocates device buffers (it keeps one status word per device
 *    in a static __device__ variable).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Every call only enqueues work on it and returns; nothing
 *    synchronises unless stated.
 *  - Return value: MX_OK (0) or a negative mx_status.  Argument errors are
 *    detected on the host before anything is launched; the output buffers are
 *    then untouched.  An empty tensor (a zero size) is a no-op returning MX_OK,
 *    and its pointers may then be NULL.
 *  - All 2-D tensors are row-major with an explicit leading dimension
 *    (elements between consecutive rows).
 *
 * Storage layout (section 2 leaves it to the implementation)
 *  - Element codes are stored "block-axis-major": one row per line along the
 *    block axis ("outer" rows of "inner" elements, inner % 32 == 0).  Quantizing
 *    an R x C tensor along C gives R rows of C codes; along R it gives C rows of
 *    R codes (transposed on the way out).  Rows are packed with no padding:
 *    8-bit formats one code per byte; FP6 four codes per 3 bytes (code j of a
 *    group in bits 6j..6j+5 of a little-endian 24-bit word); FP4 two codes per
 *    byte, the even element in the low nibble.
 *  - Element encodings: E4M3 (bias 7, NaN S.1111.111, no Inf), E5M2 (bias 15,
 *    IEEE Inf/NaN), E2M3 (bias 1), E3M2 (bias 3), E2M1 (bias 1), INT8 (two's
 *    complement, value = code * 2^-6).  Scale codes are E8M0: 2^(s-127), 0xFF
 *    is NaN.
 *  - Scales, MX_SCALES_PLAIN: outer x (inner/32) bytes, row-major.
 *    MX_SCALES_MMA: the layout the tensor cores read.  Rows are padded to a
 *    multiple of 128 and k-blocks to a multiple of 4; the buffer is a sequence
 *    of 512-byte atoms, one per (128-row block, 4-k-block group), k-groups
 *    fastest; inside an atom the byte for row r, k-block kb is at
 *    (r % 32) * 16 + ((r / 32) % 4) * 4 + (kb % 4).  Padding bytes are never
 *    written by mx_quantize.
 *    MX_SCALES_MMA_X4: the MMA layout with every atom stored four times in a
 *    row, 2048 bytes per atom (the byte above at atom * 2048 + j * 512 + its
 *    offset in the atom, j = 0..3; four times the MMA bytes).  The tensor
 *    cores read each atom into all four 32-lane quarters of tensor memory;
 *    with the copies already in memory the GEMM moves them with plain
 *    128-lane copies instead of the replicating copy (mx_gemm_x4).
 */
#ifndef MX_H
#define MX_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__) || defined(__clang__)
#define MX_API __attribute__((visibility("default")))
#else
#define MX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MX_E4M3 = 0,  /* MXFP8, 4-bit exponent, 3-bit mantissa, emax 8,  max 448   */
    MX_E5M2 = 1,  /* MXFP8, 5-bit exponent, 2-bit mantissa, emax 15, max 57344 */
    MX_E2M3 = 2,  /* MXFP6, emax 2, max 7.5 */
    MX_E3M2 = 3,  /* MXFP6, emax 4, max 28  */
    MX_E2M1 = 4,  /* MXFP4, emax 2, max 6   */
    MX_INT8 = 5   /* MXINT8, emax 0, max 127/64 (symmetric; -128 is never produced) */
} mx_fmt;

typedef enum { MX_F32 = 0, MX_BF16 = 1 } mx_dtype;

typedef enum {
    MX_RNE = 0,   /* round to nearest, ties to even mantissa (even integer for INT8) */
    MX_SR = 1     /* stochastic rounding, see mx_quantize */
} mx_round;

typedef enum { MX_SCALES_PLAIN = 0, MX_SCALES_MMA = 1, MX_SCALES_MMA_X4 = 2 } mx_scale_layout;

/* Optional preconditioning of each 32-block before the cast.
 * hadamard != 0: x_j <- s_j * x_j with s_j = +1 where bit j of sign_mask is
 * set and -1 elsewhere (j = position inside the block along the block axis),
 * then the unnormalised 32-point Sylvester Hadamard transform as five fp32
 * butterfly stages (h = 1, 2, 4, 8, 16; (a, b) -> (a + b, a - b)).  The
 * transform is orthogonal up to a factor 32, so a GEMM of two operands
 * preconditioned with the same mask along the reduction axis recovers the
 * plain product with alpha = 1/32. */
typedef struct {
    int32_t hadamard;
    uint32_t sign_mask;
} mx_precond;

#define MX_DEFAULT_SIGN_MASK 0x6A09E667u

typedef enum {
    MX_OK = 0,
    MX_ERR_ARG = -1,          /* null pointer, bad enum, negative size, ld too small   */
    MX_ERR_ALIGN = -2,        /* pointer or leading dimension breaks the 16-byte rules  */
    MX_ERR_SHAPE = -3,        /* block-axis length not a multiple of 32                 */
    MX_ERR_UNSUPPORTED = -4,  /* valid request that this build does not implement       */
    MX_ERR_SR_RANGE = -5,     /* stochastic rounding index space exceeds 2^34 elements  */
    MX_ERR_CUDA = -6,         /* a CUDA runtime/driver call or launch failed            */
    MX_ERR_TIMEOUT = -7,      /* a bounded device-side wait expired (see below)         */
    MX_ERR_BOUNDS = -8        /* debug build only: a device store or load fell outside
                                 its buffer and was skipped (see mx_last_device_status) */
} mx_status;

/*
 * mx_quantize -- Algorithm 1 of section 3 on every 32-block along block_axis.
 *
 *  x          device, rows x cols, leading dimension ldx (elements), dtype xdt.
 *             16-byte aligned; ldx * sizeof(elem) must be a multiple of 16.
 *  block_axis 1: blocks run along a row (contiguous).  codes: rows x cols.
 *             0: blocks run down a column (strided).   codes: cols x rows.
 *  fmt        element format.
 *  rnd        MX_RNE, or MX_SR: with lo <= |u| < hi the neighbouring grid
 *             points of u = V/X, F = floor(256 (|u| - lo) / (hi - lo)), and the
 *             magnitude rounds up iff F + r >= 256, where r is byte (i mod 4)
 *             of fmix32(floor(i / 4) xor (fmix32(seed_lo32) xor seed_hi32)),
 *             i the element's linear index in the output (outer * inner +
 *             position along the block axis) and fmix32 the MurmurHash3
 *             32-bit finaliser.  Results therefore do not depend on tiling.
 *  seed       only read for MX_SR.
 *  pre        NULL, or preconditioning (see mx_precond).  Non-NULL with
 *             hadamard != 0 is supported for block_axis 0 only.  Scale
 *             buffers of 4 GiB or more are not supported (MX_ERR_UNSUPPORTED).
 *  codes      device, mx_codes_bytes(fmt, outer, inner) bytes, 16-byte aligned.
 *  scales     device, mx_scales_bytes(sl, outer, inner) bytes.
 *  sl         scale layout to write.
 *
 * Per block: FP32 subnormals (after preconditioning, and bf16 subnormals,
 * which widen to FP32 subnormals) become signed zeros; a NaN or Inf anywhere
 * gives scale 0xFF and all-zero codes; amax == 0 gives scale code 0; else
 * e = clamp(floor(log2 amax) - emax, -127, 127) and the scale code is e + 127.
 * Elements are rounded to the grid with overflow clamped to +-max; FP formats
 * keep the sign of zero.
 * Errors: MX_ERR_ARG, MX_ERR_ALIGN, MX_ERR_SHAPE (inner % 32 != 0),
 * MX_ERR_UNSUPPORTED, MX_ERR_SR_RANGE, MX_ERR_CUDA; MX_ERR_TIMEOUT later through
 * mx_last_device_status if a column cast (block_axis 0) gave up its bounded
 * wait for a tile's copy into shared memory (its outputs are then incomplete).
 */
MX_API int mx_quantize(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                int block_axis, mx_fmt fmt, mx_round rnd, uint64_t seed,
                const mx_precond *pre, void *codes, void *scales, mx_scale_layout sl,
                void *stream);

/*
 * mx_quantize_dual -- both quantizations of one rows x cols tensor from a
 * single read of it: the codes and scales of mx_quantize along rows
 * (block_axis 1, for a GEMM contracting over cols) and of mx_quantize along
 * columns (block_axis 0, transposed output, for a GEMM contracting over rows).
 * The MX summary page's section 3 observes that these two quantizations of a
 * tensor differ, and a training step needs both (forward and weight
 * gradient); the FP4-pretraining abstract's fused producers motivate reading
 * the tensor once.
 *
 *  x, xdt, rows, cols, ldx, fmt, sl   as for mx_quantize; rows and cols must
 *           both be multiples of 32 (MX_ERR_SHAPE otherwise).
 *  rnd_rows, seed_rows   rounding of the along-rows output.
 *  rnd_cols, seed_cols, pre_cols   rounding and the optional fixed-sign
 *           Hadamard of the along-columns output (pre_cols may be NULL).
 *  codes_rows  device, rows x (cols * bits / 8) bytes, 16-byte aligned.
 *  scales_rows device, mx_scales_bytes(sl, rows, cols) bytes.
 *  codes_cols  device, cols x (rows * bits / 8) bytes, 16-byte aligned.
 *  scales_cols device, mx_scales_bytes(sl, cols, rows) bytes.
 * Each output is bit-identical to the corresponding mx_quantize call with the
 * same arguments.  All four buffers are owned by the caller and must not
 * overlap x or each other.  Errors as for mx_quantize.
 */
MX_API int mx_quantize_dual(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx, mx_fmt fmt,
                            mx_round rnd_rows, uint64_t seed_rows, mx_round rnd_cols, uint64_t seed_cols,
                            const mx_precond *pre_cols, void *codes_rows, void *scales_rows,
                            void *codes_cols, void *scales_cols, mx_scale_layout sl, void *stream);

/*
 * Placement of a tensor inside a larger one, for casts of shards.  The tensor
 * passed to mx_quantize_shard / mx_quantize_dual_shard is the piece whose
 * element (0, 0) is element (row0, col0) of a total_rows x total_cols tensor.
 */
typedef struct {
    int64_t row0, col0;               /* offset of the piece in the whole tensor  */
    int64_t total_rows, total_cols;   /* shape of the whole tensor                */
} mx_shard;

/*
 * mx_quantize_shard -- mx_quantize of one piece of a larger tensor, giving
 * exactly the bytes of the matching slice of the whole tensor's cast.  Only
 * stochastic rounding depends on the placement: its index i is the element's
 * position in the block-axis-major output of the WHOLE tensor, (row0 + r) *
 * total_cols + col0 + c along rows (block_axis 1) and (col0 + c) * total_rows
 * + row0 + r along columns (block_axis 0); blocks are the whole tensor's, so
 * the offset along the block axis (col0, resp. row0) and the whole tensor's
 * length along it must be multiples of 32.  This is the data-parallel split
 * of the stochastic-rounding cast ("Format-Aware Fusion for Fast FP4
 * Pretraining", abstract: row-gradient stochastic rounding, here for token
 * shards of the weight-gradient operands held by different ranks).
 *
 *  shard   host pointer, required (NULL gives MX_ERR_ARG).  The piece must
 *          lie inside the whole tensor (MX_ERR_ARG otherwise).
 *  other arguments, outputs (the piece's own codes and scales, in its local
 *  coordinates) and errors as for mx_quantize; MX_ERR_SR_RANGE applies to the
 *  whole tensor's element count.
 */
MX_API int mx_quantize_shard(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                             int block_axis, mx_fmt fmt, mx_round rnd, uint64_t seed,
                             const mx_precond *pre, const mx_shard *shard, void *codes, void *scales,
                             mx_scale_layout sl, void *stream);

/*
 * mx_quantize_dual_shard -- mx_quantize_dual of one piece of a larger tensor,
 * each output equal to the matching slice of the whole tensor's output (the
 * stochastic-rounding positions of mx_quantize_shard).  Both axes are block
 * axes here, so row0, col0, total_rows and total_cols must all be multiples
 * of 32.  shard is required; arguments and errors otherwise as for
 * mx_quantize_dual.
 */
MX_API int mx_quantize_dual_shard(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                  mx_fmt fmt, mx_round rnd_rows, uint64_t seed_rows, mx_round rnd_cols,
                                  uint64_t seed_cols, const mx_precond *pre_cols, const mx_shard *shard,
                                  void *codes_rows, void *scales_rows, void *codes_cols, void *scales_cols,
                                  mx_scale_layout sl, void *stream);

/*
 * mx_quantize_nvfp4 -- the NVFP4 cast with a global or a CTA-local scale
 * domain, the two NVFP4 variants the abstract of "Format-Aware Fusion for
 * Fast FP4 Pretraining" names next to native MXFP4.  The pages do not define
 * them; the reading taken here is the public NVFP4 format:
 *  - blocks of 16 consecutive elements along the rows (block axis 1), E2M1
 *    elements (the MXFP4 codes), one E4M3 block scale per block;
 *  - one fp32 encode scale E per domain: the whole tensor (domain_rows = 0,
 *    "global"), or each group of domain_rows consecutive rows, all columns
 *    ("CTA-local": rows that one CTA of a fused producer can own, so that in
 *    such a producer the scale needs no grid-wide reduction; this cast runs
 *    both kinds as the same two passes over the input);
 *  - with a_D the largest finite |x| of a domain, E = 2688 / a_D (6 * 448, the
 *    largest E2M1 and E4M3 values; 1 when a_D = 0, the largest finite fp32
 *    when the quotient overflows); per block, with a_b its largest |x|, the
 *    block scale is the E4M3 code of (a_b / 6) * E (round to nearest even,
 *    saturating at 448), d its value, and each code the E2M1 code of
 *    x * (E / d) (nearest even, saturating at 6; 0 when d = 0); every step one
 *    IEEE fp32 operation, no flush.  A block holding a NaN or Inf gets the
 *    E4M3 NaN code 0x7F and zero codes;
 *  - a code P in a block of scale value d stands for P * d / E.
 *
 *  x          device, rows x cols (ldx elements per row), fp32 or bf16,
 *             16-byte aligned, ldx * sizeof(elem) a multiple of 16.
 *  cols       a multiple of 16 (MX_ERR_SHAPE).
 *  codes      device, rows x cols / 2 bytes (two codes per byte, even element
 *             in the low nibble), 16-byte aligned.
 *  scales     device, mx_nvfp4_scales_bytes(sl, rows, cols) bytes: plain
 *             (rows x cols / 16), or the tensor-core atom layout of
 *             MX_SCALES_MMA (or MX_SCALES_MMA_X4) over 16-element blocks.
 *  enc_scales device, mx_nvfp4_domains(rows, domain_rows) fp32 values: E of
 *             each domain (written; the global form also uses it while it
 *             runs, starting from zero).
 * Errors: MX_ERR_ARG, MX_ERR_ALIGN, MX_ERR_SHAPE, MX_ERR_UNSUPPORTED,
 * MX_ERR_CUDA.
 */
MX_API int mx_quantize_nvfp4(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                             int64_t domain_rows, void *codes, void *scales, mx_scale_layout sl,
                             float *enc_scales, void *stream);
/* Byte size of mx_quantize_nvfp4's scales, and its number of domains. */
MX_API size_t mx_nvfp4_scales_bytes(mx_scale_layout sl, int64_t rows, int64_t cols);
MX_API int64_t mx_nvfp4_domains(int64_t rows, int64_t domain_rows);

/*
 * mx_dequantize -- v = X * P (section 2), exact, rounded once to ydt.
 *
 *  codes, scales  device, as written by mx_quantize for (outer, inner).
 *  y              device, outer x inner, leading dimension ldy (elements),
 *                 16-byte aligned, ldy * sizeof(ydt) a multiple of 16.
 * A 0xFF scale gives NaN for its whole block; values beyond the output
 * type's range become +-Inf.
 * Errors: MX_ERR_ARG, MX_ERR_ALIGN, MX_ERR_SHAPE, MX_ERR_CUDA.
 */
MX_API int mx_dequantize(const void *codes, const void *scales, mx_fmt fmt, mx_scale_layout sl,
                  int64_t outer, int64_t inner, void *y, mx_dtype ydt, int64_t ldy,
                  void *stream);

/*
 * mx_gemm -- C = alpha * A * B^T, the block-scaled matmul of section 4's
 * compute flow on the fifth-generation tensor cores.
 *
 *  a_codes  device, M x K codes of format fa, quantized along K
 *           (block_axis 1 of an M x K tensor), 16-byte aligned; 32-byte
 *           aligned when fa is FP6, or FP4 outside the kind::mxf4 case.
 *  a_scales device, MX_SCALES_MMA layout for (M, K).
 *  b_codes  device, N x K codes of format fb, quantized along K.
 *  b_scales device, MX_SCALES_MMA layout for (N, K).
 *  c        device, M x N, leading dimension ldc, type cdt (fp32 or bf16,
 *           rounded to nearest even from the fp32 accumulator).
 *  workspace / ws_bytes  reserved; pass NULL / 0 (mx_gemm_workspace_bytes
 *           returns 0 in this build).
 *  b_codes has the same alignment rule for fb.
 * Supported: fa, fb each any of MX_E4M3, MX_E5M2, MX_E2M3, MX_E3M2, MX_E2M1
 * (mixed pairs included, e.g. MXFP4 weights x MXFP6 activations), with
 * K % 128 == 0 and any M, N >= 1.  Size limit: M, N and K at most 2^31 - 1 and
 * ceil(M / 128) * ceil(N / 128) at most 2^31 - 1 (the kernels index with
 * 32-bit integers); larger sizes give MX_ERR_UNSUPPORTED before anything is
 * launched.  fa == fb == MX_E2M1 with K % 256 == 0 runs
 * kind::mxf4 on the packed codes; every other pair runs kind::mxf8f6f4, whose
 * operands the copy engine expands to one code per byte in shared memory.
 * MX_INT8 operands give MX_ERR_UNSUPPORTED (sm_100a has no block-scaled
 * integer MMA).
 * Accumulation is fp32 on the tensor cores; |C - C_exact| stays within
 * 1e-5 * |alpha| * sum_k |a_mk b_nk| in the tested configurations.
 * Errors: MX_ERR_ARG, MX_ERR_ALIGN, MX_ERR_SHAPE, MX_ERR_UNSUPPORTED,
 * MX_ERR_CUDA.  A pipeline wait that exceeds its bound ends the kernel early
 * and records MX_ERR_TIMEOUT, read with mx_last_device_status.
 */
MX_API int mx_gemm(const void *a_codes, const void *a_scales, mx_fmt fa,
            const void *b_codes, const void *b_scales, mx_fmt fb,
            int64_t M, int64_t N, int64_t K, float alpha,
            void *c, mx_dtype cdt, int64_t ldc, void *workspace, size_t ws_bytes,
            void *stream);

/*
 * mx_gemm_quantize -- C = alpha * A * B^T as mx_gemm computes it, written
 * directly as MX codes and scales of C quantized along its rows (blocks of 32
 * consecutive columns), the layout the next GEMM reads as its A operand.  The
 * FP4-pretraining abstract's principle of a producer that writes the layout
 * its consumer reads, applied to the GEMM epilogue; the quantization is
 * Algorithm 1 (section 3) on the fp32 values fl32(alpha * acc), acc being the
 * GEMM's fp32 accumulator, so the result is the bytes mx_quantize(block_axis
 * 1) would write for the fp32 C that mx_gemm returns.
 *
 *  a_codes ... alpha   as for mx_gemm (same formats, K % 128 == 0, same
 *             size limit).
 *  out_fmt    element format of C's codes (any mx_fmt, MX_INT8 included).
 *  out_rnd, out_seed   RNE, or SR with C's element index m * N + n.
 *  out_codes  device, M x (N * bits / 8) bytes, 16-byte aligned.
 *  out_scales device, mx_scales_bytes(out_sl, M, N) bytes.
 *  N must be a multiple of 32 (MX_ERR_SHAPE).  With K == 0, C = 0: all codes
 *  and every byte of the scale buffer (padding included) are set to zero.
 * Errors: as mx_gemm, plus MX_ERR_SR_RANGE; a bounded-wait expiry is reported
 * by mx_last_device_status.
 */
MX_API int mx_gemm_quantize(const void *a_codes, const void *a_scales, mx_fmt fa,
                            const void *b_codes, const void *b_scales, mx_fmt fb,
                            int64_t M, int64_t N, int64_t K, float alpha,
                            mx_fmt out_fmt, mx_round out_rnd, uint64_t out_seed,
                            void *out_codes, void *out_scales, mx_scale_layout out_sl, void *stream);

/*
 * mx_gemm_nvfp4 -- C = alpha * A * B^T on NVFP4 operands written by
 * mx_quantize_nvfp4 (MX_SCALES_MMA), each element taken as P * d / E (the
 * reading of the global / CTA-local NVFP4 variants given at
 * mx_quantize_nvfp4).  The tensor cores accumulate sum_k (P_a d_a)(P_b d_b)
 * in fp32 (kind::mxf4nvf4, E4M3 block scales); the epilogue multiplies each
 * element by fl32(fl32(alpha / E_A[m]) / E_B[n]), E_A[m] being the encode
 * scale of the domain that holds row m of A and E_B[n] that of row n of B,
 * and rounds once to cdt.
 *
 *  a_codes, b_codes  device, M x K / 2 and N x K / 2 bytes (mx_quantize_nvfp4
 *             codes of A and B, K contiguous), 16-byte aligned.
 *  a_scales, b_scales  device, mx_nvfp4_scales_bytes(MX_SCALES_MMA, M, K) and
 *             (.., N, K) bytes, 16-byte aligned.
 *  a_enc, b_enc  device, mx_nvfp4_domains(M, a_domain_rows) and
 *             mx_nvfp4_domains(N, b_domain_rows) fp32 encode scales, 4-byte
 *             aligned; read only.
 *  a_domain_rows  rows of A per domain (0: one domain).
 *  b_domain_rows  rows of B per domain: 0 or a multiple of 32
 *             (MX_ERR_UNSUPPORTED otherwise; the epilogue applies one E_B per
 *             32 columns of C).
 *  K          a multiple of 16 (MX_ERR_SHAPE) and of 256 (MX_ERR_UNSUPPORTED).
 *  c, cdt, ldc  as for mx_gemm (MX_F32 or MX_BF16).
 * Errors: MX_ERR_ARG, MX_ERR_ALIGN, MX_ERR_SHAPE, MX_ERR_UNSUPPORTED,
 * MX_ERR_CUDA; MX_ERR_TIMEOUT later through mx_last_device_status.
 */
MX_API int mx_gemm_nvfp4(const void *a_codes, const void *a_scales, const float *a_enc, int64_t a_domain_rows,
                         const void *b_codes, const void *b_scales, const float *b_enc, int64_t b_domain_rows,
                         int64_t M, int64_t N, int64_t K, float alpha, void *c, mx_dtype cdt, int64_t ldc,
                         void *stream);

/* mx_gemm_nvfp4 with both operands' block scales in MX_SCALES_MMA_X4
 * (mx_nvfp4_scales_bytes(MX_SCALES_MMA_X4, ..) bytes, written by
 * mx_quantize_nvfp4 with that layout): the same results bit for bit, with
 * the 128-lane scale copies (six per 256-element slice instead of twelve). */
MX_API int mx_gemm_nvfp4_x4(const void *a_codes, const void *a_scales, const float *a_enc, int64_t a_domain_rows,
                            const void *b_codes, const void *b_scales, const float *b_enc, int64_t b_domain_rows,
                            int64_t M, int64_t N, int64_t K, float alpha, void *c, mx_dtype cdt, int64_t ldc,
                            void *stream);

/*
 * mx_gemm_x4, mx_gemm_quantize_x4 -- mx_gemm and mx_gemm_quantize with both
 * operands' scales in MX_SCALES_MMA_X4 (mx_scales_bytes(MX_SCALES_MMA_X4, ..)
 * bytes each) instead of MX_SCALES_MMA: the same arguments (mx_gemm_x4 has no
 * workspace), the same results bit for bit.  They run the 256 x 256 CTA-pair
 * kernel for every shape, whose tensor-memory scale copies are then the
 * 128-lane shapes instead of the replicating ones: fewer copy instructions
 * per K step (measured 9-11 % faster on the MXFP4 GEMMs of the benchmark).
 * The quantizing form writes C's scales in out_sl, any layout (MX_SCALES_MMA_X4
 * for a chain of such GEMMs).  The kernel-forcing debug hook accepts only the
 * pair kernel here (MX_ERR_UNSUPPORTED otherwise).
 */
MX_API int mx_gemm_x4(const void *a_codes, const void *a_scales, mx_fmt fa,
                      const void *b_codes, const void *b_scales, mx_fmt fb,
                      int64_t M, int64_t N, int64_t K, float alpha,
                      void *c, mx_dtype cdt, int64_t ldc, void *stream);
MX_API int mx_gemm_quantize_x4(const void *a_codes, const void *a_scales, mx_fmt fa,
                               const void *b_codes, const void *b_scales, mx_fmt fb,
                               int64_t M, int64_t N, int64_t K, float alpha,
                               mx_fmt out_fmt, mx_round out_rnd, uint64_t out_seed,
                               void *out_codes, void *out_scales, mx_scale_layout out_sl, void *stream);

/* Byte sizes of the buffers above (0 for invalid arguments). */
MX_API size_t mx_codes_bytes(mx_fmt fmt, int64_t outer, int64_t inner);
MX_API size_t mx_scales_bytes(mx_scale_layout sl, int64_t outer, int64_t inner);
MX_API size_t mx_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Synchronises `stream`, then returns and clears the current device's status
 * words (one for the GEMM kernels, one for the casts): MX_OK, or
 * MX_ERR_TIMEOUT if a kernel gave up a bounded wait since the last call.
 * MX_ERR_CUDA if the synchronisation itself failed.  In the debug build
 * (libmx_debug.so, compiled with MX_DEBUG) every code and scale store of the
 * casts and the NVFP4 cast, and every code and scale load of the decode,
 * checks its byte range against its buffer's size first; a range
 * outside the buffer is skipped and reported here as MX_ERR_BOUNDS (after a
 * timeout, which takes precedence).  The release build has no such checks. */
MX_API int mx_last_device_status(void *stream);

/* Static description of a status code. */
MX_API const char *mx_status_str(int status);

/* ABI version of this header: 1. */
MX_API int mx_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MX_H */
