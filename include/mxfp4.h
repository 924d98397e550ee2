/*
 * mxfp4.h -- C ABI of the B200 (sm_100a) MXFP4 quantise-and-contract path of
 * the ALTO MXFP4 training recipe ("Training an MoE LLM in MXFP4: How We
 * Closed the Gap to BF16").
 *
 * What the path computes, and where the pages say so:
 *  - MX format: E2M1 elements with one UE8M0 (power-of-two) scale per block
 *    -- roboaidigest, "What ALTO Actually Does"; the format is the Open
 *    Compute Project Microscaling (MX) one named in that article's opening.
 *  - hybrid 1D/2D block quantisation, randomized Hadamard transforms (RHT),
 *    stochastic rounding (SR), simplified weight de-oscillation -- the
 *    abstract (foxai.news / scholarbro / paperdot) and roboaidigest "What
 *    ALTO Actually Does".
 *  - the master weight is updated in full precision while the GEMM only
 *    sees its quantised value, and weights near a bin boundary oscillate --
 *    roboaidigest "What ALTO Actually Does" (de-oscillation motivation).
 *  - the expert matrices of the MoE dominate compute and memory, so the
 *    block-scaled GEMMs of the expert linear layers are the contraction --
 *    roboaidigest "What ALTO Actually Does".
 * The pages give no bit-level rule.  The readings used by this library:
 *  - block 32; scale E = floor(log2(amax)) - 2, clamped to [-127, 127],
 *    stored as the byte E + 127; elements v = y * 2^-E saturate to +-6.
 *  - round-to-nearest onto {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the even
 *    code; the sign is kept (a negative value rounding to zero is code 8).
 *  - SR: lo <= |v| < hi adjacent grid points, f = (|v|-lo)/(hi-lo),
 *    F = floor(f * 2^16); round up iff F + r16 >= 2^16, r16 = 16 bits of a
 *    Philox4x32-10 stream; |v| >= 6 gives 6, the sign is kept.
 *  - RHT, d = 16: per 16-element chunk y = FWHT16((s .* x) / 4) as a
 *    radix-2 butterfly with strides 1, 2, 4, 8, each (a, b) -> (a+b, a-b)
 *    rounded in binary32, natural (Sylvester) output order; s in {+-1}^16.
 *  - Philox4x32-10 (Salmon et al., SC'11): key = (seed lo, seed hi);
 *    counter = (g lo, g hi, offset, tag), tag 0 = SR, tag 1 = RHT signs.
 *    RHT sign i = -1 iff bit i of word 0 of Philox(rht_seed; 0, 0, 0, 1).
 *    SR element n (row-major index in the OUTPUT layout): g = n >> 4, word
 *    w = (n >> 2) & 3 with bytes b0..b3; elements 4m..4m+3 take b2:b0, its
 *    16-bit bit reversal, b3:b1, its bit reversal (the random-bit layout of
 *    the sm_100 four-element stochastic-rounding conversion).
 *  - de-oscillation: see mxfp4_deosc_update.
 * Quantised codes, scales, SR decisions and de-oscillation state are a bit
 * contract; GEMM outputs are binary32 accumulations of exact products.
 *
 * Conventions of every entry point:
 *  - returns mxfp4_status; 0 on success, a negative code otherwise, with a
 *    message available from mxfp4_last_error().  Host-detectable argument
 *    errors are reported before anything is launched.
 *  - asynchronous on the caller's CUDA stream (`stream` is a cudaStream_t;
 *    NULL means the legacy default stream).  Device-side problems (invalid
 *    group offsets, a bounded wait that timed out) set a device status word
 *    read by mxfp4_check_device_status().
 *  - allocates nothing: the caller owns every buffer.  Pointers are device
 *    pointers unless stated otherwise and must be 16-byte aligned.
 *  - no C++ exception crosses this boundary.
 *
 * Packed layouts:
 *  - codes: a [R, C] matrix of E2M1 codes is stored as R rows of C/2 bytes;
 *    element (r, c) sits in byte r*C/2 + c/2, low nibble for even c.
 *  - canonical scales: 1D blocks -> [R, C/32] bytes; 2D 32x32 blocks ->
 *    [R/32, C/32] bytes.
 *  - tensor-core ("MMA") scales: the per-row scale matrix [R, S] (S = C/32;
 *    for 2D blocks each row repeats its block's scale) in chunks of 128
 *    rows x 4 scales = 512 bytes; byte of (r, s) at
 *      ((r/128) * ceil(S/4) + s/4) * 512 + (r%32)*16 + ((r/32)%4)*4 + s%4.
 *    Size mxfp4_mma_scale_bytes(R, S).  Bytes for rows >= R or s >= S are
 *    padding: never written, and never read for any in-range output.
 */
#ifndef MXFP4_H
#define MXFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MXFP4_API __attribute__((visibility("default")))
#else
#define MXFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXFP4_OK = 0,
    MXFP4_ERR_INVALID_ARG = -1,       /* null pointer, bad enum, negative size */
    MXFP4_ERR_UNSUPPORTED_SHAPE = -2, /* block dim not a multiple of 32, ... */
    MXFP4_ERR_MISALIGNED = -3,        /* pointer or stride not 16-byte aligned */
    MXFP4_ERR_CUDA = -4,              /* a CUDA runtime/driver call failed */
    MXFP4_ERR_DEVICE_TIMEOUT = -5,    /* a bounded device-side wait expired */
    MXFP4_ERR_DEVICE_BAD_INPUT = -6   /* device-side check failed (group offsets) */
} mxfp4_status;

enum { MXFP4_DTYPE_BF16 = 0, MXFP4_DTYPE_F32 = 1 };
enum { MXFP4_BLOCK_1X32 = 0, MXFP4_BLOCK_32X32 = 1 };
enum { MXFP4_ROUND_NEAREST = 0, MXFP4_ROUND_STOCHASTIC = 1 };
enum { MXFP4_GEMM_FPROP = 0, MXFP4_GEMM_DGRAD = 1, MXFP4_GEMM_WGRAD = 2 };

/* Quantisation recipe of one call. */
typedef struct {
    int block;          /* MXFP4_BLOCK_1X32 or MXFP4_BLOCK_32X32 */
    int along_rows;     /* 1D only.  0: blocks run along the last dim (each
                           input row is one output row).  1: blocks run along
                           dim 0 (the token dim of weight-gradient operands);
                           the output is the transpose, [cols, rows]. */
    int rht_d;          /* 0 = no RHT, 16 = RHT along the block dim */
    uint64_t rht_seed;
    int rounding;       /* MXFP4_ROUND_NEAREST or MXFP4_ROUND_STOCHASTIC */
    uint64_t sr_seed;
    uint32_t sr_offset; /* Philox counter word 2; distinct per tensor */
} mxfp4_quant_params;

/* Outputs of a quantisation call (per group, contiguous, groups back to
 * back).  Any pointer may be NULL except `codes`. */
typedef struct {
    uint8_t* codes;        /* [Ro, Co/2] packed codes (Ro, Co = output shape) */
    uint8_t* scales;       /* canonical scales (1D [Ro, Co/32]; 2D [R/32, C/32]) */
    uint8_t* scales_mma;   /* tensor-core layout of the output's per-row scales */
    uint8_t* codes_t;      /* 2D only: codes of the transpose, [C, R/2] */
    uint8_t* scales_mma_t; /* 2D only: tensor-core layout scales of the transpose */
} mxfp4_quant_outputs;

/* Bytes of a tensor-core scale buffer for a [rows, nscales] scale matrix. */
MXFP4_API size_t mxfp4_mma_scale_bytes(int64_t rows, int64_t nscales);

/* Quantise `groups` independent [rows, cols] matrices to MXFP4.
 *  in      : device, bf16 or f32; matrix g starts at in + g*rows*ld
 *            elements; rows are `ld` elements apart (ld >= cols).
 *  layout  : 1D along the last dim -> output [rows, cols]; 1D along rows ->
 *            output [cols, rows]; 2D -> output [rows, cols].
 *  shapes  : the block dim (and for 2D both dims) must be a multiple of 32;
 *            with RHT the RHT dim is the block dim; for 1D blocks groups *
 *            rows (and, along rows, groups * cols) must be below 2^31.
 *            Otherwise MXFP4_ERR_UNSUPPORTED_SHAPE.
 *  2D with rht_d = 16 applies the RHT along the last dim before blocking;
 *  codes_t/scales_mma_t are then the codes of (W R)^T.
 * Passage: the abstract, which names hybrid 1D/2D blocks, the RHT and SR as
 * the recipe's quantisation techniques; roboaidigest "What ALTO Actually
 * Does" (E2M1 + UE8M0 per block). */
MXFP4_API mxfp4_status mxfp4_quantize(const void* in, int in_dtype, int64_t groups, int64_t rows, int64_t cols,
                            int64_t ld, const mxfp4_quant_params* params, const mxfp4_quant_outputs* out,
                            void* stream);

/* Quantise one activation or gradient tensor in both 1D directions from a
 * single read of the input: the contraction-dim codes (1x32 blocks along the
 * last dim, as mxfp4_quantize with along_rows = 0) and the token-dim codes
 * (1x32 blocks along dim 0, output [cols, rows], as along_rows = 1).
 *  in, groups, rows, cols, ld : as mxfp4_quantize.
 *  row_params : the along-cols direction (along_rows must be 0, block 1x32).
 *  col_params : the along-rows direction (along_rows must be 1, block 1x32).
 *  Both directions use the same rounding and, for SR, the same sr_seed;
 *  rht_d, rht_seed and sr_offset are per direction.
 *  row_out, col_out : outputs of the two directions (codes_t/scales_mma_t
 *  must be NULL).  Every output equals, bit for bit, what the two separate
 *  mxfp4_quantize calls with these params write.
 *  shapes : rows % 32 == 0, cols % 32 == 0, groups * rows < 2^31 and
 *  groups * cols < 2^31, else MXFP4_ERR_UNSUPPORTED_SHAPE.
 * Passage: the abstract (hybrid 1D/2D blocks: activations and gradients enter
 * the forward/backward GEMMs along the contraction dim and the weight-gradient
 * GEMM along the token dim, the latter with the RHT). */
MXFP4_API mxfp4_status mxfp4_quantize_dual(const void* in, int in_dtype, int64_t groups, int64_t rows, int64_t cols,
                                 int64_t ld, const mxfp4_quant_params* row_params,
                                 const mxfp4_quant_params* col_params, const mxfp4_quant_outputs* row_out,
                                 const mxfp4_quant_outputs* col_out, void* stream);

/* Standalone randomized Hadamard transform, d = 16, in the butterfly order
 * stated above, with the signs of `seed`.
 *  axis 1: along the last dim, out[r, 16j:16j+16] = RHT(in[r, 16j:16j+16]);
 *          cols % 16 == 0.
 *  axis 0: along dim 0 (the token dim of the weight-gradient operands),
 *          out[16j:16j+16, c] = RHT(in[16j:16j+16, c]); rows % 16 == 0.
 *          This is the transform the along-rows quantisation applies before
 *          blocking, here with the output kept in the input's layout.
 *  in  : device [rows, cols] (row stride ld elements), bf16 or f32.
 *  out : device [rows, cols] contiguous, out_dtype F32 (bit contract) or
 *        BF16 (round-to-nearest-even of the F32 result; a NaN stays a NaN,
 *        its payload unspecified).
 *  Errors: MXFP4_ERR_INVALID_ARG for a null pointer, a bad dtype or axis, or
 *  d != 16; MXFP4_ERR_UNSUPPORTED_SHAPE when the transformed dim is not a
 *  multiple of 16; MXFP4_ERR_MISALIGNED for pointers or rows not 16-byte
 *  aligned.
 * Passage: the abstract, which lists randomized Hadamard transforms among the
 * recipe's techniques. */
MXFP4_API mxfp4_status mxfp4_rht(const void* in, int in_dtype, int64_t rows, int64_t cols, int64_t ld, int axis,
                                 int d, uint64_t seed, void* out, int out_dtype, void* stream);

/* De-oscillation parameters. */
typedef struct {
    uint32_t flip_threshold; /* freeze once the flip count reaches this (default 4), 1..7 */
    uint32_t reset_period;   /* 0 = never; else clear counts and frozen bits on steps
                                that are multiples of it */
    uint32_t freeze_lower;   /* 0: a weight freezes at the code of its freezing flip
                                (the new code).  1 (variant): it freezes at the
                                lower-magnitude code of that flip (code & 7; ties
                                keep the new code). */
} mxfp4_deosc_params;

/* Re-quantise fp32 master weights with 32x32 blocks and nearest rounding,
 * and update the per-weight de-oscillation state (one byte per weight:
 * bits 0-3 previous code, bits 4-6 flip count saturating at 7, bit 7
 * frozen).
 *  step == 0: initialise the state to (nearest code, 0, not frozen).
 *  step  > 0: if reset_period divides step, clear count and frozen first;
 *    q = nearest code under the block scale of the current master weights;
 *    a frozen weight emits its stored code and keeps its state; otherwise,
 *    when q differs from the stored code the count increments, q is
 *    stored, and the weight freezes once count >= flip_threshold; it emits q
 *    (with freeze_lower, a weight freezing now stores and emits the
 *    lower-magnitude of the old stored code and q instead).
 *  Scales always follow the current master weights.
 *  master: device f32 [groups, rows, cols]; state: device inout, same shape
 *  (one byte each).  out: codes [groups, rows, cols/2] plus any of the
 *  optional outputs of mxfp4_quant_outputs (2D layouts).
 * Passage: roboaidigest "What ALTO Actually Does" (why weights oscillate
 * between two bins while the master weight barely moves) and the abstract
 * (a simplified de-oscillation scheme derived from TetraJet-v2); the rule
 * itself is this library's reading. */
MXFP4_API mxfp4_status mxfp4_deosc_update(const float* master, int64_t groups, int64_t rows, int64_t cols, uint32_t step,
                                const mxfp4_deosc_params* params, uint8_t* state, const mxfp4_quant_outputs* out,
                                void* stream);

/* One operand of the grouped GEMM: packed codes (K contiguous) and its
 * per-row scales in the tensor-core layout. */
typedef struct {
    const uint8_t* codes;
    const uint8_t* scales_mma;
} mxfp4_operand;

/* Grouped block-scaled MXFP4 GEMM on tcgen05 tensor cores, binary32
 * accumulation in tensor memory, binary32 output.  Every result is
 * D = deq(A) * deq(B)^T per group, dequantised exactly.
 *  FPROP / DGRAD (groups split the rows of A):
 *    A: [M, K] (M = group_offsets[G]); B: [G, N, K] (group g's matrix at
 *    codes + g*N*K/2, scales + g*mxfp4_mma_scale_bytes(N, K/32));
 *    D: [M, N] with row stride ldo floats; rows of group g are
 *    [off[g], off[g+1]).  FPROP: Y = X W^T with B = W.  DGRAD: dX = dY W with
 *    B = W^T, i.e. the codes_t / scales_mma_t of the 2D weight quantisation.
 *  WGRAD (groups split the contraction dim):
 *    A: [M, K] (dY^T of all tokens, K = group_offsets[G]); B: [N, K] (X^T);
 *    D: [G, M, N], D_g = A[:, off[g]:off[g+1]] * B[:, off[g]:off[g+1]]^T,
 *    row stride ldo, group stride M*ldo; an empty group gives zeros.
 *  group_offsets: device int32 [G+1], non-decreasing, multiples of 128,
 *    group_offsets[0] = 0, G <= 1023.  Checked on the device: an invalid
 *    array records MXFP4_ERR_DEVICE_BAD_INPUT and the call writes nothing.
 *  M_or_total: FPROP/DGRAD M (= off[G]); WGRAD: M.  K_or_total: FPROP/DGRAD
 *    K; WGRAD: off[G].  Output tiles are 256 x 192, computed by pairs of
 *    CTAs (tcgen05 cta_group::2) for G <= 255, and 128 x 192 by single CTAs
 *    above that or when the environment sets MXFP4_GEMM_CTA_PAIRS=0 (both
 *    expert widths, 2880 and 5760, are multiples of 192; other N are
 *    clipped at the edge).  K % 64 == 0, ldo % 4 == 0, ldo >= N.
 * Passage: roboaidigest "What ALTO Actually Does" (expert matrices dominate
 * compute and memory; the GEMM only ever sees quantised values). */
MXFP4_API mxfp4_status mxfp4_grouped_gemm(int op, int num_groups, const int32_t* group_offsets, mxfp4_operand a,
                                mxfp4_operand b, int64_t M_or_total, int64_t N, int64_t K_or_total, float* out,
                                int64_t ldo, void* stream);

/* FPROP / DGRAD with a fused epilogue: instead of the binary32 D, write
 *  - y: D rounded to bf16 (nearest even), [M, N] with row stride ldy
 *    elements (ldy >= N, ldy % 8 == 0), as raw bf16 bit patterns;
 *  - q->codes [M, N/2] and q->scales [M, N/32] / q->scales_mma (either may
 *    be null): the 1x32-along-N MXFP4 quantisation of y, bit-identical to
 *    mxfp4_quantize(y, bf16, 1 group, M rows, N cols, ld = ldy) with the
 *    params qp (NULL: nearest rounding).  qp must be 1x32 along the last
 *    dim without RHT; its rounding is nearest or stochastic (sr_seed,
 *    sr_offset as for mxfp4_quantize: element n = row * N + col).
 *    q->codes_t / scales_mma_t must be null.
 * A, B, group_offsets, M, N, K as for mxfp4_grouped_gemm.  Needs the
 * CTA-pair kernel (G <= 255, not disabled by MXFP4_GEMM_CTA_PAIRS=0),
 * N % 32 == 0 and K > 0, else MXFP4_ERR_UNSUPPORTED_SHAPE.  Every 32-column
 * chunk of an output row is one lane's registers in the epilogue, so the
 * block quantisation costs no exchange and the binary32 output never
 * reaches HBM.
 * Passage: roboaidigest "What ALTO Actually Does" (activations take 1D
 * blocks; the next GEMM only ever sees quantised values) and the abstract
 * (hybrid 1D/2D block quantisation; SR on gradients, e.g. a dgrad output). */
MXFP4_API mxfp4_status mxfp4_grouped_gemm_fused(int op, int num_groups, const int32_t* group_offsets,
                                                mxfp4_operand a, mxfp4_operand b, int64_t M, int64_t N, int64_t K,
                                                uint16_t* y, int64_t ldy, const mxfp4_quant_outputs* q,
                                                const mxfp4_quant_params* qp, void* stream);

/* Tensor-pipe peak probe, a measurement helper and not a step of the path:
 * one CTA pair per two SMs (the grouped GEMM's launch shape) issues
 * mmas_per_pair block-scaled MXFP4 MMAs of the GEMM's own shape (M = 256,
 * N = 192, K = 64, UE8M0 scales) back to back on operands resident in shared
 * memory, with no loads and no output.  Asynchronous on `stream`; the caller
 * times the launch.  *flops (host) receives the launch's floating-point
 * operations, 2 M N K per MMA.  Errors: MXFP4_ERR_INVALID_ARG unless
 * 1 <= mmas_per_pair <= 2^22 and flops is non-null; MXFP4_ERR_CUDA if the
 * launch fails; a wait that runs out sets MXFP4_ERR_DEVICE_TIMEOUT for
 * mxfp4_check_device_status.
 * Passage: none; it measures the FP4 roofline that the GEMMs are compared
 * with, not an operation of the method. */
MXFP4_API mxfp4_status mxfp4_mma_peak_probe(int64_t mmas_per_pair, double* flops, void* stream);

/* Self-test of failure detection, not a step of the path: one small kernel
 * in which a thread waits, through the same bounded wait as every pipeline
 * role, on a barrier that nothing completes.  When the wait budget (2 s)
 * runs out it records a timeout for the "mma" role in the device status word
 * and sets its CTA's abort flag, which ends a second thread's wait (started
 * 50 ms later) without a second record; the kernel then returns and the
 * context stays usable.  A following mxfp4_check_device_status() returns
 * MXFP4_ERR_DEVICE_TIMEOUT naming that role only.  Asynchronous on
 * `stream`.  Errors: MXFP4_ERR_CUDA if the launch fails.
 * Passage: none; it checks the library's own failure detection. */
MXFP4_API mxfp4_status mxfp4_selftest_wait_timeout(void* stream);

/* Copy the last error message of this thread into buf (NUL-terminated,
 * truncated to len).  Returns the message length. */
MXFP4_API size_t mxfp4_last_error(char* buf, size_t len);

/* Read and clear the device status word of the current device, then
 * synchronise `stream`.  Returns MXFP4_OK, MXFP4_ERR_DEVICE_TIMEOUT or
 * MXFP4_ERR_DEVICE_BAD_INPUT (details via mxfp4_last_error), or
 * MXFP4_ERR_CUDA if the read itself fails.
 * The word is one per device, shared by every stream and every call of this
 * library in the process.  The check takes it with one atomic exchange
 * (read and clear in a single step), issued on `stream` after the work
 * already queued there, so no recorded bit is lost.  It does not wait for
 * work on other streams: a status that a kernel on another stream records
 * is reported by whichever check runs next, on whatever stream, so it can
 * be attributed to the wrong stream when calls overlap. */
MXFP4_API mxfp4_status mxfp4_check_device_status(void* stream);

/* Library version string. */
MXFP4_API const char* mxfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MXFP4_H */
