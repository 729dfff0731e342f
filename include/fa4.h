/*
 * fa4.h -- C ABI of the B200 (sm_100a) FP4 quantization + block-scaled GEMM
 * library (libfa4.so).
 *
 * The operation is the one the pages on format-aware fusion for FP4 describe:
 * a quantization producer bound to its scale domain and its consumer layout
 * ("Format-Aware Fusion: The Engineering Practice That Doubles FP4
 * Pretraining Throughput", section "The Design Philosophy of Format-Aware
 * Fusion"), i.e. block amax -> scale -> divide -> E2M1 -> two values per byte
 * ("FP4 Is No Longer Just a Hardware Feature -- The NVFP4 Software Stack Is
 * Taking Shape", section "The first change: PyTorch is bringing FP4 packing
 * into compiler fusion"), with the scales written in the storage the tensor
 * cores read, followed by the FP4 tensor-core matmul.
 *
 * Conventions for every entry point:
 *  - Pointers named x/X/dY/D/workspace and the members of fa4_qtensor are
 *    DEVICE pointers, allocated and owned by the caller.  The library never
 *    allocates device memory and never synchronizes, except
 *    fa4_check_device_status.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  All work is enqueued asynchronously on it.
 *  - Every function returns an fa4_status; nothing throws across the ABI.
 *    Argument errors are detected on the host before anything is launched.
 *    A launch failure returns FA4_ERR_CUDA (cudaGetLastError).
 *  - Shapes: a quantized operand Q[R, K] may have any number of rows R and
 *    K (the block dimension) a multiple of 32; an input x[rows, cols] has
 *    cols a multiple of 8.  GEMM: any M and N, K a multiple of 32.  Scale
 *    atoms are padded (rows to a multiple of 128, blocks to a multiple of 4,
 *    the padding written as zero bytes).  Leading dimensions in elements,
 *    multiples of 8 and >= the row length; every pointer 16-byte aligned.
 *    Anything else returns FA4_ERR_SHAPE / FA4_ERR_ALIGN.
 *  - Inputs must be finite; with a non-finite input the output bytes are
 *    unspecified (no error is raised).
 *  - Workspace: the first FA4_WS_HEADER_BYTES bytes hold a sticky device
 *    status word that bounded waits inside the kernels set on timeout.  The
 *    caller zero-fills the workspace (or calls fa4_workspace_init) once
 *    before first use; fa4_check_device_status reads and clears the word.
 *  - Thread-safe: tensor-memory-access descriptors are encoded on the host
 *    for every call and passed by value to the kernel; the only global state
 *    is the driver entry point looked up once and, for
 *    fa4_quantize_nvfp4_global_noalloc, a mutex-guarded per-device pointer
 *    to its static scratch array.
 */
#ifndef FA4_H
#define FA4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FA4_WS_HEADER_BYTES 256

/* Exported symbols (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define FA4_API __attribute__((visibility("default")))
#else
#define FA4_API
#endif

/* Scale domains ("Format-Aware Fusion...", section "The Design Philosophy of
 * Format-Aware Fusion": native mxfp, global nvfp, CTA-local nvfp).
 *  FA4_MXFP4        32-value blocks, power-of-two E8M0 scale byte.
 *  FA4_NVFP4_GLOBAL 16-value blocks, E4M3 scale byte, one FP32 decode scale
 *                   for the tensor ("FP4 Is No Longer Just a Hardware
 *                   Feature...", section "NVFP4 is more than a 4-bit value").
 *  FA4_NVFP4_CTA    as NVFP4_GLOBAL but one FP32 decode scale per 128x128
 *                   tile of the quantized operand, [ceil(R/128)][ceil(K/128)]
 *                   (a tile cut by the operand's edge takes the amax of the
 *                   values it holds).
 *  FA4_MXFP4_NOCLIP MXFP4 with the other power-of-two scale rule: the
 *                   smallest e with amax <= 6 * 2^e, so no value saturates
 *                   (FA4_MXFP4 takes floor(log2 amax) - 2 and saturates
 *                   the top of the range).  Same payload, scale layout and
 *                   scale type as FA4_MXFP4: its operands multiply in a GEMM
 *                   called with FA4_MXFP4 or FA4_MXFP4_NOCLIP alike. */
typedef enum {
  FA4_MXFP4 = 0,
  FA4_NVFP4_GLOBAL = 1,
  FA4_NVFP4_CTA = 2,
  FA4_MXFP4_NOCLIP = 3
} fa4_format;

/* E2M1 rounding: round-to-nearest-even, or stochastic rounding with 16
 * Philox4x32-7 bits u per element keyed by `seed` ("Format-Aware Fusion...",
 * section "Two Key Numerical Techniques": row-gradient stochastic rounding):
 * between the neighbouring grid values lo <= |y| < hi, with
 * t = (|y| - lo) / (hi - lo) * 65536, the value rounds up iff u < floor(t). */
typedef enum { FA4_RNE = 0, FA4_SR = 1 } fa4_round;

/* Orientation of the quantized operand Q[R, K] relative to the bf16 input
 * x[rows, cols] (row-major, leading dimension ld):
 *   FA4_ROWWISE: Q = x,   R = rows, K = cols (blocks run along a row of x)
 *   FA4_COLWISE: Q = x^T, R = cols, K = rows (blocks run down a column of x;
 *                x^T is never materialized). */
typedef enum { FA4_ROWWISE = 0, FA4_COLWISE = 1 } fa4_orient;

typedef enum { FA4_OUT_BF16 = 0, FA4_OUT_FP32 = 1 } fa4_out_dtype;

typedef enum {
  FA4_OK = 0,
  FA4_ERR_INVALID_ARG = 1, /* null pointer, bad enum value */
  FA4_ERR_SHAPE = 2,       /* K not a multiple of 32, bad ld, empty tensor */
  FA4_ERR_ALIGN = 3,       /* pointer not 16-byte aligned */
  FA4_ERR_UNSUPPORTED = 4, /* e.g. Hadamard with NVFP4, mixed GEMM formats */
  FA4_ERR_WORKSPACE = 5,   /* workspace missing or smaller than required */
  FA4_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
  FA4_ERR_TIMEOUT = 7      /* a bounded device wait gave up (device status) */
} fa4_status;

/* A quantized operand Q[R, K] (all device pointers, caller-owned):
 *  payload      R*K/2 bytes, K-major: byte j of row r holds element 2j in its
 *               low nibble and element 2j+1 in its high nibble (E2M1 code =
 *               sign<<3 | exponent<<1 | mantissa).
 *  scales       one byte per block (E8M0 for MXFP4, E4M3 for NVFP4) in the
 *               128-row x 4-block atom layout the block-scaled tensor-core
 *               MMA reads: byte offset of (row r, block kb), with Kb4 =
 *               K/block rounded up to a multiple of 4,
 *               ((r/128)*(Kb4/4) + kb/4)*512 + (r%32)*16 + ((r%128)/32)*4
 *               + kb%4.  ceil(R/128)*128*Kb4 bytes; the bytes of rows >= R
 *               and blocks >= K/block are zero.
 *  tensor_scale FP32 decode scales: NVFP4_GLOBAL 1 value, NVFP4_CTA
 *               ceil(R/128)*ceil(K/128) values, row-major; unused (may be
 *               NULL) for MXFP4.  value = e2m1 * block scale * tensor_scale. */
typedef struct {
  void *payload;
  void *scales;
  float *tensor_scale;
} fa4_qtensor;

/* Sizes of a quantized operand of the bf16 input x[rows, cols] and the
 * workspace fa4_quantize needs.  Host only; any output pointer may be NULL.
 * Errors: FA4_ERR_SHAPE, FA4_ERR_INVALID_ARG. */
FA4_API fa4_status fa4_quant_sizes(int64_t rows, int64_t cols, fa4_format fmt, fa4_orient orient,
                           size_t *payload_bytes, size_t *scale_bytes, size_t *tscale_count,
                           size_t *workspace_bytes);

/* Quantize bf16 x[rows, cols] (leading dimension ld elements) into `out`
 * ("FP4 Is No Longer Just a Hardware Feature...", section "The first change":
 * block amax, scale, divide, convert to E2M1, pack two values per byte).
 * MXFP4 and NVFP4_CTA read x once; NVFP4_GLOBAL reads it twice (tensor amax,
 * then quantize).  The scale rules:
 *  MXFP4: e = floor(log2 amax_b) - 2 clamped to [-127, 127] (amax_b = 0 gives
 *         -127); scale byte e + 127; y = x * 2^-e.
 *  NVFP4: s_enc = 2688 / amax_t (1 when amax_t is 0 or the quotient is not
 *         finite), decode scale 1/s_enc; block scale (amax_b / 6) * s_enc
 *         clamped to [2^-9, 448] and rounded to E4M3; y = x * (s_enc / that
 *         E4M3 value).  amax_t is the tensor amax (GLOBAL) or the 128x128
 *         tile amax of Q (CTA).  All binary32, round-to-nearest-even.
 * Then y -> E2M1 by RNE (|y| >= 6 gives 6, the sign is kept) or SR.  SR bits
 * for element Q[r][k] come from counter (r*K + k) >> 3 of Philox4x32-7 keyed
 * by `seed`.  Errors: SHAPE, ALIGN, INVALID_ARG, WORKSPACE, CUDA. */
FA4_API fa4_status fa4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld, fa4_format fmt,
                        fa4_round rnd, fa4_orient orient, uint64_t seed, fa4_qtensor out,
                        void *workspace, size_t workspace_bytes, void *stream);

/* Column-wise MXFP4 quantization of x[rows, cols] with a fixed-sign 32-point
 * Hadamard applied to each 32-value block first ("Format-Aware Fusion...",
 * section "Two Key Numerical Techniques": fixed-sign 32-value Hadamard
 * weight-gradient preconditioning).  For each block v of 32 consecutive
 * elements down a column: y = H32 (s .* v), H32 the unnormalised Sylvester
 * matrix (H H^T = 32 I), s_j = -1 iff bit j of sign_mask, computed by the
 * butterfly with strides 1,2,4,8,16; then MXFP4 as in fa4_quantize.  A GEMM
 * of two such operands carries a factor 32: pass alpha = 1/32.
 * Errors: as fa4_quantize. */
FA4_API fa4_status fa4_hadamard32_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld,
                                   uint32_t sign_mask, fa4_round rnd, uint64_t seed,
                                   fa4_qtensor out, void *workspace, size_t workspace_bytes,
                                   void *stream);

/* Dual-orientation producer: one read of bf16 x[rows, cols] writes two
 * quantized operands ("Format-Aware Fusion...", section "The Design
 * Philosophy of Format-Aware Fusion": the producer fused with its consumers'
 * layouts; what the backward pass keeps of an activation is then its
 * column-wise FP4 operand for the weight gradient):
 *   row_out = fa4_quantize(x, row_fmt, row_rnd, FA4_ROWWISE, row_seed)
 *   col_out = col_hadamard ? fa4_hadamard32_quantize(x, sign_mask, col_rnd, col_seed)
 *                          : fa4_quantize(x, FA4_MXFP4, col_rnd, FA4_COLWISE, col_seed)
 * byte for byte.  For an activation X this is the forward operand and the
 * saved wgrad operand; for dY the dgrad and wgrad operands.  The column-wise
 * operand is always MXFP4.  Workspace: as fa4_quantize for row_fmt (the
 * NVFP4-global amax pass reads x once more).  Errors: as fa4_quantize. */
FA4_API fa4_status fa4_quantize_dual(const void *x, int64_t rows, int64_t cols, int64_t ld,
                             fa4_format row_fmt, fa4_round row_rnd, uint64_t row_seed,
                             fa4_qtensor row_out, int col_hadamard, uint32_t sign_mask,
                             fa4_round col_rnd, uint64_t col_seed, fa4_qtensor col_out,
                             void *workspace, size_t workspace_bytes, void *stream);

/* The SwiGLU producer of a down projection, fused with its quantizer
 * ("Format-Aware Fusion...", section "The Design Philosophy of Format-Aware
 * Fusion": each quantization producer co-designed with its consumer; the
 * gated-MLP activation is the producer of the down projection's input).
 * z[T, 2F] is the bf16 gate+up output (row-major, leading dimension ld):
 * gate = z[:, 0:F], up = z[:, F:2F].  h = bf16(silu(gate) * up) with
 * silu(g) = g / (1 + exp(-g)) in binary32, rounded once to bf16, where exp is
 * computed step by step: x clamped to [-87, 88], n = rint(x * RN(log2 e)),
 * r = x - n ln2 by two fused multiply-adds (ln2 = 0.693145751953125 +
 * 1.42860677e-6), p = 1 + r(1 + r(1/2 + r(1/6 + r(1/24 + r(1/120 + r/720)))))
 * by fused multiply-adds with the binary32 coefficients, exp = p * 2^n.
 * h is quantized row-wise into row_out (Q = h [T, F]; row_fmt FA4_MXFP4,
 * FA4_MXFP4_NOCLIP or FA4_NVFP4_CTA, rounding row_rnd with row_seed) and,
 * when col != 0, column-wise into col_out (Q = h^T [F, T], MXFP4, with the
 * fixed-sign Hadamard when col_hadamard != 0, rounding col_rnd with
 * col_seed).  Bytes equal fa4_quantize / fa4_quantize_dual applied to h; h
 * itself is never written.  Requirements: F a multiple of 32, T >= 1 (a
 * multiple of 32 when col), ld >= 2F and a multiple of 8, pointers 16-byte
 * aligned.  Errors: INVALID_ARG, SHAPE, ALIGN, UNSUPPORTED (NVFP4-global:
 * its tensor amax would need h twice), CUDA.  No workspace. */
FA4_API fa4_status fa4_swiglu_quantize(const void *z, int64_t T, int64_t F, int64_t ld,
                                       fa4_format row_fmt, fa4_round row_rnd, uint64_t row_seed,
                                       fa4_qtensor row_out, int col, int col_hadamard,
                                       uint32_t sign_mask, fa4_round col_rnd, uint64_t col_seed,
                                       fa4_qtensor col_out, void *stream);

/* Block-scaled FP4 GEMM on the tcgen05 tensor cores:
 *   D[m][n] = alpha * sum_k A[m][k] * B[n][k]       (D = alpha A B^T)
 * with A[M, K] and B[N, K] quantized operands in the same format (both
 * K-major).  NVFP4_GLOBAL multiplies by the two tensor decode scales;
 * NVFP4_CTA multiplies every 128-wide K chunk by tsA[m/128][kc] *
 * tsB[n/128][kc].  FP32 accumulation.  D is row-major [M, N] with leading
 * dimension ldd elements (a multiple of 8, at least N), bf16 or fp32.  Any
 * M and N; K a multiple of 32 (the tiles past M, N or K compute on zero
 * payload and zero scales).  Workspace: at least
 * FA4_WS_HEADER_BYTES (the bounded-wait status word).
 * Errors: SHAPE, ALIGN, INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
FA4_API fa4_status fa4_gemm_blockscaled(fa4_qtensor A, fa4_qtensor B, int64_t M, int64_t N, int64_t K,
                                fa4_format fmt, float alpha, void *D, int64_t ldd,
                                fa4_out_dtype out_dtype, void *workspace, size_t workspace_bytes,
                                void *stream);

/* The same GEMM with the quantizer fused into its epilogue ("Format-Aware
 * Fusion...", section "The Design Philosophy of Format-Aware Fusion": the
 * producer of the next operand is the GEMM that computes it): the bf16
 * output D = alpha * A B^T is written (when D is not NULL) and its row-wise
 * MXFP4 operand (RNE) goes to Dq ([M, N/2] payload, scale bytes in the
 * padded atom layout of an [M, N] operand), byte-identical to
 * fa4_quantize(D, FA4_MXFP4, FA4_RNE, FA4_ROWWISE) of that bf16 D, without
 * reading D back.  N a multiple of 32.  fmt MXFP4 or NVFP4_GLOBAL
 * (FA4_ERR_UNSUPPORTED for NVFP4_CTA).  Other requirements and errors as
 * fa4_gemm_blockscaled. */
FA4_API fa4_status fa4_gemm_blockscaled_mxout(fa4_qtensor A, fa4_qtensor B, int64_t M, int64_t N,
                                      int64_t K, fa4_format fmt, float alpha, void *D, int64_t ldd,
                                      fa4_qtensor Dq, void *workspace, size_t workspace_bytes,
                                      void *stream);

/* Linear layer compositions for T tokens, Cin inputs, Cout outputs (the
 * configurations the pages' Llama-3-8B results train: "Format-Aware
 * Fusion...", section "Empirical Results").  bf16 activations row-major;
 * T, Cin and Cout multiples of 32 (each is the block dimension of some
 * operand).
 *
 * fa4_linear_fwd:   Y[T, Cout] (bf16) = X[T, Cin] W^T.  X is quantized
 *                   row-wise (RNE) in `fmt` into the workspace; Wq is W[Cout,
 *                   Cin] quantized row-wise in the same format.
 * fa4_linear_dgrad: dX[T, Cin] (bf16) = dY[T, Cout] W.  dY is quantized
 *                   row-wise with `rnd` (SR = row-gradient stochastic
 *                   rounding) into the workspace; Wq_col is W quantized
 *                   column-wise ([Cin, Cout] operand) in the same format.
 * fa4_linear_wgrad: dW[Cout, Cin] = dY^T X, MXFP4: dY and X are quantized
 *                   column-wise with the fixed-sign Hadamard (sign_mask) and
 *                   `rnd`, then multiplied with alpha = 1/32.
 * fa4_linear_ws_bytes gives the workspace each needs (kind 0 fwd, 1 dgrad,
 * 2 wgrad, 3 fwd_save, 4 bwd; below).  Errors: as the calls they are made of. */
FA4_API fa4_status fa4_linear_ws_bytes(int kind, int64_t T, int64_t Cin, int64_t Cout, fa4_format fmt,
                               size_t *workspace_bytes);
FA4_API fa4_status fa4_linear_fwd(const void *X, fa4_qtensor Wq, int64_t T, int64_t Cin, int64_t Cout,
                          fa4_format fmt, void *Y, void *workspace, size_t workspace_bytes,
                          void *stream);
FA4_API fa4_status fa4_linear_dgrad(const void *dY, fa4_qtensor Wq_col, int64_t T, int64_t Cin,
                            int64_t Cout, fa4_format fmt, fa4_round rnd, uint64_t seed, void *dX,
                            void *workspace, size_t workspace_bytes, void *stream);
FA4_API fa4_status fa4_linear_wgrad(const void *dY, const void *X, int64_t T, int64_t Cin, int64_t Cout,
                            uint32_t sign_mask, fa4_round rnd, uint64_t seed, void *dW,
                            fa4_out_dtype out_dtype, void *workspace, size_t workspace_bytes,
                            void *stream);

/* Training form of the linear layer, forward half: Y = X W^T as
 * fa4_linear_fwd (X row-wise in `fmt`, RNE), and from the same read of X its
 * column-wise MXFP4 operand with the fixed-sign Hadamard (RNE) into the
 * caller's Xcol ([Cin, T]: payload Cin*T/2 bytes, scales as fa4_quant_sizes), the
 * state the backward half needs instead of the bf16 X ("Format-Aware
 * Fusion...", section "The Design Philosophy of Format-Aware Fusion": the
 * state kept for the backward pass is the FP4 operand, not the bf16 X).  Y and Xcol equal fa4_linear_fwd and
 * fa4_hadamard32_quantize(X, sign_mask, FA4_RNE) byte for byte.
 * Workspace: fa4_linear_ws_bytes(kind 3).  Errors: as fa4_linear_fwd. */
FA4_API fa4_status fa4_linear_fwd_save(const void *X, fa4_qtensor Wq, int64_t T, int64_t Cin,
                               int64_t Cout, fa4_format fmt, uint32_t sign_mask, void *Y,
                               fa4_qtensor Xcol, void *workspace, size_t workspace_bytes,
                               void *stream);

/* Training form, backward half: one read of dY gives its row-wise operand
 * (`fmt`, rounding rnd with seed) and its column-wise MXFP4 Hadamard operand
 * (RNE); then dX = dY W (bf16, with Wq_col the column-wise W as in
 * fa4_linear_dgrad) and dW = dY^T X = (1/32) * GEMM(dY col, Xcol) (fp32 or
 * bf16 by dw_dtype) with Xcol from fa4_linear_fwd_save and the same
 * sign_mask.  dX equals fa4_linear_dgrad(dY, Wq_col, fmt, rnd, seed) and dW
 * equals fa4_linear_wgrad(dY, X, sign_mask, FA4_RNE, ...) byte for byte.
 * Workspace: fa4_linear_ws_bytes(kind 4).  Errors: as fa4_linear_dgrad. */
FA4_API fa4_status fa4_linear_bwd(const void *dY, fa4_qtensor Wq_col, fa4_qtensor Xcol, int64_t T,
                          int64_t Cin, int64_t Cout, fa4_format fmt, fa4_round rnd, uint64_t seed,
                          uint32_t sign_mask, void *dX, void *dW, fa4_out_dtype dw_dtype,
                          void *workspace, size_t workspace_bytes, void *stream);

/* NVFP4-global quantization that allocates nothing and takes no workspace.
 * (No counterpart on the pages: it exists for callers, not for the method.)
 * For callers that cannot provide device scratch: a runtime that reserves
 * all device memory up front under a fixed plan, or code that must not call
 * cudaMalloc at that point (it can synchronize the device, or the allocator
 * belongs to someone else).  Same result, bytes and error checks as
 * fa4_quantize(x, rows, cols, ld, FA4_NVFP4_GLOBAL, rnd, orient, seed, out,
 * ...); the amax pass keeps its per-CTA partial maxima in a fixed array of
 * 1184 floats (4736 bytes) inside the library, which every GPU that loads
 * the library holds until the process exits.  A call needing more partials
 * than that returns FA4_ERR_WORKSPACE (the launch configuration never does).
 * The first call on a device looks up that array's device address (once per
 * device ordinal, in the context current at that call); make that first
 * call before any stream capture.  The address is kept for the process: it
 * does not survive cudaDeviceReset, and it is only valid in the device's
 * primary context (the CUDA runtime's), so after a reset, or under a
 * driver-API context of the caller's own, this entry point must not be used
 * on that device.  A timed-out wait inside the quantize kernel has no status
 * word to report to here (it leaves the output incomplete); the kernel's
 * only wait is on its own tile loads.  Every call
 * shares the one array per device: calls that may run at the same time on
 * the GPU (different streams, no ordering between them) race on it and must
 * be serialized by the caller.  Errors: SHAPE, ALIGN, INVALID_ARG, WORKSPACE,
 * CUDA, UNSUPPORTED (device ordinal >= 64). */
FA4_API fa4_status fa4_quantize_nvfp4_global_noalloc(const void *x, int64_t rows, int64_t cols,
                                                     int64_t ld, fa4_round rnd, fa4_orient orient,
                                                     uint64_t seed, fa4_qtensor out, void *stream);

/* Zero the workspace header (stream-ordered memset of FA4_WS_HEADER_BYTES). */
FA4_API fa4_status fa4_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* Synchronize `stream`, read the sticky device status word of `workspace`
 * and clear it.  Returns FA4_OK, FA4_ERR_TIMEOUT (a bounded wait in a kernel
 * gave up; the kernel returned early and its output is incomplete) or
 * FA4_ERR_CUDA. */
FA4_API fa4_status fa4_check_device_status(void *workspace, void *stream);

/* Static description of a status code; never NULL. */
FA4_API const char *fa4_status_string(fa4_status s);

/* Library version as major*10000 + minor*100 + patch. */
FA4_API int fa4_version(void);

/* Diagnostics: run the device element conversions the quantizers use on n
 * fp32 inputs (device pointers).  rne_codes[i] = E2M1 RNE code of y[i];
 * sr_codes[i] = E2M1 SR code of y[i] with the 16 random bits u16[i] (may be
 * NULL to skip); e4m3_codes[i] = E4M3 RNE code of the clamped block scale
 * y[i] (may be NULL to skip).  sr_bits[i] (may be NULL) = the 16 Philox bits
 * of element index idx[i] under `seed`. */
FA4_API fa4_status fa4_debug_convert(const float *y, const uint32_t *u16, int64_t n, uint8_t *rne_codes,
                             uint8_t *sr_codes, uint8_t *e4m3_codes, void *stream);
FA4_API fa4_status fa4_debug_sr_bits(uint64_t seed, const uint64_t *idx, int64_t n, uint32_t *bits,
                             void *stream);

/* Diagnostics: the NVFP4 block-scale step of the quantizers, on n block
 * amaxes (device pointers, non-negative and finite) under one encode scale
 * s_enc ("FP4 Is No Longer Just a Hardware Feature...", section "NVFP4 is
 * more than a 4-bit value": E4M3 block scale under the FP32 tensor scale;
 * section "The third change": the clamp).  codes[i] = E4M3 code of
 * (amax[i] / 6) * s_enc clamped to [2^-9, 448]; mults[i] = the element
 * multiplier s_enc / decode(codes[i]) the quantizers apply.  Computed by
 * the same device code as fa4_quantize (an exactly rounded division by 6 and
 * a table of multipliers).  Errors: INVALID_ARG, CUDA. */
FA4_API fa4_status fa4_debug_nv_block_scale(const float *amax, float s_enc, int64_t n, uint8_t *codes,
                                            float *mults, void *stream);

/* Diagnostics: silu(g) = g / (1 + exp(-g)) in binary32 exactly as
 * fa4_swiglu_quantize computes it (the exp defined step by step, the
 * correctly rounded quotient), for n bf16 gate values g (device pointer, bf16
 * bits, finite) into out[n] (device, binary32).  The gated-MLP activation is
 * the producer of the down projection's input ("Format-Aware Fusion: The
 * Engineering Practice That Doubles FP4 Pretraining Throughput", section
 * "The Design Philosophy of Format-Aware Fusion").  Errors: INVALID_ARG,
 * CUDA. */
FA4_API fa4_status fa4_debug_silu(const void *g, int64_t n, float *out, void *stream);

/* Diagnostics for the bounded waits: fa4_gemm_blockscaled (fp32 output,
 * alpha 1) with every wait limited to timeout_ns (0 < timeout_ns <= 2 s)
 * and, when skip_k_tile >= 0, a producer that never loads the skip_k_tile-th
 * k-tile it owns, so the consumer's wait must run out.  The kernel then sets
 * the workspace status word, waits for its own copies in flight, releases
 * its tensor memory and returns; fa4_check_device_status reports
 * FA4_ERR_TIMEOUT and the context stays usable. */
FA4_API fa4_status fa4_debug_gemm_timeout(fa4_qtensor A, fa4_qtensor B, int64_t M, int64_t N, int64_t K,
                                  fa4_format fmt, void *D, int64_t ldd, int skip_k_tile,
                                  uint64_t timeout_ns, void *workspace, size_t workspace_bytes,
                                  void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FA4_H */
