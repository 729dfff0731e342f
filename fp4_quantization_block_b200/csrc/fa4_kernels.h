// fa4_kernels.h -- internal launch interface between the C ABI (fa4_api.cu)
// and the kernels.  Not installed; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa4 {

// Upper bound on the per-CTA partial maxima of the NVFP4-global amax pass.
constexpr int kMaxAmaxPartials = 1184;  // 8 CTAs x 148 SMs

int amax_partials_count(int64_t rows, int64_t cols);
cudaError_t launch_tensor_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                               float *partials, int n_partials, cudaStream_t st);
// One quantize launch: x[T, C] (bf16, leading dimension ld) to the row-wise
// operand (Q = x), the column-wise operand (Q = x^T), or both.  A format of
// -1 skips that orientation.  When both are produced the column-wise operand
// is MXFP4 (optionally through the fixed-sign Hadamard).
struct QuantArgs {
  const uint16_t *x;
  int64_t T, C, ld;
  int row_fmt = -1, row_rnd = 0;
  uint8_t *row_payload = nullptr, *row_scales = nullptr;
  float *row_ts = nullptr;
  uint64_t row_seed = 0;
  int col_fmt = -1, col_rnd = 0;
  bool hadamard = false;
  uint32_t sign_mask = 0;
  uint8_t *col_payload = nullptr, *col_scales = nullptr;
  float *col_ts = nullptr;
  uint64_t col_seed = 0;
  const float *partials = nullptr;  // NVFP4-global amax partials (either orientation)
  int n_partials = 0;
  uint32_t *status = nullptr;  // bounded-wait status word (may be null)
  uint64_t timeout_ns = 2000000000ull;
};
cudaError_t launch_quantize(const QuantArgs &a, cudaStream_t st);
// The SwiGLU producer fused with its quantizer: z[T, 2F] (gate | up, row
// stride ld) -> h = bf16(silu(gate) * up) quantized row-wise (row_fmt MXFP4,
// MXFP4 without clipping or CTA-local NVFP4) and, with col, column-wise MXFP4
// (hadamard: with the fixed-sign Hadamard).
struct SwigluArgs {
  const uint16_t *z;
  int64_t T, F, ld;
  int row_fmt, row_rnd;
  uint8_t *row_payload, *row_scales;
  float *row_ts;
  uint64_t row_seed;
  bool col, hadamard;
  uint32_t sign_mask;
  int col_rnd;
  uint8_t *col_payload, *col_scales;
  uint64_t col_seed;
};
cudaError_t launch_swiglu_quantize(const SwigluArgs &a, cudaStream_t st);
// Tensor map of a bf16 matrix [rows, cols] (row stride ld elements) in
// 128 x 128 boxes, no swizzle, zero fill past the edges.
bool make_bf16_tile_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld);
cudaError_t launch_debug_convert(const float *y, const uint32_t *u16, int64_t n, uint8_t *rne,
                                 uint8_t *sr, uint8_t *e4m3, cudaStream_t st);
cudaError_t launch_debug_nv_block_scale(const float *amax, float s_enc, int64_t n, uint8_t *codes,
                                        float *mults, cudaStream_t st);
cudaError_t launch_debug_silu(const uint16_t *g, int64_t n, float *out, cudaStream_t st);
cudaError_t launch_debug_sr_bits(uint64_t seed, const uint64_t *idx, int64_t n, uint32_t *bits,
                                 cudaStream_t st);

// Block-scaled GEMM.  status: device word for bounded-wait timeouts.
struct GemmArgs {
  const uint8_t *a_payload, *a_scales;
  const float *a_ts;
  const uint8_t *b_payload, *b_scales;
  const float *b_ts;
  int64_t M, N, K;
  int fmt;
  float alpha;
  void *D;
  int64_t ldd;
  int out_fp32;
  uint32_t *status;
  int debug_skip_stage;     // < 0 normally; >= 0: the producer never loads that k-tile (test hook)
  uint64_t timeout_ns;      // bounded-wait limit
  // optional: the bf16 output's row-wise MXFP4 operand written by the
  // epilogue (payload [M, N/2], scales in the atom layout); null: none.
  // D may then be null (the bf16 output is not stored).
  uint8_t *q_payload = nullptr, *q_scales = nullptr;
};
cudaError_t launch_gemm_blockscaled(const GemmArgs &a, cudaStream_t st);

}  // namespace fa4
