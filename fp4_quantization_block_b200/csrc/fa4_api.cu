// fa4_api.cu -- the C ABI declared in include/fa4.h: argument checks on the
// host, workspace carving, and kernel launches.  No device memory is
// allocated here and nothing synchronizes except fa4_check_device_status.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "../../include/fa4.h"
#include "fa4_kernels.h"

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait
constexpr size_t kHdr = FA4_WS_HEADER_BYTES;

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline bool fmt_ok(int f) {
  return f == FA4_MXFP4 || f == FA4_NVFP4_GLOBAL || f == FA4_NVFP4_CTA || f == FA4_MXFP4_NOCLIP;
}
inline bool is_mx(int f) { return f == FA4_MXFP4 || f == FA4_MXFP4_NOCLIP; }
inline int block_of(int f) { return is_mx(f) ? 32 : 16; }
inline cudaStream_t S(void *s) { return reinterpret_cast<cudaStream_t>(s); }

size_t partials_bytes() { return align256(sizeof(float) * fa4::kMaxAmaxPartials); }

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t qt_payload(int64_t R, int64_t K) { return (size_t)(R * (K / 2)); }
// scale atoms: rows padded to a multiple of 128, blocks to a multiple of 4
size_t qt_scales(int64_t R, int64_t K, int fmt) {
  return (size_t)(ceil_div(R, 128) * 128 * (ceil_div(K / block_of(fmt), 4) * 4));
}
size_t qt_ts(int64_t R, int64_t K, int fmt) {
  if (fmt == FA4_NVFP4_GLOBAL) return 1;
  if (fmt == FA4_NVFP4_CTA) return (size_t)(ceil_div(R, 128) * ceil_div(K, 128));
  return 0;
}
// Shape rule of a quantized operand Q[R, K] read from x[rows, cols]: any
// positive R; K a multiple of 32 (whole MX blocks, and payload rows of a
// multiple of 16 bytes for the GEMM's tensor-memory-access loads); x rows
// read in 16-byte pieces, so cols is a multiple of 8.
bool quant_shape_ok(int64_t rows, int64_t cols, int orient) {
  if (rows <= 0 || cols <= 0 || cols % 8) return false;
  const int64_t K = orient == FA4_ROWWISE ? cols : rows;
  return K % 32 == 0;
}
size_t quant_ws(int fmt) { return kHdr + (fmt == FA4_NVFP4_GLOBAL ? partials_bytes() : 0); }
// bytes of a quantized operand carved from a workspace (256-aligned parts)
size_t qt_ws_bytes(int64_t R, int64_t K, int fmt) {
  return align256(qt_payload(R, K)) + align256(qt_scales(R, K, fmt)) +
         align256(sizeof(float) * (qt_ts(R, K, fmt) ? qt_ts(R, K, fmt) : 1));
}
fa4_qtensor carve_qt(uint8_t *base, int64_t R, int64_t K, int fmt) {
  fa4_qtensor q;
  q.payload = base;
  base += align256(qt_payload(R, K));
  q.scales = base;
  base += align256(qt_scales(R, K, fmt));
  q.tensor_scale = reinterpret_cast<float *>(base);
  return q;
}

// x[rows, cols] read for the given orientations (row-wise, column-wise or
// both)
fa4_status check_input(const void *x, int64_t rows, int64_t cols, int64_t ld, bool row = true,
                       bool col = false) {
  if (!x) return FA4_ERR_INVALID_ARG;
  if ((row && !quant_shape_ok(rows, cols, FA4_ROWWISE)) ||
      (col && !quant_shape_ok(rows, cols, FA4_COLWISE)))
    return FA4_ERR_SHAPE;
  if (ld < cols || ld % 8) return FA4_ERR_SHAPE;
  if (!aligned16(x)) return FA4_ERR_ALIGN;
  return FA4_OK;
}

fa4_status check_qt(const fa4_qtensor &q, int fmt) {
  if (!q.payload || !q.scales) return FA4_ERR_INVALID_ARG;
  if (!is_mx(fmt) && !q.tensor_scale) return FA4_ERR_INVALID_ARG;
  if (!aligned16(q.payload) || !aligned16(q.scales)) return FA4_ERR_ALIGN;
  if (q.tensor_scale && !aligned4(q.tensor_scale)) return FA4_ERR_ALIGN;
  return FA4_OK;
}

fa4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FA4_OK : FA4_ERR_CUDA; }

// Quantize into `out` using the header + partials at `ws` (already checked).
fa4_status do_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld, int fmt, int rnd,
                       int orient, bool hadamard, uint32_t sign_mask, uint64_t seed,
                       const fa4_qtensor &out, uint8_t *ws, cudaStream_t st) {
  fa4::QuantArgs q;
  q.x = static_cast<const uint16_t *>(x);
  q.T = rows;
  q.C = cols;
  q.ld = ld;
  q.status = reinterpret_cast<uint32_t *>(ws);
  q.timeout_ns = kDefaultTimeoutNs;
  if (fmt == FA4_NVFP4_GLOBAL) {
    q.partials = reinterpret_cast<float *>(ws + kHdr);
    q.n_partials = fa4::amax_partials_count(rows, cols);
    cudaError_t e = fa4::launch_tensor_amax(q.x, rows, cols, ld, reinterpret_cast<float *>(ws + kHdr),
                                            q.n_partials, st);
    if (e != cudaSuccess) return FA4_ERR_CUDA;
  }
  if (orient == FA4_ROWWISE) {
    q.row_fmt = fmt;
    q.row_rnd = rnd;
    q.row_payload = static_cast<uint8_t *>(out.payload);
    q.row_scales = static_cast<uint8_t *>(out.scales);
    q.row_ts = out.tensor_scale;
    q.row_seed = seed;
  } else {
    q.col_fmt = fmt;
    q.col_rnd = rnd;
    q.hadamard = hadamard;
    q.sign_mask = sign_mask;
    q.col_payload = static_cast<uint8_t *>(out.payload);
    q.col_scales = static_cast<uint8_t *>(out.scales);
    q.col_ts = out.tensor_scale;
    q.col_seed = seed;
  }
  return cuda_status(fa4::launch_quantize(q, st));
}

// Both orientations from one read of x (the row-wise NVFP4-global amax pass
// first, when needed).
fa4_status do_quantize_dual(const void *x, int64_t rows, int64_t cols, int64_t ld, int row_fmt,
                            int row_rnd, uint64_t row_seed, const fa4_qtensor &row_out,
                            bool hadamard, uint32_t sign_mask, int col_rnd, uint64_t col_seed,
                            const fa4_qtensor &col_out, uint8_t *ws, cudaStream_t st) {
  fa4::QuantArgs q;
  q.x = static_cast<const uint16_t *>(x);
  q.T = rows;
  q.C = cols;
  q.ld = ld;
  q.status = reinterpret_cast<uint32_t *>(ws);
  q.timeout_ns = kDefaultTimeoutNs;
  if (row_fmt == FA4_NVFP4_GLOBAL) {
    q.partials = reinterpret_cast<float *>(ws + kHdr);
    q.n_partials = fa4::amax_partials_count(rows, cols);
    cudaError_t e = fa4::launch_tensor_amax(q.x, rows, cols, ld, reinterpret_cast<float *>(ws + kHdr),
                                            q.n_partials, st);
    if (e != cudaSuccess) return FA4_ERR_CUDA;
  }
  q.row_fmt = row_fmt;
  q.row_rnd = row_rnd;
  q.row_payload = static_cast<uint8_t *>(row_out.payload);
  q.row_scales = static_cast<uint8_t *>(row_out.scales);
  q.row_ts = row_out.tensor_scale;
  q.row_seed = row_seed;
  q.col_fmt = FA4_MXFP4;
  q.col_rnd = col_rnd;
  q.hadamard = hadamard;
  q.sign_mask = sign_mask;
  q.col_payload = static_cast<uint8_t *>(col_out.payload);
  q.col_scales = static_cast<uint8_t *>(col_out.scales);
  q.col_ts = nullptr;
  q.col_seed = col_seed;
  return cuda_status(fa4::launch_quantize(q, st));
}

fa4_status do_gemm(const fa4_qtensor &A, const fa4_qtensor &B, int64_t M, int64_t N, int64_t K,
                   int fmt, float alpha, void *D, int64_t ldd, int out_dtype, uint8_t *ws,
                   cudaStream_t st, int skip, uint64_t timeout_ns,
                   const fa4_qtensor *dq = nullptr) {
  fa4::GemmArgs a;
  a.a_payload = static_cast<const uint8_t *>(A.payload);
  a.a_scales = static_cast<const uint8_t *>(A.scales);
  a.a_ts = A.tensor_scale;
  a.b_payload = static_cast<const uint8_t *>(B.payload);
  a.b_scales = static_cast<const uint8_t *>(B.scales);
  a.b_ts = B.tensor_scale;
  a.M = M;
  a.N = N;
  a.K = K;
  a.fmt = fmt == FA4_MXFP4_NOCLIP ? FA4_MXFP4 : fmt;  // same layout and scale type
  a.alpha = alpha;
  a.D = D;
  a.ldd = ldd;
  a.out_fp32 = out_dtype == FA4_OUT_FP32;
  a.status = reinterpret_cast<uint32_t *>(ws);
  a.debug_skip_stage = skip;
  a.timeout_ns = timeout_ns;
  if (dq) {
    a.q_payload = static_cast<uint8_t *>(dq->payload);
    a.q_scales = static_cast<uint8_t *>(dq->scales);
  }
  return cuda_status(fa4::launch_gemm_blockscaled(a, st));
}

fa4_status check_gemm(const fa4_qtensor &A, const fa4_qtensor &B, int64_t M, int64_t N, int64_t K,
                      int fmt, const void *D, int64_t ldd, int out_dtype, const void *ws,
                      size_t ws_bytes) {
  if (!fmt_ok(fmt)) return FA4_ERR_INVALID_ARG;
  if (out_dtype != FA4_OUT_BF16 && out_dtype != FA4_OUT_FP32) return FA4_ERR_INVALID_ARG;
  if (!D) return FA4_ERR_INVALID_ARG;
  fa4_status s = check_qt(A, fmt);
  if (s != FA4_OK) return s;
  if ((s = check_qt(B, fmt)) != FA4_OK) return s;
  if (M <= 0 || N <= 0 || K <= 0 || K % 32) return FA4_ERR_SHAPE;
  if (ldd < N || ldd % 8) return FA4_ERR_SHAPE;
  if (!aligned16(D)) return FA4_ERR_ALIGN;
  if (!ws || ws_bytes < kHdr) return FA4_ERR_WORKSPACE;
  if (!aligned16(ws)) return FA4_ERR_ALIGN;
  return FA4_OK;
}

}  // namespace

extern "C" {

int fa4_version(void) { return 100; }

const char *fa4_status_string(fa4_status s) {
  switch (s) {
    case FA4_OK: return "ok";
    case FA4_ERR_INVALID_ARG: return "invalid argument";
    case FA4_ERR_SHAPE: return "unsupported shape or leading dimension";
    case FA4_ERR_ALIGN: return "pointer not 16-byte aligned";
    case FA4_ERR_UNSUPPORTED: return "unsupported combination";
    case FA4_ERR_WORKSPACE: return "workspace missing or too small";
    case FA4_ERR_CUDA: return "CUDA error";
    case FA4_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

fa4_status fa4_quant_sizes(int64_t rows, int64_t cols, fa4_format fmt, fa4_orient orient,
                           size_t *payload_bytes, size_t *scale_bytes, size_t *tscale_count,
                           size_t *workspace_bytes) {
  if (!fmt_ok(fmt) || (orient != FA4_ROWWISE && orient != FA4_COLWISE)) return FA4_ERR_INVALID_ARG;
  if (!quant_shape_ok(rows, cols, orient)) return FA4_ERR_SHAPE;
  const int64_t R = orient == FA4_ROWWISE ? rows : cols, K = orient == FA4_ROWWISE ? cols : rows;
  if (payload_bytes) *payload_bytes = qt_payload(R, K);
  if (scale_bytes) *scale_bytes = qt_scales(R, K, fmt);
  if (tscale_count) *tscale_count = qt_ts(R, K, fmt);
  if (workspace_bytes) *workspace_bytes = quant_ws(fmt);
  return FA4_OK;
}

fa4_status fa4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld, fa4_format fmt,
                        fa4_round rnd, fa4_orient orient, uint64_t seed, fa4_qtensor out,
                        void *workspace, size_t workspace_bytes, void *stream) {
  if (!fmt_ok(fmt) || (rnd != FA4_RNE && rnd != FA4_SR) ||
      (orient != FA4_ROWWISE && orient != FA4_COLWISE))
    return FA4_ERR_INVALID_ARG;
  fa4_status s = check_input(x, rows, cols, ld, orient == FA4_ROWWISE, orient == FA4_COLWISE);
  if (s != FA4_OK) return s;
  if ((s = check_qt(out, fmt)) != FA4_OK) return s;
  if (!workspace || workspace_bytes < quant_ws(fmt)) return FA4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA4_ERR_ALIGN;
  return do_quantize(x, rows, cols, ld, fmt, rnd, orient, false, 0u, seed, out,
                     static_cast<uint8_t *>(workspace), S(stream));
}

fa4_status fa4_hadamard32_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld,
                                   uint32_t sign_mask, fa4_round rnd, uint64_t seed,
                                   fa4_qtensor out, void *workspace, size_t workspace_bytes,
                                   void *stream) {
  if (rnd != FA4_RNE && rnd != FA4_SR) return FA4_ERR_INVALID_ARG;
  fa4_status s = check_input(x, rows, cols, ld, false, true);
  if (s != FA4_OK) return s;
  if ((s = check_qt(out, FA4_MXFP4)) != FA4_OK) return s;
  if (!workspace || workspace_bytes < quant_ws(FA4_MXFP4)) return FA4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA4_ERR_ALIGN;
  return do_quantize(x, rows, cols, ld, FA4_MXFP4, rnd, FA4_COLWISE, true, sign_mask, seed, out,
                     static_cast<uint8_t *>(workspace), S(stream));
}

fa4_status fa4_quantize_dual(const void *x, int64_t rows, int64_t cols, int64_t ld,
                             fa4_format row_fmt, fa4_round row_rnd, uint64_t row_seed,
                             fa4_qtensor row_out, int col_hadamard, uint32_t sign_mask,
                             fa4_round col_rnd, uint64_t col_seed, fa4_qtensor col_out,
                             void *workspace, size_t workspace_bytes, void *stream) {
  if (!fmt_ok(row_fmt) || (row_rnd != FA4_RNE && row_rnd != FA4_SR) ||
      (col_rnd != FA4_RNE && col_rnd != FA4_SR))
    return FA4_ERR_INVALID_ARG;
  fa4_status s = check_input(x, rows, cols, ld, true, true);
  if (s != FA4_OK) return s;
  if ((s = check_qt(row_out, row_fmt)) != FA4_OK) return s;
  if ((s = check_qt(col_out, FA4_MXFP4)) != FA4_OK) return s;
  if (!workspace || workspace_bytes < quant_ws(row_fmt)) return FA4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA4_ERR_ALIGN;
  return do_quantize_dual(x, rows, cols, ld, row_fmt, row_rnd, row_seed, row_out, col_hadamard != 0,
                          sign_mask, col_rnd, col_seed, col_out, static_cast<uint8_t *>(workspace),
                          S(stream));
}

fa4_status fa4_swiglu_quantize(const void *z, int64_t T, int64_t F, int64_t ld, fa4_format row_fmt,
                               fa4_round row_rnd, uint64_t row_seed, fa4_qtensor row_out, int col,
                               int col_hadamard, uint32_t sign_mask, fa4_round col_rnd,
                               uint64_t col_seed, fa4_qtensor col_out, void *stream) {
  if (!z || !fmt_ok(row_fmt) || (row_rnd != FA4_RNE && row_rnd != FA4_SR) ||
      (col && col_rnd != FA4_RNE && col_rnd != FA4_SR))
    return FA4_ERR_INVALID_ARG;
  if (row_fmt == FA4_NVFP4_GLOBAL) return FA4_ERR_UNSUPPORTED;
  if (T <= 0 || F <= 0 || F % 32 || (col && T % 32) || ld < 2 * F || ld % 8) return FA4_ERR_SHAPE;
  if (!aligned16(z)) return FA4_ERR_ALIGN;
  fa4_status s = check_qt(row_out, row_fmt);
  if (s != FA4_OK) return s;
  if (col && (s = check_qt(col_out, FA4_MXFP4)) != FA4_OK) return s;
  fa4::SwigluArgs a;
  a.z = static_cast<const uint16_t *>(z);
  a.T = T;
  a.F = F;
  a.ld = ld;
  a.row_fmt = row_fmt;
  a.row_rnd = row_rnd;
  a.row_payload = static_cast<uint8_t *>(row_out.payload);
  a.row_scales = static_cast<uint8_t *>(row_out.scales);
  a.row_ts = row_out.tensor_scale;
  a.row_seed = row_seed;
  a.col = col != 0;
  a.hadamard = col_hadamard != 0;
  a.sign_mask = sign_mask;
  a.col_rnd = col_rnd;
  a.col_payload = col ? static_cast<uint8_t *>(col_out.payload) : nullptr;
  a.col_scales = col ? static_cast<uint8_t *>(col_out.scales) : nullptr;
  a.col_seed = col_seed;
  return cuda_status(fa4::launch_swiglu_quantize(a, S(stream)));
}

fa4_status fa4_gemm_blockscaled(fa4_qtensor A, fa4_qtensor B, int64_t M, int64_t N, int64_t K,
                                fa4_format fmt, float alpha, void *D, int64_t ldd,
                                fa4_out_dtype out_dtype, void *workspace, size_t workspace_bytes,
                                void *stream) {
  fa4_status s = check_gemm(A, B, M, N, K, fmt, D, ldd, out_dtype, workspace, workspace_bytes);
  if (s != FA4_OK) return s;
  return do_gemm(A, B, M, N, K, fmt, alpha, D, ldd, out_dtype, static_cast<uint8_t *>(workspace),
                 S(stream), -1, kDefaultTimeoutNs);
}

fa4_status fa4_linear_ws_bytes(int kind, int64_t T, int64_t Cin, int64_t Cout, fa4_format fmt,
                               size_t *workspace_bytes) {
  if (!workspace_bytes || !fmt_ok(fmt)) return FA4_ERR_INVALID_ARG;
  if (T <= 0 || Cin <= 0 || Cout <= 0 || T % 32 || Cin % 32 || Cout % 32) return FA4_ERR_SHAPE;
  size_t b = kHdr + partials_bytes();
  switch (kind) {
    case 0: b += qt_ws_bytes(T, Cin, fmt); break;
    case 1: b += qt_ws_bytes(T, Cout, fmt); break;
    case 2: b += qt_ws_bytes(Cout, T, FA4_MXFP4) + qt_ws_bytes(Cin, T, FA4_MXFP4); break;
    case 3: b += qt_ws_bytes(T, Cin, fmt); break;
    case 4: b += qt_ws_bytes(T, Cout, fmt) + qt_ws_bytes(Cout, T, FA4_MXFP4); break;
    default: return FA4_ERR_INVALID_ARG;
  }
  *workspace_bytes = b;
  return FA4_OK;
}

fa4_status fa4_linear_fwd(const void *X, fa4_qtensor Wq, int64_t T, int64_t Cin, int64_t Cout,
                          fa4_format fmt, void *Y, void *workspace, size_t workspace_bytes,
                          void *stream) {
  size_t need;
  fa4_status s = fa4_linear_ws_bytes(0, T, Cin, Cout, fmt, &need);
  if (s != FA4_OK) return s;
  if ((s = check_input(X, T, Cin, Cin)) != FA4_OK) return s;
  if (!workspace || workspace_bytes < need) return FA4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA4_ERR_ALIGN;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  fa4_qtensor xq = carve_qt(ws + kHdr + partials_bytes(), T, Cin, fmt);
  if ((s = check_gemm(xq, Wq, T, Cout, Cin, fmt, Y, Cout, FA4_OUT_BF16, ws, workspace_bytes)) != FA4_OK)
    return s;
  if ((s = do_quantize(X, T, Cin, Cin, fmt, FA4_RNE, FA4_ROWWISE, false, 0u, 0u, xq, ws, S(stream))) != FA4_OK)
    return s;
  return do_gemm(xq, Wq, T, Cout, Cin, fmt, 1.0f, Y, Cout, FA4_OUT_BF16, ws, S(stream), -1,
                 kDefaultTimeoutNs);
}

fa4_status fa4_linear_dgrad(const void *dY, fa4_qtensor Wq_col, int64_t T, int64_t Cin,
                            int64_t Cout, fa4_format fmt, fa4_round rnd, uint64_t seed, void *dX,
                            void *workspace, size_t workspace_bytes, void *stream) {
  if (rnd != FA4_RNE && rnd != FA4_SR) return FA4_ERR_INVALID_ARG;
  size_t need;
  fa4_status s = fa4_linear_ws_bytes(1, T, Cin, Cout, fmt, &need);
  if (s != FA4_OK) return s;
  if ((s = check_input(dY, T, Cout, Cout)) != FA4_OK) return s;
  if (!workspace || workspace_bytes < need) return FA4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA4_ERR_ALIGN;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  fa4_qtensor gq = carve_qt(ws + kHdr + partials_bytes(), T, Cout, fmt);
  if ((s = check_gemm(gq, Wq_col, T, Cin, Cout, fmt, dX, Cin, FA4_OUT_BF16, ws, workspace_bytes)) != FA4_OK)
    return s;
  if ((s = do_quantize(dY, T, Cout, Cout, fmt, rnd, FA4_ROWWISE, false, 0u, seed, gq, ws, S(stream))) != FA4_OK)
    return s;
  return do_gemm(gq, Wq_col, T, Cin, Cout, fmt, 1.0f, dX, Cin, FA4_OUT_BF16, ws, S(stream), -1,
                 kDefaultTimeoutNs);
}

fa4_status fa4_linear_wgrad(const void *dY, const void *X, int64_t T, int64_t Cin, int64_t Cout,
                            uint32_t sign_mask, fa4_round rnd, uint64_t seed, void *dW,
                            fa4_out_dtype out_dtype, void *workspace, size_t workspace_bytes,
                            void *stream) {
  if (rnd != FA4_RNE && rnd != FA4_SR) return FA4_ERR_INVALID_ARG;
  size_t need;
  fa4_status s = fa4_linear_ws_bytes(2, T, Cin, Cout, FA4_MXFP4, &need);
  if (s != FA4_OK) return s;
  if ((s = check_input(dY, T, Cout, Cout, false, true)) != FA4_OK) return s;
  if ((s = check_input(X, T, Cin, Cin, false, true)) != FA4_OK) return s;
  if (!workspace || workspace_bytes < need) return FA4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA4_ERR_ALIGN;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint8_t *base = ws + kHdr + partials_bytes();
  fa4_qtensor gq = carve_qt(base, Cout, T, FA4_MXFP4);
  fa4_qtensor xq = carve_qt(base + qt_ws_bytes(Cout, T, FA4_MXFP4), Cin, T, FA4_MXFP4);
  if ((s = check_gemm(gq, xq, Cout, Cin, T, FA4_MXFP4, dW, Cin, out_dtype, ws, workspace_bytes)) != FA4_OK)
    return s;
  if ((s = do_quantize(dY, T, Cout, Cout, FA4_MXFP4, rnd, FA4_COLWISE, true, sign_mask, seed, gq, ws,
                       S(stream))) != FA4_OK)
    return s;
  if ((s = do_quantize(X, T, Cin, Cin, FA4_MXFP4, rnd, FA4_COLWISE, true, sign_mask, seed + 1, xq, ws,
                       S(stream))) != FA4_OK)
    return s;
  return do_gemm(gq, xq, Cout, Cin, T, FA4_MXFP4, 1.0f / 32.0f, dW, Cin, out_dtype, ws, S(stream),
                 -1, kDefaultTimeoutNs);
}

fa4_status fa4_linear_fwd_save(const void *X, fa4_qtensor Wq, int64_t T, int64_t Cin, int64_t Cout,
                               fa4_format fmt, uint32_t sign_mask, void *Y, fa4_qtensor Xcol,
                               void *workspace, size_t workspace_bytes, void *stream) {
  size_t need;
  fa4_status s = fa4_linear_ws_bytes(3, T, Cin, Cout, fmt, &need);
  if (s != FA4_OK) return s;
  if ((s = check_input(X, T, Cin, Cin, true, true)) != FA4_OK) return s;
  if ((s = check_qt(Xcol, FA4_MXFP4)) != FA4_OK) return s;
  if (!workspace || workspace_bytes < need) return FA4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA4_ERR_ALIGN;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  fa4_qtensor xq = carve_qt(ws + kHdr + partials_bytes(), T, Cin, fmt);
  if ((s = check_gemm(xq, Wq, T, Cout, Cin, fmt, Y, Cout, FA4_OUT_BF16, ws, workspace_bytes)) != FA4_OK)
    return s;
  if ((s = do_quantize_dual(X, T, Cin, Cin, fmt, FA4_RNE, 0u, xq, true, sign_mask, FA4_RNE, 0u, Xcol,
                            ws, S(stream))) != FA4_OK)
    return s;
  return do_gemm(xq, Wq, T, Cout, Cin, fmt, 1.0f, Y, Cout, FA4_OUT_BF16, ws, S(stream), -1,
                 kDefaultTimeoutNs);
}

fa4_status fa4_linear_bwd(const void *dY, fa4_qtensor Wq_col, fa4_qtensor Xcol, int64_t T,
                          int64_t Cin, int64_t Cout, fa4_format fmt, fa4_round rnd, uint64_t seed,
                          uint32_t sign_mask, void *dX, void *dW, fa4_out_dtype dw_dtype,
                          void *workspace, size_t workspace_bytes, void *stream) {
  if (rnd != FA4_RNE && rnd != FA4_SR) return FA4_ERR_INVALID_ARG;
  size_t need;
  fa4_status s = fa4_linear_ws_bytes(4, T, Cin, Cout, fmt, &need);
  if (s != FA4_OK) return s;
  if ((s = check_input(dY, T, Cout, Cout, true, true)) != FA4_OK) return s;
  if (!workspace || workspace_bytes < need) return FA4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA4_ERR_ALIGN;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint8_t *base = ws + kHdr + partials_bytes();
  fa4_qtensor gq = carve_qt(base, T, Cout, fmt);
  fa4_qtensor gc = carve_qt(base + qt_ws_bytes(T, Cout, fmt), Cout, T, FA4_MXFP4);
  if ((s = check_gemm(gq, Wq_col, T, Cin, Cout, fmt, dX, Cin, FA4_OUT_BF16, ws, workspace_bytes)) != FA4_OK)
    return s;
  if ((s = check_gemm(gc, Xcol, Cout, Cin, T, FA4_MXFP4, dW, Cin, dw_dtype, ws, workspace_bytes)) != FA4_OK)
    return s;
  if ((s = do_quantize_dual(dY, T, Cout, Cout, fmt, rnd, seed, gq, true, sign_mask, FA4_RNE, 0u, gc,
                            ws, S(stream))) != FA4_OK)
    return s;
  if ((s = do_gemm(gq, Wq_col, T, Cin, Cout, fmt, 1.0f, dX, Cin, FA4_OUT_BF16, ws, S(stream), -1,
                   kDefaultTimeoutNs)) != FA4_OK)
    return s;
  return do_gemm(gc, Xcol, Cout, Cin, T, FA4_MXFP4, 1.0f / 32.0f, dW, Cin, dw_dtype, ws, S(stream),
                 -1, kDefaultTimeoutNs);
}

fa4_status fa4_gemm_blockscaled_mxout(fa4_qtensor A, fa4_qtensor B, int64_t M, int64_t N,
                                      int64_t K, fa4_format fmt, float alpha, void *D, int64_t ldd,
                                      fa4_qtensor Dq, void *workspace, size_t workspace_bytes,
                                      void *stream) {
  if (!fmt_ok(fmt)) return FA4_ERR_INVALID_ARG;
  if (fmt == FA4_NVFP4_CTA) return FA4_ERR_UNSUPPORTED;
  if (N % 32) return FA4_ERR_SHAPE;  // D's MXFP4 blocks run along N
  fa4_status s = check_qt(Dq, FA4_MXFP4);
  if (s != FA4_OK) return s;
  // D is optional: checked as a bf16 output when given
  static const uint8_t dummy[16] __attribute__((aligned(16))) = {};
  const void *dcheck = D ? D : static_cast<const void *>(dummy);
  if ((s = check_gemm(A, B, M, N, K, fmt, dcheck, D ? ldd : N, FA4_OUT_BF16, workspace,
                      workspace_bytes)) != FA4_OK)
    return s;
  return do_gemm(A, B, M, N, K, fmt, alpha, D, D ? ldd : N, FA4_OUT_BF16,
                 static_cast<uint8_t *>(workspace), S(stream), -1, kDefaultTimeoutNs, &Dq);
}

fa4_status fa4_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
  if (!workspace || workspace_bytes < kHdr) return FA4_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(workspace, 0, kHdr, S(stream)));
}

fa4_status fa4_check_device_status(void *workspace, void *stream) {
  if (!workspace) return FA4_ERR_WORKSPACE;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return FA4_ERR_CUDA;
  uint32_t hdr[2] = {0, 0};
  if (cudaMemcpy(hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FA4_ERR_CUDA;
  if (hdr[0] == 0) return FA4_OK;
  if (cudaMemset(workspace, 0, sizeof(hdr)) != cudaSuccess) return FA4_ERR_CUDA;
  return hdr[0] == 7u ? FA4_ERR_TIMEOUT : FA4_ERR_CUDA;
}

fa4_status fa4_debug_convert(const float *y, const uint32_t *u16, int64_t n, uint8_t *rne_codes,
                             uint8_t *sr_codes, uint8_t *e4m3_codes, void *stream) {
  if (n < 0 || (n > 0 && (!y || !rne_codes))) return FA4_ERR_INVALID_ARG;
  if (sr_codes && !u16) return FA4_ERR_INVALID_ARG;
  return cuda_status(fa4::launch_debug_convert(y, u16, n, rne_codes, sr_codes, e4m3_codes, S(stream)));
}

fa4_status fa4_debug_nv_block_scale(const float *amax, float s_enc, int64_t n, uint8_t *codes,
                                    float *mults, void *stream) {
  if (n < 0 || (n > 0 && (!amax || !codes || !mults))) return FA4_ERR_INVALID_ARG;
  return cuda_status(fa4::launch_debug_nv_block_scale(amax, s_enc, n, codes, mults, S(stream)));
}

fa4_status fa4_debug_silu(const void *g, int64_t n, float *out, void *stream) {
  if (n < 0 || (n > 0 && (!g || !out))) return FA4_ERR_INVALID_ARG;
  return cuda_status(fa4::launch_debug_silu(static_cast<const uint16_t *>(g), n, out, S(stream)));
}

fa4_status fa4_debug_sr_bits(uint64_t seed, const uint64_t *idx, int64_t n, uint32_t *bits,
                             void *stream) {
  if (n < 0 || (n > 0 && (!idx || !bits))) return FA4_ERR_INVALID_ARG;
  return cuda_status(fa4::launch_debug_sr_bits(seed, idx, n, bits, S(stream)));
}

fa4_status fa4_debug_gemm_timeout(fa4_qtensor A, fa4_qtensor B, int64_t M, int64_t N, int64_t K,
                                  fa4_format fmt, void *D, int64_t ldd, int skip_k_tile,
                                  uint64_t timeout_ns, void *workspace, size_t workspace_bytes,
                                  void *stream) {
  fa4_status s = check_gemm(A, B, M, N, K, fmt, D, ldd, FA4_OUT_FP32, workspace, workspace_bytes);
  if (s != FA4_OK) return s;
  if (timeout_ns == 0 || timeout_ns > kDefaultTimeoutNs) return FA4_ERR_INVALID_ARG;
  return do_gemm(A, B, M, N, K, fmt, 1.0f, D, ldd, FA4_OUT_FP32, static_cast<uint8_t *>(workspace),
                 S(stream), skip_k_tile, timeout_ns);
}

}  // extern "C"
