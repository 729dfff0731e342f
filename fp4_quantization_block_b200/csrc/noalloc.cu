// noalloc.cu -- NVFP4-global quantization for callers that cannot allocate
// device memory.
//
// fa4_quantize with FA4_NVFP4_GLOBAL needs scratch for the per-CTA partial
// maxima of its tensor-amax pass, which fa4_quantize takes from the caller's
// workspace.  Some callers have no workspace to give: a runtime that reserves
// all device memory up front under a fixed plan and hands out no scratch, or
// code that must not call cudaMalloc at that point (it can synchronize the
// device and stall other streams, or the allocator belongs to another
// library).  fa4_quantize_nvfp4_global_noalloc keeps that scratch in a
// file-scope __device__ array instead: kMaxAmaxPartials floats (4736 bytes),
// which every GPU that loads this library holds until the process exits.
//
// The kernels are the same as fa4_quantize's; only the scratch differs.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/fa4.h"
#include "fa4_kernels.h"

namespace {

// One partial maximum per CTA of the amax pass; never more than
// kMaxAmaxPartials CTAs are launched.  Every call overwrites the partials it
// reads, so nothing has to start at zero.
__device__ __align__(256) float g_amax_scratch[fa4::kMaxAmaxPartials];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
float *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_amax_scratch on the current device.  In host code the
// symbol's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
fa4_status scratch_for_current_device(float **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA4_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA4_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_amax_scratch) != cudaSuccess || !p) return FA4_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<float *>(p);
  }
  *out = g_scratch_ptr[dev];
  return FA4_OK;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

fa4_status fa4_quantize_nvfp4_global_noalloc(const void *x, int64_t rows, int64_t cols, int64_t ld,
                                             fa4_round rnd, fa4_orient orient, uint64_t seed,
                                             fa4_qtensor out, void *stream) {
  if ((rnd != FA4_RNE && rnd != FA4_SR) || (orient != FA4_ROWWISE && orient != FA4_COLWISE))
    return FA4_ERR_INVALID_ARG;
  if (!x || !out.payload || !out.scales || !out.tensor_scale) return FA4_ERR_INVALID_ARG;
  // Q[R, K]: any R, K a multiple of 32; x rows read in 16-byte pieces
  const int64_t K = orient == FA4_ROWWISE ? cols : rows;
  if (rows <= 0 || cols <= 0 || cols % 8 || K % 32 || ld < cols || ld % 8) return FA4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(out.payload) || !aligned16(out.scales) ||
      (reinterpret_cast<uintptr_t>(out.tensor_scale) & 3u))
    return FA4_ERR_ALIGN;
  // the partial maxima this call needs must fit in the static scratch
  const int np = fa4::amax_partials_count(rows, cols);
  if (np > fa4::kMaxAmaxPartials) return FA4_ERR_WORKSPACE;
  float *partials = nullptr;
  fa4_status s = scratch_for_current_device(&partials);
  if (s != FA4_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  fa4::QuantArgs q;
  q.x = static_cast<const uint16_t *>(x);
  q.T = rows;
  q.C = cols;
  q.ld = ld;
  q.partials = partials;
  q.n_partials = np;
  if (fa4::launch_tensor_amax(q.x, rows, cols, ld, partials, np, st) != cudaSuccess) return FA4_ERR_CUDA;
  if (orient == FA4_ROWWISE) {
    q.row_fmt = FA4_NVFP4_GLOBAL;
    q.row_rnd = rnd;
    q.row_payload = static_cast<uint8_t *>(out.payload);
    q.row_scales = static_cast<uint8_t *>(out.scales);
    q.row_ts = out.tensor_scale;
    q.row_seed = seed;
  } else {
    q.col_fmt = FA4_NVFP4_GLOBAL;
    q.col_rnd = rnd;
    q.col_payload = static_cast<uint8_t *>(out.payload);
    q.col_scales = static_cast<uint8_t *>(out.scales);
    q.col_ts = out.tensor_scale;
    q.col_seed = seed;
  }
  return fa4::launch_quantize(q, st) == cudaSuccess ? FA4_OK : FA4_ERR_CUDA;
}

}  // extern "C"
