// quantize.cu -- fused FP4 quantization producers for sm_100a.
//
// One kernel per orientation (and one for both) does the whole producer of "FP4 Is No Longer
// Just a Hardware Feature -- The NVFP4 Software Stack Is Taking Shape",
// section "The first change" (block amax -> scale -> divide -> E2M1 -> pack
// two values per byte) in registers, and writes the scale bytes straight into
// the 128x4 atoms the block-scaled MMA reads, so nothing intermediate goes to
// memory (the unfused pipeline that section warns about writes amax and
// scales and re-reads the tensor).  The scale domain is a template parameter
// ("Format-Aware Fusion: The Engineering Practice That Doubles FP4
// Pretraining Throughput", section "The Design Philosophy of Format-Aware
// Fusion"): native MX, global NV (second pass after tensor_amax_kernel) or
// CTA-local NV (the 128x128 tile amax is reduced inside the CTA that
// quantizes the tile, so the tensor is read once).
//
// Work unit: one CTA of 256 threads per 128x128 tile of the quantized
// operand Q.  The tile (32 KB of bf16) is loaded with 16-byte coalesced
// loads, all issued before any arithmetic.
//
// Ragged shapes: Q[R, K] with any R and K a multiple of 32.  Tiles cut by
// the tensor's edge run the EDGE variant of the kernel, which reads zeros
// outside the tensor -- zeros change no block, tile or tensor amax -- and
// stores only the payload inside it; every scale byte of the padded atoms
// (rows up to the next multiple of 128, blocks up to the next multiple of
// 4) is written, zero outside the tensor.  When only R is ragged the uncut
// tiles run the unmasked kernel; when K is, every tile runs the EDGE
// variant (the atom stride along K is then the padded one).
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa4_device.cuh"
#include "fa4_kernels.h"

namespace fa4 {

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void unpack8(const uint4 &w, float *f) {
  f[0] = bf16lo(w.x); f[1] = bf16hi(w.x);
  f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
  f[4] = bf16lo(w.z); f[5] = bf16hi(w.z);
  f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
}

__device__ __forceinline__ float absmax8(const uint4 &w) {
  // |bf16| max on the packed pairs: clear sign bits, max of the magnitudes
  // as unsigned integers orders non-negative floats correctly
  const uint32_t m = 0x7FFF7FFFu;
  uint32_t a = __vmaxu2(w.x & m, w.y & m);
  uint32_t b = __vmaxu2(w.z & m, w.w & m);
  a = __vmaxu2(a, b);
  const uint32_t hi = a >> 16, lo = a & 0xFFFFu;
  return __uint_as_float((hi > lo ? hi : lo) << 16);
}

// CTA-wide max of one value per thread (256 threads).
__device__ __forceinline__ float cta_max256(float v, float *red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) r = fmaxf(r, red[i]);
  return r;
}

// Largest of the NV-global amax partials, read by every CTA.
__device__ __forceinline__ float reduce_partials(const float *partials, int n, float *red) {
  float m = 0.0f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, partials[i]);
  return cta_max256(m, red);
}

// --------------------------------------------------------------------------
// Tensor amax (NVFP4-global, pass 1): grid-stride over x[rows, cols] in
// 8-element chunks; one partial maximum per CTA.
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) tensor_amax_kernel(const uint16_t *__restrict__ x,
                                                          int64_t rows, int64_t cols, int64_t ld,
                                                          float *__restrict__ partials) {
  __shared__ float red[8];
  const int64_t cpr = cols >> 3;  // chunks per row
  const int64_t n = rows * cpr;
  float m = 0.0f;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (; i + 3 * stride < n; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t c = i + u * stride;
      v[u] = ld_stream(x + (c / cpr) * ld + (c % cpr) * 8);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) m = fmaxf(m, absmax8(v[u]));
  }
  for (; i < n; i += stride) m = fmaxf(m, absmax8(ld_stream(x + (i / cpr) * ld + (i % cpr) * 8)));
  m = cta_max256(m, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

// --------------------------------------------------------------------------
// Row-wise quantizer: Q = x[R, K], blocks along a row.
// Thread layout in a 128x128 tile: warp w, lane l -> rows 16*s + 2*w + (l>>4)
// for steps s = 0..7, columns 8*(l&15) .. +8.  A half-warp covers one row;
// NV blocks (16) are lane pairs, MX blocks (32) lane quads.
// --------------------------------------------------------------------------
// Row-wise quantization of one 128x128 tile of Q held in registers: v[s] is
// row r0 + 16 s + 2 w + (l >> 4), columns k0 + 8 (l & 15) .. + 8.  s_enc is the
// NVFP4 encode scale (unused for MXFP4).
// EDGE: Q has R rows; chunks outside Q hold zeros and are not stored.
template <int FMT, int RND, bool EDGE>
__device__ __forceinline__ void rowwise_tile(const uint4 (&v)[8], int64_t r0, int64_t k0, int64_t R,
                                             int64_t K, uint8_t *__restrict__ payload,
                                             uint8_t *__restrict__ scales, float s_enc,
                                             uint64_t seed) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int c = l & 15;          // 8-element chunk within the 128-wide row
  const int64_t kc = k0 + 8 * c;  // first column of the chunk
  const int64_t kb = is_mx<FMT>() ? (K >> 5) : (K >> 4);  // blocks per row
  // blocks per atom row: padded to a multiple of 4 (already one unless EDGE)
  const int64_t kbt = EDGE ? ((kb + 3) & ~int64_t(3)) : kb;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int64_t r = r0 + 16 * s + 2 * w + (l >> 4);
    const bool inside = !EDGE || (r < R && kc < K);
    float f[8];
    unpack8(v[s], f);
    float amax = absmax8(v[s]);
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
    if constexpr (is_mx<FMT>()) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
    uint32_t sbyte;
    if constexpr (is_mx<FMT>()) {
      sbyte = mx_byte<FMT>(amax);
      const float mult = mx_multiplier(sbyte);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(f[e], mult);
    } else {
      float mult;
      sbyte = nv_block_scale(amax, s_enc, &mult);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(f[e], mult);
    }
    if (EDGE && !inside) sbyte = 0u;  // padding scale bytes are zero
    uint32_t codes;
    if constexpr (RND == kSR) {
      codes = e2m1x8_sr(f, sr_block_bits(seed, (uint64_t)(r * K + kc) >> 3));
    } else {
      codes = e2m1x8_rne(f);
    }
    if (inside) *reinterpret_cast<uint32_t *>(payload + r * (K >> 1) + (kc >> 1)) = codes;

    // gather four consecutive block scales of the row into one word
    uint32_t word;
    if constexpr (is_mx<FMT>()) {
      word = sbyte << (8 * (c >> 2));
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 4);
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 8);
      if (c == 0) *reinterpret_cast<uint32_t *>(scales + sf_offset(r, k0 >> 5, kbt)) = word;
    } else {
      word = sbyte << (8 * ((c >> 1) & 3));
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 4);
      // a word whose first block is past the row's last one lies outside
      // the padded atoms (only in an EDGE tile)
      if ((c & 7) == 0 && (!EDGE || (k0 >> 4) + 4 * (c >> 3) < kb))
        *reinterpret_cast<uint32_t *>(scales + sf_offset(r, (k0 >> 4) + 4 * (c >> 3), kbt)) = word;
    }
  }
}

// Loads of one 128x128 tile in the row-wise thread layout (16-byte lanes, all
// issued before any arithmetic).  EDGE: chunks outside x[rows, cols] read as
// zeros (cols is a multiple of 8, so a chunk is wholly inside or outside).
template <bool EDGE>
__device__ __forceinline__ void load_tile_rowwise(const uint16_t *__restrict__ x, int64_t ld,
                                                  int64_t r0, int64_t k0, int64_t rows,
                                                  int64_t cols, uint4 (&v)[8]) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int64_t r = r0 + 16 * s + 2 * w + (l >> 4);
    if (!EDGE || (r < rows && k0 + 8 * (l & 15) < cols))
      v[s] = ld_stream(x + r * ld + k0 + 8 * (l & 15));
    else
      v[s] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Tiles of an EDGE launch: blockIdx + (a0, b0) in a grid of n_a tiles along
// the blockIdx.x dimension.  The unmasked launch covers the tiles from
// (0, 0) with the grid's own extent.
struct EdgeTiles {
  int a0, b0, n_a;
};

// NVFP4 encode scale of the tile's domain: CTA-local (this tile's amax, ts
// written at ts_index) or global (reduced from the amax partials, ts[0]
// written by the first tile); 1 for MXFP4.
template <int FMT>
__device__ __forceinline__ float tile_encode_scale(const uint4 (&v)[8], float *__restrict__ ts,
                                                   int64_t ts_index, bool first_tile,
                                                   const float *__restrict__ partials,
                                                   int n_partials, float *red) {
  float s_enc = 1.0f;
  if constexpr (FMT == kNVC) {
    float m = 0.0f;
#pragma unroll
    for (int s = 0; s < 8; ++s) m = fmaxf(m, absmax8(v[s]));
    s_enc = nv_encode_scale(cta_max256(m, red));
    if (threadIdx.x == 0) ts[ts_index] = nv_decode_scale(s_enc);
  } else if constexpr (FMT == kNVG) {
    s_enc = nv_encode_scale(reduce_partials(partials, n_partials, red));
    if (threadIdx.x == 0 && first_tile) ts[0] = nv_decode_scale(s_enc);
  }
  return s_enc;
}

// tiles: x along K, y along R; the CTA-local ts index is [R tile][K tile]
template <int FMT, int RND, bool EDGE>
__global__ void __launch_bounds__(256) quant_rowwise_kernel(
    const uint16_t *__restrict__ x, int64_t R, int64_t K, int64_t ld, uint8_t *__restrict__ payload,
    uint8_t *__restrict__ scales, float *__restrict__ ts, const float *__restrict__ partials,
    int n_partials, uint64_t seed, EdgeTiles e) {
  __shared__ float red[8];
  const int64_t tk = (int64_t)blockIdx.x + (EDGE ? e.a0 : 0);
  const int64_t tr = (int64_t)blockIdx.y + (EDGE ? e.b0 : 0);
  const int64_t k0 = tk * 128, r0 = tr * 128;
  uint4 v[8];
  load_tile_rowwise<EDGE>(x, ld, r0, k0, R, K, v);
  const float s_enc = tile_encode_scale<FMT>(v, ts, tr * (EDGE ? e.n_a : gridDim.x) + tk,
                                             tk == 0 && tr == 0, partials, n_partials, red);
  rowwise_tile<FMT, RND, EDGE>(v, r0, k0, R, K, payload, scales, s_enc, seed);
}

// --------------------------------------------------------------------------
// Column-wise quantizer: Q = x^T, x[T, C] row-major; Q[R = C, K = T].
// The 128(tokens) x 128(channels) tile is staged in shared memory; each
// thread then owns two adjacent channels and one 32-token block, reading
// down the columns (a warp reads 128 contiguous bytes per token: no bank
// conflicts) and keeping all 64 values in registers, so the optional
// Hadamard-32 is an in-register butterfly.
// --------------------------------------------------------------------------
// In-place butterfly with strides 1, 2, 4, 8, 16, (a, b) -> (a + b, a - b),
// on packed pairs: lane lo and lane hi are two independent 32-value blocks
// (two channels) taking the same steps.
__device__ __forceinline__ void fwht32x2(uint64_t *v) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & h) == 0) {
        const uint64_t a = v[i], b = v[i + h];
        v[i] = f2_add(a, b);
        v[i + h] = f2_sub(a, b);
      }
    }
  }
}

// Column-wise quantization of the 128 (tokens) x 128 (channels) tile staged
// in shared memory (tile[token][channel]; complete before the call): Q = x^T,
// rows c0 .. c0+127 of Q, K range t0 .. t0+127.  sbuf holds 128 x 8 scale
// bytes.  Ends with the tile's scale words written.  EDGE: Q has C rows and
// T (a multiple of 32) columns; outside them the staged tile holds zeros.
template <int FMT, int RND, bool HAD, bool EDGE>
__device__ __forceinline__ void colwise_tile(const uint16_t *tile, uint8_t *sbuf, int64_t c0,
                                             int64_t t0, int64_t C, int64_t T,
                                             uint8_t *__restrict__ payload,
                                             uint8_t *__restrict__ scales, float s_enc,
                                             uint64_t seed, uint32_t sign_mask) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int p = (w & 1) * 32 + l;  // channel pair within the tile: 2p, 2p+1
  const int j = w >> 1;            // 32-token block within the tile
  float v0[32], v1[32];  // channels 2p and 2p+1
  if constexpr (HAD) {
    // the two channels' blocks take the same signs and butterfly: run them
    // as packed pairs; a sign is the bf16 sign bit, flipped before widening
    uint64_t w2[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      uint32_t pair = *reinterpret_cast<const uint32_t *>(&tile[(32 * j + t) * 128 + 2 * p]);
      if ((sign_mask >> t) & 1u) pair ^= 0x80008000u;
      w2[t] = f2_pack(bf16lo(pair), bf16hi(pair));
    }
    fwht32x2(w2);
#pragma unroll
    for (int t = 0; t < 32; ++t) f2_unpack(w2[t], v0[t], v1[t]);
  } else {
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const uint32_t pair = *reinterpret_cast<const uint32_t *>(&tile[(32 * j + t) * 128 + 2 * p]);
      v0[t] = bf16lo(pair);
      v1[t] = bf16hi(pair);
    }
  }
  const int64_t kb = is_mx<FMT>() ? (T >> 5) : (T >> 4);  // blocks per row of Q
  // blocks per atom row: padded to a multiple of 4 (already one unless EDGE)
  const int64_t kbt = EDGE ? ((kb + 3) & ~int64_t(3)) : kb;

  // block scales of both channels (MX: one 32-block each; NV: two 16-blocks
  // each, multiplier mult[half][hb])
  const int64_t kfirst = t0 + 32 * j;  // first K index of this 32-block
  float mult[2][2];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const float *v = half ? v1 : v0;
    const int cl = 2 * p + half;  // channel within the tile
    // the thread's 32-token block is wholly inside or outside (T % 32 == 0)
    const bool inside = !EDGE || (c0 + cl < C && kfirst < T);
    if constexpr (is_mx<FMT>()) {
      float amax = 0.0f;
#pragma unroll
      for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(v[t]));
      const uint32_t sbyte = mx_byte<FMT>(amax);
      mult[half][0] = mult[half][1] = mx_multiplier(sbyte);
      sbuf[cl * 8 + j] = (EDGE && !inside) ? (uint8_t)0 : (uint8_t)sbyte;
    } else {
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        float amax = 0.0f;
#pragma unroll
        for (int t = 0; t < 16; ++t) amax = fmaxf(amax, fabsf(v[16 * hb + t]));
        const uint32_t sbyte = nv_block_scale(amax, s_enc, &mult[half][hb]);
        sbuf[cl * 8 + 2 * j + hb] = (EDGE && !inside) ? (uint8_t)0 : (uint8_t)sbyte;
      }
    }
  }
  // y = x * multiplier, both channels at once
#pragma unroll
  for (int t = 0; t < 32; ++t)
    f2_unpack(f2_mul(f2_pack(v0[t], v1[t]), f2_pack(mult[0][t >> 4], mult[1][t >> 4])), v0[t],
              v1[t]);

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float *v = half ? v1 : v0;
    const int cl = 2 * p + half;  // channel within the tile
    const int64_t r = c0 + cl;
    const bool inside = !EDGE || (r < C && kfirst < T);
    uint32_t codes[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if constexpr (RND == kSR) {
        codes[q] = e2m1x8_sr(&v[8 * q], sr_block_bits(seed, (uint64_t)(r * T + kfirst + 8 * q) >> 3));
      } else {
        codes[q] = e2m1x8_rne(&v[8 * q]);
      }
    }
    if (inside)
      *reinterpret_cast<uint4 *>(payload + r * (T >> 1) + (kfirst >> 1)) =
          make_uint4(codes[0], codes[1], codes[2], codes[3]);
  }
  __syncthreads();
  // scale words: MX 4 blocks (one word) per channel, NV 8 blocks (two words)
  if constexpr (is_mx<FMT>()) {
    if (threadIdx.x < 128) {
      const int cl = threadIdx.x;
      const uint32_t word = *reinterpret_cast<const uint32_t *>(&sbuf[cl * 8]);
      *reinterpret_cast<uint32_t *>(scales + sf_offset(c0 + cl, t0 >> 5, kbt)) = word;
    }
  } else {
    const int cl = threadIdx.x >> 1, h = threadIdx.x & 1;
    const uint32_t word = *reinterpret_cast<const uint32_t *>(&sbuf[cl * 8 + 4 * h]);
    if (!EDGE || (t0 >> 4) + 4 * h < kb)  // else past the padded atoms
      *reinterpret_cast<uint32_t *>(scales + sf_offset(c0 + cl, (t0 >> 4) + 4 * h, kbt)) = word;
  }
}

// tiles: x along channels (rows of Q), y along tokens (K of Q); the
// CTA-local ts index is [channel tile][token tile]
template <int FMT, int RND, bool HAD, bool EDGE>
__global__ void __launch_bounds__(256) quant_colwise_kernel(
    const uint16_t *__restrict__ x, int64_t T, int64_t C, int64_t ld, uint8_t *__restrict__ payload,
    uint8_t *__restrict__ scales, float *__restrict__ ts, const float *__restrict__ partials,
    int n_partials, uint64_t seed, uint32_t sign_mask, EdgeTiles e, int n_t) {
  __shared__ __align__(16) uint16_t tile[128 * 128];  // [token][channel]
  __shared__ __align__(16) uint8_t sbuf[128 * 8];     // [channel][block in tile]
  __shared__ float red[8];
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int64_t tc = (int64_t)blockIdx.x + (EDGE ? e.a0 : 0);
  const int64_t tt = (int64_t)blockIdx.y + (EDGE ? e.b0 : 0);
  const int64_t c0 = tc * 128;  // channel = row of Q
  const int64_t t0 = tt * 128;  // token = K of Q
  // stage the tile: half-warp per token row, 16 bytes per lane
  uint4 v[8];
  load_tile_rowwise<EDGE>(x, ld, t0, c0, T, C, v);
#pragma unroll
  for (int s = 0; s < 8; ++s)
    *reinterpret_cast<uint4 *>(&tile[(16 * s + 2 * w + (l >> 4)) * 128 + 8 * (l & 15)]) = v[s];
  // the CTA-local tile of Q = x^T is this tile transposed: same maximum;
  // its ts entry is [c0 / 128][t0 / 128]
  const float s_enc = tile_encode_scale<FMT>(v, ts, tc * (EDGE ? n_t : gridDim.y) + tt,
                                             tc == 0 && tt == 0, partials, n_partials, red);
  __syncthreads();
  colwise_tile<FMT, RND, HAD, EDGE>(tile, sbuf, c0, t0, C, T, payload, scales, s_enc, seed,
                                    sign_mask);
}

// --------------------------------------------------------------------------
// Dual-orientation producer: one read of x[T, C] emits the row-wise operand
// (Q = x, any format) and the column-wise MXFP4 operand (Q = x^T, optionally
// with the fixed-sign Hadamard), e.g. the forward operand and the saved
// weight-gradient operand of an activation, or the data-gradient and
// weight-gradient operands of dY.  Bytes equal those of the two single-
// orientation kernels.
// --------------------------------------------------------------------------
// tiles: x along channels, y along tokens; the row-wise operand's CTA-local
// ts index is [token tile][channel tile].  EDGE launches cover every tile
// (either orientation's atom stride along K may be the padded one).
template <int RFMT, int RRND, int CRND, bool HAD, bool EDGE>
__global__ void __launch_bounds__(256) quant_dual_kernel(
    const uint16_t *__restrict__ x, int64_t T, int64_t C, int64_t ld, uint8_t *__restrict__ row_payload,
    uint8_t *__restrict__ row_scales, float *__restrict__ row_ts, uint8_t *__restrict__ col_payload,
    uint8_t *__restrict__ col_scales, const float *__restrict__ partials, int n_partials,
    uint64_t row_seed, uint64_t col_seed, uint32_t sign_mask) {
  __shared__ __align__(16) uint16_t tile[128 * 128];  // [token][channel]
  __shared__ __align__(16) uint8_t sbuf[128 * 8];
  __shared__ float red[8];
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int64_t c0 = (int64_t)blockIdx.x * 128, t0 = (int64_t)blockIdx.y * 128;
  uint4 v[8];
  load_tile_rowwise<EDGE>(x, ld, t0, c0, T, C, v);
#pragma unroll
  for (int s = 0; s < 8; ++s)
    *reinterpret_cast<uint4 *>(&tile[(16 * s + 2 * w + (l >> 4)) * 128 + 8 * (l & 15)]) = v[s];
  const float s_enc = tile_encode_scale<RFMT>(v, row_ts, (int64_t)blockIdx.y * gridDim.x + blockIdx.x,
                                              blockIdx.x == 0 && blockIdx.y == 0, partials,
                                              n_partials, red);
  rowwise_tile<RFMT, RRND, EDGE>(v, t0, c0, T, C, row_payload, row_scales, s_enc, row_seed);
  __syncthreads();
  colwise_tile<kMX, CRND, HAD, EDGE>(tile, sbuf, c0, t0, C, T, col_payload, col_scales, 1.0f,
                                     col_seed, sign_mask);
}

// --------------------------------------------------------------------------
// Diagnostics kernels (element conversions and SR bits, as the quantizers
// use them).
// --------------------------------------------------------------------------
__global__ void debug_convert_kernel(const float *y, const uint32_t *u16, int64_t n, uint8_t *rne,
                                     uint8_t *sr, uint8_t *e4m3) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = y[i];
  rne[i] = (uint8_t)(e2m1x2_rne(v, 0.0f) & 0xF);
  if (sr) sr[i] = (uint8_t)(e2m1x2_sr(v, 0.0f, u16[i] & 0xFFFFu) & 0xFu);
  if (e4m3) {
    const float sb = fminf(fmaxf(v, 0.001953125f), 448.0f);
    e4m3[i] = (uint8_t)e4m3_rne(sb);
  }
}

__global__ void debug_sr_bits_kernel(uint64_t seed, const uint64_t *idx, int64_t n, uint32_t *bits) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint64_t e = idx[i];
  bits[i] = sr_half(sr_block_bits(seed, e >> 3), (int)(e & 7));
}

// --------------------------------------------------------------------------
// Host-side launchers (called by the C ABI after validation).
// --------------------------------------------------------------------------
int amax_partials_count(int64_t rows, int64_t cols) {
  const int64_t chunks = rows * (cols >> 3);
  int64_t blocks = (chunks + 256 * 8 - 1) / (256 * 8);
  if (blocks > kMaxAmaxPartials) blocks = kMaxAmaxPartials;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

cudaError_t launch_tensor_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                               float *partials, int n_partials, cudaStream_t st) {
  tensor_amax_kernel<<<n_partials, 256, 0, st>>>(x, rows, cols, ld, partials);
  return cudaGetLastError();
}

static unsigned tiles_of(int64_t n) { return (unsigned)((n + 127) / 128); }

// Row-wise: K ragged -> every tile EDGE; else R ragged -> the last row of
// tiles EDGE, the rest unmasked.
template <int FMT, int RND>
static void launch_row(cudaStream_t st, const uint16_t *x, int64_t R, int64_t K, int64_t ld,
                       uint8_t *p, uint8_t *s, float *ts, const float *part, int np, uint64_t seed) {
  const unsigned na = tiles_of(K), nb = tiles_of(R);
  EdgeTiles e = {0, 0, (int)na};
  if (K % 128) {
    quant_rowwise_kernel<FMT, RND, true><<<dim3(na, nb), 256, 0, st>>>(x, R, K, ld, p, s, ts, part,
                                                                       np, seed, e);
    return;
  }
  const unsigned inner = (R % 128) ? nb - 1 : nb;
  if (inner)
    quant_rowwise_kernel<FMT, RND, false><<<dim3(na, inner), 256, 0, st>>>(x, R, K, ld, p, s, ts,
                                                                           part, np, seed, e);
  if (inner < nb) {
    e.b0 = (int)inner;
    quant_rowwise_kernel<FMT, RND, true><<<dim3(na, 1), 256, 0, st>>>(x, R, K, ld, p, s, ts, part,
                                                                      np, seed, e);
  }
}

cudaError_t launch_quant_rowwise(int fmt, int rnd, const uint16_t *x, int64_t R, int64_t K,
                                 int64_t ld, uint8_t *payload, uint8_t *scales, float *ts,
                                 const float *partials, int n_partials, uint64_t seed,
                                 cudaStream_t st) {
#define FA4_ROW(F, Q) \
  if (fmt == F && rnd == Q) launch_row<F, Q>(st, x, R, K, ld, payload, scales, ts, partials, n_partials, seed);
  FA4_ROW(kMX, kRNE) FA4_ROW(kMX, kSR) FA4_ROW(kNVG, kRNE) FA4_ROW(kNVG, kSR) FA4_ROW(kNVC, kRNE)
  FA4_ROW(kMXN, kRNE) FA4_ROW(kMXN, kSR)
  FA4_ROW(kNVC, kSR)
#undef FA4_ROW
  return cudaGetLastError();
}

// Column-wise (Q = x^T): T (K of Q) ragged -> every tile EDGE; else C (rows
// of Q) ragged -> the last column of tiles EDGE, the rest unmasked.
template <int FMT, int RND, bool HAD>
static void launch_col(cudaStream_t st, const uint16_t *x, int64_t T, int64_t C, int64_t ld,
                       uint8_t *p, uint8_t *s, float *ts, const float *part, int np, uint64_t seed,
                       uint32_t mask) {
  const unsigned na = tiles_of(C), nb = tiles_of(T);
  EdgeTiles e = {0, 0, (int)na};
  if (T % 128) {
    quant_colwise_kernel<FMT, RND, HAD, true><<<dim3(na, nb), 256, 0, st>>>(
        x, T, C, ld, p, s, ts, part, np, seed, mask, e, (int)nb);
    return;
  }
  const unsigned inner = (C % 128) ? na - 1 : na;
  if (inner)
    quant_colwise_kernel<FMT, RND, HAD, false><<<dim3(inner, nb), 256, 0, st>>>(
        x, T, C, ld, p, s, ts, part, np, seed, mask, e, (int)nb);
  if (inner < na) {
    e.a0 = (int)inner;
    quant_colwise_kernel<FMT, RND, HAD, true><<<dim3(1, nb), 256, 0, st>>>(
        x, T, C, ld, p, s, ts, part, np, seed, mask, e, (int)nb);
  }
}

cudaError_t launch_quant_colwise(int fmt, int rnd, bool hadamard, uint32_t sign_mask,
                                 const uint16_t *x, int64_t T, int64_t C, int64_t ld,
                                 uint8_t *payload, uint8_t *scales, float *ts,
                                 const float *partials, int n_partials, uint64_t seed,
                                 cudaStream_t st) {
#define FA4_COL(F, Q, H)                                                                   \
  if (fmt == F && rnd == Q && hadamard == H)                                               \
    launch_col<F, Q, H>(st, x, T, C, ld, payload, scales, ts, partials, n_partials, seed, \
                        sign_mask);
  FA4_COL(kMX, kRNE, false) FA4_COL(kMX, kSR, false) FA4_COL(kMX, kRNE, true)
  FA4_COL(kMX, kSR, true) FA4_COL(kNVG, kRNE, false) FA4_COL(kNVG, kSR, false)
  FA4_COL(kMXN, kRNE, false) FA4_COL(kMXN, kSR, false)
  FA4_COL(kNVC, kRNE, false) FA4_COL(kNVC, kSR, false)
#undef FA4_COL
  return cudaGetLastError();
}

// Both orientations: either extent ragged -> every tile EDGE.
template <int RF, int RR, int CR, bool H>
static void launch_dual_t(cudaStream_t st, const uint16_t *x, int64_t T, int64_t C, int64_t ld,
                          uint8_t *rp, uint8_t *rs, float *rts, uint8_t *cp, uint8_t *cs,
                          const float *part, int np, uint64_t rseed, uint64_t cseed, uint32_t mask) {
  const dim3 g(tiles_of(C), tiles_of(T));
  if ((T % 128) || (C % 128))
    quant_dual_kernel<RF, RR, CR, H, true><<<g, 256, 0, st>>>(x, T, C, ld, rp, rs, rts, cp, cs, part,
                                                              np, rseed, cseed, mask);
  else
    quant_dual_kernel<RF, RR, CR, H, false><<<g, 256, 0, st>>>(x, T, C, ld, rp, rs, rts, cp, cs,
                                                               part, np, rseed, cseed, mask);
}

cudaError_t launch_quant_dual(int row_fmt, int row_rnd, int col_rnd, bool hadamard,
                              uint32_t sign_mask, const uint16_t *x, int64_t T, int64_t C,
                              int64_t ld, uint8_t *row_payload, uint8_t *row_scales, float *row_ts,
                              uint8_t *col_payload, uint8_t *col_scales, const float *partials,
                              int n_partials, uint64_t row_seed, uint64_t col_seed,
                              cudaStream_t st) {
#define FA4_DUAL(F, RR, CR, H)                                                               \
  if (row_fmt == F && row_rnd == RR && col_rnd == CR && hadamard == H)                       \
    launch_dual_t<F, RR, CR, H>(st, x, T, C, ld, row_payload, row_scales, row_ts, col_payload, \
                                col_scales, partials, n_partials, row_seed, col_seed, sign_mask);
#define FA4_DUAL_F(F)                                                                 \
  FA4_DUAL(F, kRNE, kRNE, false) FA4_DUAL(F, kRNE, kRNE, true) FA4_DUAL(F, kRNE, kSR, false) \
  FA4_DUAL(F, kRNE, kSR, true) FA4_DUAL(F, kSR, kRNE, false) FA4_DUAL(F, kSR, kRNE, true)    \
  FA4_DUAL(F, kSR, kSR, false) FA4_DUAL(F, kSR, kSR, true)
  FA4_DUAL_F(kMX) FA4_DUAL_F(kNVG) FA4_DUAL_F(kNVC) FA4_DUAL_F(kMXN)
#undef FA4_DUAL_F
#undef FA4_DUAL
  return cudaGetLastError();
}

cudaError_t launch_debug_convert(const float *y, const uint32_t *u16, int64_t n, uint8_t *rne,
                                 uint8_t *sr, uint8_t *e4m3, cudaStream_t st) {
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (n > 0) debug_convert_kernel<<<blocks, 256, 0, st>>>(y, u16, n, rne, sr, e4m3);
  return cudaGetLastError();
}

cudaError_t launch_debug_sr_bits(uint64_t seed, const uint64_t *idx, int64_t n, uint32_t *bits,
                                 cudaStream_t st) {
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (n > 0) debug_sr_bits_kernel<<<blocks, 256, 0, st>>>(seed, idx, n, bits);
  return cudaGetLastError();
}

}  // namespace fa4
