// quantize.cu -- fused FP4 quantization producers for sm_100a.
//
// One kernel template does the whole producer of "FP4 Is No Longer Just a
// Hardware Feature -- The NVFP4 Software Stack Is Taking Shape", section
// "The first change" (block amax -> scale -> divide -> E2M1 -> pack two
// values per byte) in registers, and writes the scale bytes straight into the
// 128x4 atoms the block-scaled MMA reads, so nothing intermediate goes to
// memory (the unfused pipeline that section warns about writes amax and
// scales and re-reads the tensor).  The scale domain is a template parameter
// ("Format-Aware Fusion: The Engineering Practice That Doubles FP4
// Pretraining Throughput", section "The Design Philosophy of Format-Aware
// Fusion"): native MX, global NV (second pass after tensor_amax_kernel) or
// CTA-local NV (the 128x128 tile amax is reduced inside the CTA that
// quantizes the tile, so the tensor is read once).  One read of x emits the
// row-wise operand (Q = x), the column-wise operand (Q = x^T, optionally
// through the fixed-sign 32-point Hadamard of "Two Key Numerical
// Techniques"), or both.
//
// Structure: persistent CTAs of 256 threads, two per SM.  Each CTA walks
// 128 x 128 tiles of x; one thread brings tiles into a three-stage
// shared-memory ring with bulk-tensor (TMA) loads issued two tiles ahead, so
// the loads in flight do not depend on registers.  A TMA load past the edge
// of x fills zeros, which change no block, tile or tensor amax.
//   row-wise pass  warp w, lane l: rows 16 s + 2 w + (l >> 4) (s = 0..7),
//                  columns 8 (l & 15) .. + 8 (16-byte shared-memory reads;
//                  an MX block is a lane quad, an NV block a lane pair);
//   column-wise    thread -> two adjacent channels and one 32-token block,
//   pass           reading down the columns (a warp reads 128 contiguous
//                  bytes per token), all 64 values in registers as packed
//                  binary32 pairs, so the Hadamard is an in-register
//                  butterfly on f32x2 adds.
// Scale bytes are stored one byte per block straight into their atom slot.
// Tiles cut by the tensor's edge take the EDGE path, which stores only the
// payload inside the tensor and writes every scale byte of the padded atoms
// (rows up to the next multiple of 128, blocks up to the next multiple of 4),
// zero outside the tensor.
//
// Instruction economy (the SR and Hadamard producers are bound by issue
// slots): block amax on packed bf16 pairs (max.xorsign.abs), the MX scale
// byte read off the bf16 exponent field, NV block scales with an exactly
// rounded division by 6 and a per-tile table of the element multipliers
// s_enc / decode(code), unpack-and-scale on packed pairs, the Philox round
// keys as kernel parameters, and four values per stochastic conversion.
//
// Every wait on a tile load is bounded: past `timeout_ns` the CTA sets the
// status word (when given), waits (bounded) for its own loads in flight and
// returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa4_device.cuh"
#include "fa4_kernels.h"
#include "launch.cuh"

namespace fa4 {

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float absmax8(const uint4 &w) {
  return __uint_as_float((absmax8_bf16(w) & 0x7FFFu) << 16);
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

// --------------------------------------------------------------------------
// Tensor amax (NVFP4-global, pass 1): grid-stride over x[rows, cols] in
// 8-element chunks; one partial maximum per CTA.  Each thread tracks the
// (row, chunk) of its position and advances it by the grid stride without
// dividing.  The loads mark a fraction keep_frac of the lines L2 evict-last: the
// quantizing pass that follows re-reads x (with evict-first loads), and the
// part of x kept in the 126 MB L2 is then read from L2 instead of HBM.
// --------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_keep(const void *p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

__global__ void __launch_bounds__(256) tensor_amax_kernel(const uint16_t *__restrict__ x,
                                                          int64_t rows, int64_t cols, int64_t ld,
                                                          float keep_frac,
                                                          float *__restrict__ partials) {
  __shared__ float red[8];
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.L2::evict_unchanged.b64 %0, %1;"
               : "=l"(pol) : "f"(keep_frac));
  grid_dependency_wait();
  grid_dependents_launch();
  const int64_t cpr = cols >> 3;  // chunks per row
  const int64_t n = rows * cpr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t sr = stride / cpr, sc = stride - sr * cpr;  // the stride in rows + chunks
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t r = i / cpr, c = i - r * cpr;
  float m = 0.0f;
  for (; i + 3 * stride < n; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      v[u] = ld_keep(x + r * ld + c * 8, pol);
      r += sr;
      c += sc;
      if (c >= cpr) {
        c -= cpr;
        ++r;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) m = fmaxf(m, absmax8(v[u]));
  }
  for (; i < n; i += stride) {
    m = fmaxf(m, absmax8(ld_keep(x + r * ld + c * 8, pol)));
    r += sr;
    c += sc;
    if (c >= cpr) {
      c -= cpr;
      ++r;
    }
  }
  m = cta_max256(m, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

namespace qk {

constexpr int kThreads = 256;
constexpr int kStages = 3;
constexpr int kTileBytes = 128 * 128 * 2;  // one 128 x 128 bf16 tile
constexpr int kNone = -1;                  // orientation not produced
constexpr uint32_t kStatusTimeout = 7;

struct Params {
  int64_t T, C;  // x[T, C]
  int tiles_c, tiles_t, ntiles;
  // row-wise operand Q = x [T, C]
  uint8_t *rp, *rs;
  float *rts;
  // column-wise operand Q = x^T [C, T]
  uint8_t *cp, *cs;
  float *cts;
  // Philox4x32 round keys of the two seeds (the last round's complemented,
  // see sr_bits_not)
  uint32_t rkey0[kSrRounds], rkey1[kSrRounds], ckey0[kSrRounds], ckey1[kSrRounds];
  // round-1 constants of each seed for counters below 2^32 (sr_bits_not32)
  uint32_t rpre_hi, rpre_lo, cpre_hi, cpre_lo;
  // fixed-sign Hadamard: 0x80000000 where token t of a 32-block is negated
  uint32_t sgn[32];
  const float *partials;  // NVFP4-global amax partials
  int np;
  uint32_t *status;  // may be null
  uint64_t timeout_ns;
};

struct Ctrl {
  uint64_t full[kStages];
  uint32_t done[kStages];     // warps finished with the stage's current tile
  uint32_t nissued[kStages];  // loads issued into the stage so far
  float red[8];
  float tab_r[128];  // NVFP4 row-wise element multipliers s_enc / decode(code)
  float tab_c[128];  // column-wise
};
constexpr int kSmemBytes = kStages * kTileBytes + (int)sizeof(Ctrl) + 128;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// One bounded probe of a barrier phase; the suspend-time hint (1 ms) lets
// the hardware park a waiting warp until the tile lands.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000000;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > timeout_ns) return false;
  return true;
}
// Every element of x is read once here: the tile loads are evict-first in
// L2, leaving L2 to the quantized outputs (which the GEMM reads next).
__device__ __forceinline__ void issue_tile(uint8_t *smem, Ctrl *cb, const CUtensorMap *map,
                                           const Params &p, int t, int s) {
  const uint32_t bar = smem_u32(&cb->full[s]);
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(kTileBytes)
               : "memory");
  const int x = (t % p.tiles_c) * 128, y = (t / p.tiles_c) * 128;
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem + s * kTileBytes)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(pol)
      : "memory");
}

__device__ __forceinline__ uint4 lds128(const void *p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ uint32_t lds32(const void *p) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
  return v;
}

// The complement of sr_block_bits(seed, i8) (65535 - u in every 16-bit
// half, the form e2m1x8_sr_not takes), with the round keys in
// kernel parameters.
__device__ __forceinline__ u32x4 sr_bits_not(const uint32_t (&k0)[kSrRounds],
                                             const uint32_t (&k1)[kSrRounds], uint64_t i8) {
  uint32_t c0 = (uint32_t)i8, c1 = (uint32_t)(i8 >> 32), c2 = 0u, c3 = 0u;
#pragma unroll
  for (int r = 0; r < kSrRounds; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0[r], n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1[r];
    c1 = (uint32_t)p1;
    c3 = (uint32_t)p0;
    c0 = n0;
    c2 = n2;
  }
  return {c0, ~c1, c2, ~c3};
}
// The same for a counter below 2^32 (its high word zero): in round 0 three
// of the four words are zero, and round 1 multiplies the constant k0[0], so
// pre_hi = hi(0xD2511F53 * k0[0]) ^ k1[1] and pre_lo = lo(0xD2511F53 * k0[0])
// come from the host and the first two rounds cost one product each.
__device__ __forceinline__ u32x4 sr_bits_not32(const uint32_t (&k0)[kSrRounds],
                                               const uint32_t (&k1)[kSrRounds], uint32_t pre_hi,
                                               uint32_t pre_lo, uint32_t i8) {
  const uint64_t q0 = (uint64_t)0xD2511F53u * i8;  // round 0: c = (i8, 0, 0, 0)
  const uint64_t q1 = (uint64_t)0xCD9E8D57u * ((uint32_t)(q0 >> 32) ^ k1[0]);  // round 1
  uint32_t c0 = (uint32_t)(q1 >> 32) ^ k0[1], c1 = (uint32_t)q1;
  uint32_t c2 = (uint32_t)q0 ^ pre_hi, c3 = pre_lo;
#pragma unroll
  for (int r = 2; r < kSrRounds; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0[r], n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1[r];
    c1 = (uint32_t)p1;
    c3 = (uint32_t)p0;
    c0 = n0;
    c2 = n2;
  }
  return {c0, ~c1, c2, ~c3};
}

// MX scale byte from the bf16 bits of a block amax (either half of m): the
// binary32 exponent field of a bf16 value is its own exponent field, so
// e = floor(log2 amax) - 2 clamped at -127 gives byte max(E - 2, 0); without
// clipping, one more when the mantissa exceeds 1.5 (bf16 mantissa > 0x40).
template <int FMT>
__device__ __forceinline__ uint32_t mx_byte_bf16(uint32_t m) {
  const int E = (int)((m >> 7) & 0xFFu);
  if constexpr (FMT == kMXN) {
    if (E == 0) return 0u;
    return (uint32_t)max(E - 2 + ((m & 0x7Fu) > 0x40u ? 1 : 0), 0);
  } else {
    return (uint32_t)max(E - 2, 0);
  }
}

// NVFP4 block scale of a block amax (binary32) under encode scale s_enc:
// s_b = (amax / 6) * s_enc clamped to [2^-9, 448], its E4M3 code, and the
// element multiplier s_enc / decode(code) from the table.
__device__ __forceinline__ uint32_t nv_code(float amax, float s_enc) {
  float sb = __fmul_rn(div6_rn(amax), s_enc);
  sb = fminf(fmaxf(sb, 0.001953125f), 448.0f);
  return e4m3_rne(sb);
}
// tab[code] = s_enc / decode(code) for every E4M3 code (threads 0..127; the
// caller synchronizes before use).  Codes 0 and 127 never occur.
__device__ __forceinline__ void build_tab(float *tab, float s_enc) {
  if (threadIdx.x < 128) tab[threadIdx.x] = __fdiv_rn(s_enc, e4m3_to_float(threadIdx.x));
}

// y = bf16 x * mult for the eight values of w, on packed pairs
__device__ __forceinline__ void unpack_scale8(const uint4 &w, float mult, float *f) {
  const uint64_t mm = f2_pack(mult, mult);
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    f2_unpack(f2_mul(f2_pack_bits(ws[i] << 16, ws[i] & 0xFFFF0000u), mm), f[2 * i], f[2 * i + 1]);
}

// ---------------------------------------------------------- row-wise pass
// Q = x: rows t0.., K range c0..; R = T, K = C.
// C32: every linear index of the operand is below 2^32 (32-bit SR counters)
template <int FMT, int RND, bool EDGE, bool C32>
__device__ __forceinline__ void row_pass(const uint16_t *tile, const Params &p, int tt, int tc,
                                         float s_enc, const float *tab) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, c = l & 15;
  const int base = 2 * w + (l >> 4);  // row within the tile, minus 16 s
  const int64_t K = p.C;
  const int64_t r0 = (int64_t)tt * 128 + base, kc = (int64_t)tc * 128 + 8 * c;
  const int64_t kb = is_mx<FMT>() ? (K >> 5) : (K >> 4);  // blocks per row
  const int64_t kbt = (kb + 3) & ~int64_t(3);              // per atom row
  uint8_t *pay = p.rp + r0 * (K >> 1) + (kc >> 1);
  // this lane's scale byte (the first lane of its block) for s = 0; row
  // 16 s + base of the tile sits at (s & 1) * 256 + (s >> 1) * 4 further
  const int64_t bidx = is_mx<FMT>() ? (kc >> 5) : (kc >> 4);  // block index
  uint8_t *sb0 = p.rs + ((int64_t)tt * (kbt >> 2) + (bidx >> 2)) * 512 + base * 16 + (bidx & 3);
  const bool lead = is_mx<FMT>() ? (c & 3) == 0 : (c & 1) == 0;
  // (C32) linear index of this lane's first element, and the step to row 16 s
  const uint32_t idx32 = (uint32_t)(r0 * K + kc), step32 = (uint32_t)(16 * K);
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int rr = 16 * s + base;
    const uint4 v = lds128(tile + rr * 128 + 8 * c);
    uint32_t m = absmax8_bf16(v);
    m = hmax_abs2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    uint32_t sbyte;
    float mult;
    if constexpr (is_mx<FMT>()) {
      m = hmax_abs2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      sbyte = mx_byte_bf16<FMT>(m);
      mult = mx_multiplier(sbyte);
    } else {
      sbyte = nv_code(__uint_as_float((m & 0x7FFFu) << 16), s_enc);
      mult = tab[sbyte];
    }
    float f[8];
    unpack_scale8(v, mult, f);
    uint32_t codes;
    if constexpr (RND == kSR && C32)
      codes = e2m1x8_sr_not(f, sr_bits_not32(p.rkey0, p.rkey1, p.rpre_hi, p.rpre_lo,
                                             (idx32 + (uint32_t)s * step32) >> 3));
    else if constexpr (RND == kSR)
      codes = e2m1x8_sr_not(f, sr_bits_not(p.rkey0, p.rkey1, (uint64_t)((r0 + 16 * s) * K + kc) >> 3));
    else
      codes = e2m1x8_rne(f);
    const bool inside = !EDGE || (r0 + 16 * s < p.T && kc < K);
    if (inside) *reinterpret_cast<uint32_t *>(pay + (int64_t)16 * s * (K >> 1)) = codes;
    if (lead && (!EDGE || bidx < kbt))
      sb0[(s & 1) * 256 + (s >> 1) * 4] = (EDGE && !inside) ? (uint8_t)0 : (uint8_t)sbyte;
  }
}

// ------------------------------------------------------- column-wise pass
// Q = x^T: rows c0.. (channels), K range t0.. (tokens); R = C, K = T.
// In-place butterfly with strides 1, 2, 4, 8, 16, (a, b) -> (a + b, a - b),
// on packed pairs (two channels' blocks taking the same steps).
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
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int FMT, int RND, bool HAD, bool EDGE, bool C32>
__device__ __forceinline__ void col_pass(const uint16_t *tile, const Params &p, int tt, int tc,
                                         float s_enc, const float *tab) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int pr = (w & 1) * 32 + l;  // channel pair within the tile: 2 pr, 2 pr + 1
  const int j = w >> 1;             // 32-token block within the tile
  const int64_t T = p.T;
  const int64_t kb = is_mx<FMT>() ? (T >> 5) : (T >> 4);  // blocks per row of Q
  const int64_t kbt = (kb + 3) & ~int64_t(3);
  const int64_t kfirst = (int64_t)tt * 128 + 32 * j;  // first K index of the 32-block
  const uint16_t *src = tile + (32 * j) * 128 + 2 * pr;

  uint64_t v2[32];  // token t: (channel 2 pr, channel 2 pr + 1)
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    const uint32_t wd = lds32(src + t * 128);
    if constexpr (HAD) {
      // the sign flip rides on the unpack: + 0x80000000 flips bit 31 of
      // (wd << 16), XOR flips it of the high half
      v2[t] = f2_pack_bits(wd * 65536u + p.sgn[t], (wd & 0xFFFF0000u) ^ p.sgn[t]);
    } else {
      v2[t] = f2_pack_bits(wd << 16, wd & 0xFFFF0000u);
    }
  }
  if constexpr (HAD) fwht32x2(v2);
  float v0[32], v1[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) f2_unpack(v2[t], v0[t], v1[t]);

  // block scales of both channels (MX: one 32-block each; NV: two 16-blocks)
  float mult[2][2];
  uint32_t sbyte[2][2];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const float *v = half ? v1 : v0;
    if constexpr (is_mx<FMT>()) {
      float a = fabsf(v[0]);
#pragma unroll
      for (int t = 1; t < 31; t += 2) a = fmax3(a, fabsf(v[t]), fabsf(v[t + 1]));
      a = fmaxf(a, fabsf(v[31]));
      sbyte[half][0] = mx_byte<FMT>(a);
      mult[half][0] = mult[half][1] = mx_multiplier(sbyte[half][0]);
    } else {
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        float a = fabsf(v[16 * hb]);
#pragma unroll
        for (int t = 1; t < 15; t += 2) a = fmax3(a, fabsf(v[16 * hb + t]), fabsf(v[16 * hb + t + 1]));
        a = fmaxf(a, fabsf(v[16 * hb + 15]));
        sbyte[half][hb] = nv_code(a, s_enc);
        mult[half][hb] = tab[sbyte[half][hb]];
      }
    }
  }
  // y = x * multiplier, both channels at once
#pragma unroll
  for (int t = 0; t < 32; ++t)
    f2_unpack(f2_mul(f2_pack(v0[t], v1[t]), f2_pack(mult[0][t >> 4], mult[1][t >> 4])), v0[t], v1[t]);

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float *v = half ? v1 : v0;
    const int cl = 2 * pr + half;  // channel within the tile
    const int64_t r = (int64_t)tc * 128 + cl;
    const bool inside = !EDGE || (r < p.C && kfirst < T);
    uint32_t codes[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if constexpr (RND == kSR && C32)
        codes[q] = e2m1x8_sr_not(&v[8 * q], sr_bits_not32(p.ckey0, p.ckey1, p.cpre_hi, p.cpre_lo,
                                                          ((uint32_t)(r * T + kfirst) + 8u * q) >> 3));
      else if constexpr (RND == kSR)
        codes[q] = e2m1x8_sr_not(&v[8 * q], sr_bits_not(p.ckey0, p.ckey1, (uint64_t)(r * T + kfirst + 8 * q) >> 3));
      else
        codes[q] = e2m1x8_rne(&v[8 * q]);
    }
    if (inside)
      *reinterpret_cast<uint4 *>(p.cp + r * (T >> 1) + (kfirst >> 1)) =
          make_uint4(codes[0], codes[1], codes[2], codes[3]);
    // scale bytes at their atom slots: row r = channel, block kfirst / bs
    const int64_t bidx = is_mx<FMT>() ? (kfirst >> 5) : (kfirst >> 4);
    uint8_t *dst = p.cs + ((int64_t)tc * (kbt >> 2) + (bidx >> 2)) * 512 + (cl & 31) * 16 +
                   ((cl >> 5) & 3) * 4 + (bidx & 3);
    if constexpr (is_mx<FMT>()) {
      *dst = (EDGE && !inside) ? (uint8_t)0 : (uint8_t)sbyte[half][0];
    } else {
      // the block pair 2j, 2j+1 is adjacent in its atom word
      if (!EDGE || bidx < kbt)
        *reinterpret_cast<uint16_t *>(dst) =
            (EDGE && !inside) ? (uint16_t)0 : (uint16_t)(sbyte[half][0] | (sbyte[half][1] << 8));
    }
  }
}

// --------------------------------------------------------------- kernel
template <int RF, int RR, int CF, int CR, bool HAD, bool C32>
__global__ void __launch_bounds__(kThreads, 2)
    quant_kernel(const __grid_constant__ CUtensorMap xmap, const Params p) {
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(qsmem_raw) + 127) &
                                              ~uintptr_t(127));
  Ctrl *cb = reinterpret_cast<Ctrl *>(smem + kStages * kTileBytes);
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&cb->full[s])) : "memory");
      cb->done[s] = 0;
      cb->nissued[s] = 0;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  grid_dependency_wait();
  grid_dependents_launch();
  __syncthreads();
  if (tid == 0)
    for (int k = 0; k < kStages; ++k) {
      const int t = (int)blockIdx.x + k * (int)gridDim.x;
      if (t < p.ntiles) {
        issue_tile(smem, cb, &xmap, p, t, k);
        cb->nissued[k] = 1;
      }
    }

  // NVFP4-global: the encode scale from the amax partials, once per CTA
  float senc_g = 1.0f;
  if constexpr (RF == kNVG || CF == kNVG) {
    float m = 0.0f;
    for (int i = tid; i < p.np; i += kThreads) m = fmaxf(m, p.partials[i]);
    senc_g = nv_encode_scale(cta_max256(m, cb->red));
    if (blockIdx.x == 0 && tid == 0) {
      if (RF == kNVG) p.rts[0] = nv_decode_scale(senc_g);
      if (CF == kNVG) p.cts[0] = nv_decode_scale(senc_g);
    }
    if (RF == kNVG) build_tab(cb->tab_r, senc_g);
    if (CF == kNVG) build_tab(cb->tab_c, senc_g);
    __syncthreads();
  }

  // Warps run through the tiles without CTA barriers: a warp releases a
  // stage when it is done with the tile, and the last warp to release it
  // loads the tile kStages ahead into it.  (CTA-local NVFP4 needs the
  // tile's amax from every warp, so it synchronizes the CTA per tile.)
  constexpr bool kLocal = RF == kNVC || CF == kNVC;
  const int lane = tid & 31;
  int it = 0;
  bool failed = false;
  for (int t = (int)blockIdx.x; t < p.ntiles; t += (int)gridDim.x, ++it) {
    const int s = it % kStages;
    const bool ok = wait_bounded(smem_u32(&cb->full[s]), (uint32_t)((it / kStages) & 1), p.timeout_ns);
    // the decision to stop is uniform over the CTA (CTA-local) or the warp
    // (a lane that saw the load land still stops with a lane that gave up)
    if (kLocal ? __syncthreads_or(!ok) : !__all_sync(0xFFFFFFFFu, ok)) {
      failed = true;
      if (p.status && atomicCAS(p.status, 0u, kStatusTimeout) == 0u)
        atomicExch(p.status + 1, 0x600u | (uint32_t)s);
      break;
    }
    const uint16_t *tile = reinterpret_cast<const uint16_t *>(smem + s * kTileBytes);
    const int tc = t % p.tiles_c, tt = t / p.tiles_c;
    float senc_r = senc_g, senc_c = senc_g;
    if constexpr (kLocal) {
      // CTA-local: the tile's amax (Q's tile in either orientation holds the
      // same values), its decode scale and multiplier table
      const int w = tid >> 5;
      float m = 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        m = fmaxf(m, absmax8(lds128(tile + (16 * k + 2 * w + (lane >> 4)) * 128 + 8 * (lane & 15))));
      const float se = nv_encode_scale(cta_max256(m, cb->red));
      if constexpr (RF == kNVC) {
        senc_r = se;
        if (tid == 0) p.rts[(int64_t)tt * p.tiles_c + tc] = nv_decode_scale(se);
        build_tab(cb->tab_r, se);
      }
      if constexpr (CF == kNVC) {
        senc_c = se;
        if (tid == 0) p.cts[(int64_t)tc * p.tiles_t + tt] = nv_decode_scale(se);
        build_tab(cb->tab_c, se);
      }
      __syncthreads();
    }
    const bool edge = ((int64_t)tt * 128 + 128 > p.T) || ((int64_t)tc * 128 + 128 > p.C);
    if constexpr (RF != kNone) {
      if (edge)
        row_pass<RF, RR, true, C32>(tile, p, tt, tc, senc_r, cb->tab_r);
      else
        row_pass<RF, RR, false, C32>(tile, p, tt, tc, senc_r, cb->tab_r);
    }
    if constexpr (CF != kNone) {
      if (edge)
        col_pass<CF, CR, HAD, true, C32>(tile, p, tt, tc, senc_c, cb->tab_c);
      else
        col_pass<CF, CR, HAD, false, C32>(tile, p, tt, tc, senc_c, cb->tab_c);
    }
    if constexpr (kLocal) __syncthreads();  // the multiplier tables are rewritten next tile
    // release stage s; the last warp out refills it (its reads, and every
    // other warp's, are ordered before the load by the fence and the
    // counter's read-modify-write)
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&cb->done[s], 1u) == kThreads / 32 - 1) {
        atomicExch(&cb->done[s], 0u);
        const int tn = t + kStages * (int)gridDim.x;
        if (tn < p.ntiles) {
          issue_tile(smem, cb, &xmap, p, tn, s);
          atomicAdd(&cb->nissued[s], 1u);
        }
      }
    }
  }
  if (failed && lane == 0) {
    // loads still in flight write this CTA's shared memory: let them land
    // before the warp leaves (the n-th load into a stage completes the
    // phase of parity (n - 1) & 1)
    for (int k = 0; k < kStages; ++k) {
      const uint32_t n = *(volatile uint32_t *)&cb->nissued[k];
      if (n == 0) continue;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(&cb->full[k]), (n - 1) & 1u))
        if (globaltimer() - t0 > p.timeout_ns) break;
    }
  }
}

// ------------------------------------------------ SwiGLU producer, fused
// The producer of the down projection's input, fused with its quantizer:
// z[T, 2F] (the gate+up output: gate = z[:, :F], up = z[:, F:]) ->
// h = bf16(silu(gate) * up), quantized row-wise (MXFP4, MXFP4 without
// clipping, or CTA-local NVFP4) and optionally column-wise MXFP4 (with the
// fixed-sign Hadamard: the down projection's saved weight-gradient operand).
// h never leaves the chip.  The arithmetic is fixed step by step (binary32,
// one bf16 rounding at the end): silu(g) = g / (1 + exp(-g)) with
//   exp(x): clamp x to [-87, 88]; n = rint(x * RN(log2 e));
//           r = x - n * ln2 in two fused steps (ln2 = a 15-bit head + tail,
//           the Cody-Waite additive reduction); p = degree-6 Taylor
//           polynomial of e^r by fused multiply-adds from 1/720; p * 2^n.
// Two values at a time on packed binary32 pairs (each lane rounds exactly as
// the scalar step).  rint(y) for |y| < 2^22 is RN(y + 1.5 * 2^23) - 1.5 *
// 2^23 (the sum has unit spacing and an even offset, so ties go to even as
// rint's), and the sum's low bits are n itself, which gives 2^n as an
// integer.  The quotient g / d (d = 1 + exp(-g) >= 1) is the correctly
// rounded one through Markstein's correction ("Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): a hardware reciprocal estimate y0, one Newton step y1 = y0 + y0 (1
// - d y0), q0 = g y1, the exact remainder r = g - d q0 (one fused
// multiply-add), q = q0 + r y1.  Both g and d are first scaled by 2^-k, k =
// min(max(n, 0), 126), which is exact and keeps d in [0.7, 2.9] (1/d would
// be subnormal for d >= 2^126).  Checked bit for bit against the IEEE quotient for every
// finite bf16 gate value (fa4_debug_silu).
// One CTA of 256 threads per 128 x 128 tile of h: each thread loads its
// gate and up chunks (16-byte loads, all issued before any arithmetic),
// computes its 64 values of h into the shared-memory tile, and the row-wise
// and column-wise passes of the quantizer run on the tile.
__device__ __forceinline__ uint64_t f2_splat(float v) { return f2_pack(v, v); }
__device__ __forceinline__ float rcp_estimate(float d) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(d));
  return y;
}
// silu of the two bf16 values in the halves of gw, as a packed binary32 pair
__device__ __forceinline__ uint64_t silu2(uint32_t gw) {
  const float g0 = bf16lo(gw), g1 = bf16hi(gw);
  const uint64_t x = f2_pack(fminf(fmaxf(-g0, -87.0f), 88.0f), fminf(fmaxf(-g1, -87.0f), 88.0f));
  const uint64_t shift = f2_splat(12582912.0f);  // 1.5 * 2^23
  const uint64_t t = f2_add(f2_mul(x, f2_splat(1.44269502162933349609375f)), shift);
  const uint64_t nn = f2_sub(shift, t);  // -n, exactly
  uint64_t r = f2_fma(nn, f2_splat(0.693145751953125f), x);
  r = f2_fma(nn, f2_splat(1.42860677e-6f), r);
  uint64_t p = f2_fma(f2_splat(1.38888892e-3f), r, f2_splat(8.33333377e-3f));
  p = f2_fma(p, r, f2_splat(4.16666679e-2f));
  p = f2_fma(p, r, f2_splat(1.66666672e-1f));
  p = f2_fma(p, r, f2_splat(0.5f));
  p = f2_fma(p, r, f2_splat(1.0f));
  p = f2_fma(p, r, f2_splat(1.0f));
  uint32_t t0, t1;
  f2_unpack_bits(t, t0, t1);
  // n << 23 (two's complement) from the low bits of t; 2^n and 2^-max(n, 0)
  const int a0 = (int)(t0 << 23), a1 = (int)(t1 << 23);
  const uint64_t e = f2_mul(p, f2_pack_bits((uint32_t)a0 + 0x3F800000u, (uint32_t)a1 + 0x3F800000u));
  const uint64_t d = f2_add(f2_splat(1.0f), e);
  // 2^-k, k = max(n, 0) capped at 126 (2^-127 is not a normal number):
  // 0x3F800000 - (n << 23) clamped to [2^-126, 1]
  const uint32_t s0 = (uint32_t)min(max(0x3F800000 - a0, 0x00800000), 0x3F800000);
  const uint32_t s1 = (uint32_t)min(max(0x3F800000 - a1, 0x00800000), 0x3F800000);
  // with negated numerator and reciprocal, so that q keeps the sign of a
  // zero g: -gs, -y0, -y1, q0 = (-gs)(-y1), -r = ds q0 - gs, q = q0 + (-r)(-y1)
  const uint64_t ds = f2_mul(d, f2_pack_bits(s0, s1));
  const uint64_t dn = f2_mul(d, f2_pack_bits(s0 | 0x80000000u, s1 | 0x80000000u));  // -ds
  const uint64_t gn = f2_mul(f2_pack(g0, g1), f2_pack_bits(s0 | 0x80000000u, s1 | 0x80000000u));
  float d0, d1;
  f2_unpack(dn, d0, d1);
  const uint64_t y0n = f2_pack(rcp_estimate(d0), rcp_estimate(d1));
  const uint64_t y1n = f2_fma(y0n, f2_fma(ds, y0n, f2_splat(1.0f)), y0n);
  const uint64_t q0 = f2_mul(gn, y1n);
  return f2_fma(f2_fma(ds, q0, gn), y1n, q0);
}
// bf16 bits of silu(g) * u for the bf16 values in the halves of gw, uw
__device__ __forceinline__ uint32_t swiglu2(uint32_t gw, uint32_t uw) {
  float h0, h1;
  f2_unpack(f2_mul(silu2(gw), f2_pack(bf16lo(uw), bf16hi(uw))), h0, h1);
  const __nv_bfloat162 b = __floats2bfloat162_rn(h0, h1);
  return *reinterpret_cast<const uint32_t *>(&b);
}

constexpr int kSwigluCtasPerSm = 2;
template <int RF, int RR, int CF, int CR, bool HAD, bool C32>
__global__ void __launch_bounds__(kThreads, kSwigluCtasPerSm)
    swiglu_quant_kernel(const Params p, const uint16_t *__restrict__ z, int64_t ld) {
  __shared__ __align__(16) uint16_t tile[128 * 128];
  __shared__ float red[8];
  __shared__ float tab[128];
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const int tc = (int)blockIdx.x, tt = (int)blockIdx.y;
  const int64_t F = p.C, r0 = (int64_t)tt * 128, c0 = (int64_t)tc * 128;
  grid_dependency_wait();
  grid_dependents_launch();
  uint4 g[8], u[8];
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int64_t r = r0 + 16 * s + 2 * w + (l >> 4), c = c0 + 8 * (l & 15);
    if (r < p.T && c < F) {
      g[s] = ld_stream(z + r * ld + c);
      u[s] = ld_stream(z + r * ld + F + c);
    } else {
      g[s] = u[s] = make_uint4(0u, 0u, 0u, 0u);  // h = silu(0) * 0 = 0 outside
    }
  }
  uint32_t mb = 0u;  // largest |h| of this thread's values (bf16 bits), for the tile amax
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const uint4 h = make_uint4(swiglu2(g[s].x, u[s].x), swiglu2(g[s].y, u[s].y),
                               swiglu2(g[s].z, u[s].z), swiglu2(g[s].w, u[s].w));
    *reinterpret_cast<uint4 *>(&tile[(16 * s + 2 * w + (l >> 4)) * 128 + 8 * (l & 15)]) = h;
    if constexpr (RF == kNVC) mb = hmax_abs2(mb, absmax8_bf16(h));
  }
  float senc = 1.0f;
  if constexpr (RF == kNVC) {
    // (cta_max256 synchronizes the CTA before its exchange, which also
    // orders the tile stores above before the passes below)
    senc = nv_encode_scale(cta_max256(__uint_as_float((mb & 0x7FFFu) << 16), red));
    if (tid == 0) p.rts[(int64_t)tt * p.tiles_c + tc] = nv_decode_scale(senc);
    build_tab(tab, senc);
  }
  __syncthreads();
  const bool edge = (r0 + 128 > p.T) || (c0 + 128 > F);
  if (edge)
    row_pass<RF, RR, true, C32>(tile, p, tt, tc, senc, tab);
  else
    row_pass<RF, RR, false, C32>(tile, p, tt, tc, senc, tab);
  if constexpr (CF != kNone) {
    if (edge)
      col_pass<CF, CR, HAD, true, C32>(tile, p, tt, tc, 1.0f, nullptr);
    else
      col_pass<CF, CR, HAD, false, C32>(tile, p, tt, tc, 1.0f, nullptr);
  }
}

}  // namespace qk

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

// The NVFP4 block-scale step exactly as the quantizers run it (qk::nv_code
// and the multiplier table).
__global__ void debug_nv_block_scale_kernel(const float *amax, float s_enc, int64_t n, uint8_t *codes,
                                            float *mults) {
  __shared__ float tab[128];
  qk::build_tab(tab, s_enc);
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t code = qk::nv_code(amax[i], s_enc);
  codes[i] = (uint8_t)code;
  mults[i] = tab[code];
}

// silu(g) exactly as the SwiGLU producer computes it, for n bf16 values
// (pairs; an odd tail value is paired with zero).
__global__ void debug_silu_kernel(const uint16_t *g, int64_t n, float *out) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const uint32_t gw = (uint32_t)g[i] | (i + 1 < n ? (uint32_t)g[i + 1] << 16 : 0u);
  float s0, s1;
  f2_unpack(qk::silu2(gw), s0, s1);
  out[i] = s0;
  if (i + 1 < n) out[i + 1] = s1;
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
  // keep at most ~80 MB of x (of the 126 MB L2) for the quantizing pass
  const double bytes = 2.0 * (double)rows * (double)cols;
  const float keep = bytes <= 80.0e6 ? 1.0f : (float)(80.0e6 / bytes);
  const cudaError_t e = launch_pdl(tensor_amax_kernel, dim3((unsigned)n_partials), dim3(256), 0, st, x,
                                   rows, cols, ld, keep, partials);
  return e != cudaSuccess ? e : cudaGetLastError();
}

namespace {

// Philox4x32 key schedule (the Weyl sequence of the two key words), the last
// round's words complemented so that the kernel's last XOR yields the
// complemented bits directly.
void philox_round_keys(uint64_t seed, uint32_t *k0, uint32_t *k1) {
  uint32_t a = (uint32_t)seed, b = (uint32_t)(seed >> 32);
  for (int r = 0; r < kSrRounds; ++r) {
    k0[r] = r == kSrRounds - 1 ? ~a : a;
    k1[r] = r == kSrRounds - 1 ? ~b : b;
    a += 0x9E3779B9u;
    b += 0xBB67AE85u;
  }
}

// Round-1 constants of sr_bits_not32 from a seed's round keys.
void philox_round1_consts(const uint32_t *k0, const uint32_t *k1, uint32_t *pre_hi, uint32_t *pre_lo) {
  const uint64_t prod = (uint64_t)0xD2511F53u * k0[0];
  *pre_hi = (uint32_t)(prod >> 32) ^ k1[1];
  *pre_lo = (uint32_t)prod;
}

template <int RF, int RR, int CF, int CR, bool H>
cudaError_t launch_q(const CUtensorMap &map, const qk::Params &p, cudaStream_t st) {
  auto kern = qk::quant_kernel<RF, RR, CF, CR, H, false>;
  // stochastic rounding with every linear index below 2^32: 32-bit counters
  if constexpr (RR == kSR || CR == kSR)
    if ((uint64_t)p.T * (uint64_t)p.C < (uint64_t(1) << 32)) kern = qk::quant_kernel<RF, RR, CF, CR, H, true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, qk::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.ntiles < 2 * sms ? p.ntiles : 2 * sms;
  e = launch_pdl(kern, dim3((unsigned)grid), dim3(qk::kThreads), qk::kSmemBytes, st, map, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Dispatch on (row format, row rounding): the column-wise side fixed.
template <int CF, int CR, bool H>
cudaError_t dispatch_row(int rf, int rr, const CUtensorMap &map, const qk::Params &p, cudaStream_t st) {
#define FA4_Q_ROW(F)                                                              \
  if (rf == F) return rr == kSR ? launch_q<F, kSR, CF, CR, H>(map, p, st)       \
                                : launch_q<F, kRNE, CF, CR, H>(map, p, st);
  FA4_Q_ROW(kMX) FA4_Q_ROW(kNVG) FA4_Q_ROW(kNVC) FA4_Q_ROW(kMXN)
#undef FA4_Q_ROW
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_quantize(const QuantArgs &a, cudaStream_t st) {
  qk::Params p = {};
  p.T = a.T;
  p.C = a.C;
  p.tiles_c = (int)((a.C + 127) / 128);
  p.tiles_t = (int)((a.T + 127) / 128);
  p.ntiles = p.tiles_c * p.tiles_t;
  p.rp = a.row_payload;
  p.rs = a.row_scales;
  p.rts = a.row_ts;
  p.cp = a.col_payload;
  p.cs = a.col_scales;
  p.cts = a.col_ts;
  philox_round_keys(a.row_seed, p.rkey0, p.rkey1);
  philox_round_keys(a.col_seed, p.ckey0, p.ckey1);
  philox_round1_consts(p.rkey0, p.rkey1, &p.rpre_hi, &p.rpre_lo);
  philox_round1_consts(p.ckey0, p.ckey1, &p.cpre_hi, &p.cpre_lo);
  for (int t = 0; t < 32; ++t) p.sgn[t] = ((a.sign_mask >> t) & 1u) ? 0x80000000u : 0u;
  p.partials = a.partials;
  p.np = a.n_partials;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  CUtensorMap map;
  if (!make_bf16_tile_map(&map, a.x, a.T, a.C, a.ld)) return cudaErrorInvalidValue;
  const int rf = a.row_fmt, rr = a.row_rnd, cf = a.col_fmt, cr = a.col_rnd;
  using namespace qk;
  if (cf == kNone) return dispatch_row<kNone, kRNE, false>(rf, rr, map, p, st);
  if (rf == kNone) {
    // column-wise only
#define FA4_Q_COL(F, H)                                                              \
  if (cf == F && a.hadamard == H)                                                    \
    return cr == kSR ? launch_q<kNone, kRNE, F, kSR, H>(map, p, st)                  \
                     : launch_q<kNone, kRNE, F, kRNE, H>(map, p, st);
    FA4_Q_COL(kMX, false) FA4_Q_COL(kMX, true) FA4_Q_COL(kNVG, false) FA4_Q_COL(kNVC, false)
    FA4_Q_COL(kMXN, false)
#undef FA4_Q_COL
    return cudaErrorInvalidValue;
  }
  // both orientations: the column-wise operand is MXFP4 (optionally Hadamard)
  if (cf != kMX) return cudaErrorInvalidValue;
  if (a.hadamard)
    return cr == kSR ? dispatch_row<kMX, kSR, true>(rf, rr, map, p, st)
                     : dispatch_row<kMX, kRNE, true>(rf, rr, map, p, st);
  return cr == kSR ? dispatch_row<kMX, kSR, false>(rf, rr, map, p, st)
                   : dispatch_row<kMX, kRNE, false>(rf, rr, map, p, st);
}

namespace {
template <int RF, int RR, int CF, int CR, bool H>
cudaError_t launch_sw(const qk::Params &p, const uint16_t *z, int64_t ld, cudaStream_t st) {
  auto kern = qk::swiglu_quant_kernel<RF, RR, CF, CR, H, false>;
  // stochastic rounding with every linear index below 2^32: 32-bit counters
  if constexpr (RR == kSR || CR == kSR)
    if ((uint64_t)p.T * (uint64_t)p.C < (uint64_t(1) << 32)) kern = qk::swiglu_quant_kernel<RF, RR, CF, CR, H, true>;
  const cudaError_t e = launch_pdl(kern, dim3((unsigned)p.tiles_c, (unsigned)p.tiles_t), dim3(qk::kThreads),
                                   0, st, p, z, ld);
  return e != cudaSuccess ? e : cudaGetLastError();
}
template <int CF, int CR, bool H>
cudaError_t dispatch_sw(int rf, int rr, const qk::Params &p, const uint16_t *z, int64_t ld,
                        cudaStream_t st) {
#define FA4_SW_ROW(F)                                                              \
  if (rf == F) return rr == kSR ? launch_sw<F, kSR, CF, CR, H>(p, z, ld, st)      \
                                : launch_sw<F, kRNE, CF, CR, H>(p, z, ld, st);
  FA4_SW_ROW(kMX) FA4_SW_ROW(kMXN) FA4_SW_ROW(kNVC)
#undef FA4_SW_ROW
  return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_swiglu_quantize(const SwigluArgs &a, cudaStream_t st) {
  qk::Params p = {};
  p.T = a.T;
  p.C = a.F;
  p.tiles_c = (int)((a.F + 127) / 128);
  p.tiles_t = (int)((a.T + 127) / 128);
  p.ntiles = p.tiles_c * p.tiles_t;
  p.rp = a.row_payload;
  p.rs = a.row_scales;
  p.rts = a.row_ts;
  p.cp = a.col_payload;
  p.cs = a.col_scales;
  philox_round_keys(a.row_seed, p.rkey0, p.rkey1);
  philox_round_keys(a.col_seed, p.ckey0, p.ckey1);
  philox_round1_consts(p.rkey0, p.rkey1, &p.rpre_hi, &p.rpre_lo);
  philox_round1_consts(p.ckey0, p.ckey1, &p.cpre_hi, &p.cpre_lo);
  for (int t = 0; t < 32; ++t) p.sgn[t] = ((a.sign_mask >> t) & 1u) ? 0x80000000u : 0u;
  const int rf = a.row_fmt, rr = a.row_rnd, cr = a.col_rnd;
  using qk::kNone;
  if (!a.col) return dispatch_sw<kNone, kRNE, false>(rf, rr, p, a.z, a.ld, st);
  if (a.hadamard)
    return cr == kSR ? dispatch_sw<kMX, kSR, true>(rf, rr, p, a.z, a.ld, st)
                     : dispatch_sw<kMX, kRNE, true>(rf, rr, p, a.z, a.ld, st);
  return cr == kSR ? dispatch_sw<kMX, kSR, false>(rf, rr, p, a.z, a.ld, st)
                   : dispatch_sw<kMX, kRNE, false>(rf, rr, p, a.z, a.ld, st);
}

cudaError_t launch_debug_convert(const float *y, const uint32_t *u16, int64_t n, uint8_t *rne,
                                 uint8_t *sr, uint8_t *e4m3, cudaStream_t st) {
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (n > 0) debug_convert_kernel<<<blocks, 256, 0, st>>>(y, u16, n, rne, sr, e4m3);
  return cudaGetLastError();
}

cudaError_t launch_debug_nv_block_scale(const float *amax, float s_enc, int64_t n, uint8_t *codes,
                                        float *mults, cudaStream_t st) {
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (n > 0) debug_nv_block_scale_kernel<<<blocks, 256, 0, st>>>(amax, s_enc, n, codes, mults);
  return cudaGetLastError();
}

cudaError_t launch_debug_silu(const uint16_t *g, int64_t n, float *out, cudaStream_t st) {
  const unsigned blocks = (unsigned)(((n + 1) / 2 + 255) / 256);
  if (n > 0) debug_silu_kernel<<<blocks, 256, 0, st>>>(g, n, out);
  return cudaGetLastError();
}

cudaError_t launch_debug_sr_bits(uint64_t seed, const uint64_t *idx, int64_t n, uint32_t *bits,
                                 cudaStream_t st) {
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (n > 0) debug_sr_bits_kernel<<<blocks, 256, 0, st>>>(seed, idx, n, bits);
  return cudaGetLastError();
}

}  // namespace fa4
