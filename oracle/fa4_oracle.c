/*
 * fa4_oracle.c -- CPU oracle for FP4 block quantization and the block-scaled
 * FP4 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant generator with the CUDA path and must never be
 * used as a fallback for it.
 *
 * Plain, slow, one element at a time.  Every floating-point step that decides
 * a stored byte is a single IEEE binary32 operation in round-to-nearest-even,
 * in the order written here; the library is compiled with -ffp-contract=off so
 * no multiply-add is fused.  The GEMM accumulates in binary64.
 *
 * Sources (web pages on format-aware fusion for FP4):
 *  [FAF]  "Format-Aware Fusion: The Engineering Practice That Doubles FP4
 *         Pretraining Throughput" -- sections "Why FP4 Speedups Often Remain
 *         Theoretical", "The Design Philosophy of Format-Aware Fusion",
 *         "Two Key Numerical Techniques".
 *  [NVS]  "FP4 Is No Longer Just a Hardware Feature -- The NVFP4 Software Stack
 *         Is Taking Shape" -- sections "NVFP4 is more than a 4-bit value",
 *         "The first change: PyTorch is bringing FP4 packing into compiler
 *         fusion", "The second change: Triton is beginning to measure FP4 as
 *         FP4", "The third change: oneDNN is defining a safe numerical range
 *         for FP4 scales".
 *  [FP4G] "4-Bit Floating Point (FP4) on GPUs: How It Works and When It Pays
 *         Off" -- section "How Does 4-Bit Floating Point Work in Practice?".
 *
 * Where the pages leave a step open, the reading taken is stated at the
 * function.  Parity pins for each function live in tests/test_oracle_*.py.
 *
 * PLANT_* macros: each one, when defined at compile time, introduces one
 * plausible mistake (a wrong tie rule, a swapped nibble, a wrong index...).
 * They are never defined in the library the tests and benchmark use; the
 * planted-mistake tests build separate copies with one macro set and check
 * that the pins catch it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_MXFP4 0
#define ORC_NVFP4_GLOBAL 1
#define ORC_NVFP4_CTA 2
#define ORC_MXFP4_NOCLIP 3
#define ORC_IS_MX(f) ((f) == ORC_MXFP4 || (f) == ORC_MXFP4_NOCLIP)
#define ORC_RNE 0
#define ORC_SR 1

/* ------------------------------------------------------------------------ */
/* bf16 input                                                               */
/* ------------------------------------------------------------------------ */

/* A bf16 value is the upper half of a binary32; widening is exact. */
static float bf16_to_float(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

double orc_bf16_to_double(uint16_t h) { return (double)bf16_to_float(h); }

/* ------------------------------------------------------------------------ */
/* E2M1 element format                                                      */
/* [FP4G "How Does 4-Bit..."], [NVS "NVFP4 is more than a 4-bit value"]:     */
/* 1 sign bit, 2 exponent bits, 1 mantissa bit, sixteen values, max +-6.     */
/* Reading: exponent bias 1 with a subnormal at exponent field 0 -- the only */
/* 1-2-1 layout whose largest finite value is 6.                             */
/* ------------------------------------------------------------------------ */

/* code = s<<3 | e<<1 | m */
double orc_e2m1_decode(int code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

/* magnitude (a grid value) -> 3-bit magnitude code */
static int e2m1_mag_code(double v) {
  for (int c = 0; c < 8; ++c)
    if (orc_e2m1_decode(c) == v) return c;
  return -1; /* unreachable for grid values */
}

/* Spacing of E2M1 values around magnitude a (a < 6): 0.5 below 1 (subnormal
 * range), 2^(E-1) in binade [2^E, 2^(E+1)). */
static double e2m1_quantum(double a) {
  if (a < 1.0) return 0.5;
  int ex;
  frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1): floor(log2 a) = ex - 1 */
  return ldexp(1.0, (ex - 1) - 1);
}

/* Round-to-nearest-even into E2M1 with saturation to +-6.
 * Reading (the pages say only "rounded into the E2M1 range",
 * [NVS "The first change"]): IEEE round-half-to-even on the E2M1 grid, values
 * of magnitude >= 6 saturate to 6, the sign is kept (a negative value that
 * rounds to zero gives code 0x8). */
int orc_e2m1_rne(float y) {
  int s = signbit(y) ? 1 : 0;
  double a = fabs((double)y);
  int mc;
  if (a >= 6.0) {
    mc = 7;
  } else {
    double q = e2m1_quantum(a);
#ifdef PLANT_TIE_AWAY
    double n = round(a / q);
#else
    double n = rint(a / q); /* a/q exact (q is a power of two); rint = half-even */
#endif
    double v = n * q;
    if (v > 6.0) v = 6.0;
    mc = e2m1_mag_code(v);
  }
  return (s << 3) | mc;
}

/* Stochastic rounding into E2M1 with 16 random bits.
 * [FAF "Two Key Numerical Techniques"]: round up or down with a probability
 * set by the distance, so that the expectation equals the input.
 * Reading: lo <= |y| < hi are the neighbouring grid values, g = hi - lo, the
 * fraction f = (|y| - lo)/g is exact in binary32 (g is a power of two); with
 * t = f * 65536 the value rounds up iff u16 < floor(t), i.e. for floor(t) of
 * the 65536 draws (bias below g/65536).  |y| >= 6 gives 6.  Sign kept. */
int orc_e2m1_sr(float y, uint32_t u16) {
  int s = signbit(y) ? 1 : 0;
  float a = fabsf(y);
  int mc;
  if (a >= 6.0f) {
    mc = 7;
  } else {
    double q = e2m1_quantum((double)a);
    double lo = floor((double)a / q) * q;
    float f = (a - (float)lo) / (float)q;  /* both exact */
    float t = f * 65536.0f;                /* exact */
    /* round up iff u < floor(t): the integer part of t is the number of
     * the 65536 draws that round up (P(up) = floor(t) / 65536) */
#ifdef PLANT_SR_LE
    int up = ((float)(u16 & 0xFFFFu) <= floorf(t)) ? 1 : 0;
#elif defined(PLANT_SR_NOFLOOR)
    int up = ((float)(u16 & 0xFFFFu) < t) ? 1 : 0;
#else
    int up = ((float)(u16 & 0xFFFFu) < floorf(t)) ? 1 : 0;
#endif
    double v = up ? lo + q : lo;
    mc = e2m1_mag_code(v);
  }
  return (s << 3) | mc;
}

/* ------------------------------------------------------------------------ */
/* E4M3 block scale (NVFP4) [NVS "NVFP4 is more than a 4-bit value"]:        */
/* FP8 E4M3, bias 7, 3 mantissa bits, largest finite 448 (0x7E), 0x7F NaN,   */
/* subnormals m * 2^-9 at exponent field 0.  Unsigned use only here.         */
/* ------------------------------------------------------------------------ */

double orc_e4m3_decode(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = ldexp((double)m, -9);
  else mag = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

/* Round-to-nearest-even into E4M3, saturating to 448 (never NaN). */
int orc_e4m3_rne(float v) {
  int s = signbit(v) ? 1 : 0;
  double a = fabs((double)v);
  if (a >= 448.0) return (s << 7) | 0x7E;
  double q;
  if (a < ldexp(1.0, -6)) {
    q = ldexp(1.0, -9); /* subnormal spacing */
  } else {
    int ex;
    frexp(a, &ex);
    q = ldexp(1.0, (ex - 1) - 3);
  }
  double r = rint(a / q) * q;
  if (r > 448.0) r = 448.0;
  for (int c = 0; c < 0x7F; ++c)
    if (orc_e4m3_decode(c) == r) return (s << 7) | c;
  return -1;
}

/* ------------------------------------------------------------------------ */
/* MXFP4 scale: 32-value block, power-of-two E8M0 scale.                     */
/* [FAF "The Design Philosophy..."] names "native mxfp".  Reading: the OCP   */
/* MX rule -- the shared exponent is floor(log2 amax) minus the largest      */
/* element exponent of E2M1 (2), clamped to the E8M0 range [-127, 127];      */
/* amax = 0 gives -127.  Stored byte = exponent + 127.                       */
/* ------------------------------------------------------------------------ */

int orc_mx_exponent(float amax) {
  if (!(amax > 0.0f)) return -127;
  int ex;
  frexpf(amax, &ex); /* exact for normals and subnormals */
#ifdef PLANT_MX_EMAX
  int e = (ex - 1) - 1;
#else
  int e = (ex - 1) - 2;
#endif
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* MXFP4 without clipping: the smallest e with amax <= 6 * 2^e (so no element
 * of the block saturates), clamped to [-127, 127]; amax = 0 gives -127.
 * With amax = m * 2^E, 1 <= m < 2: e = E - 2 when m <= 1.5, else E - 1. */
int orc_mx_exponent_noclip(float amax) {
  if (!(amax > 0.0f)) return -127;
  int ex;
  float fr = frexpf(amax, &ex); /* amax = fr * 2^ex, 0.5 <= fr < 1 */
  int E = ex - 1;                /* m = 2 fr */
#ifdef PLANT_MX_NOCLIP_FLOOR
  int e = E - 2; /* the clipping rule's exponent */
  (void)fr;
#else
  int e = (2.0f * fr <= 1.5f) ? E - 2 : E - 1;
#endif
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 scales [NVS "NVFP4 is more than a 4-bit value"]: one E4M3 scale per */
/* 16 values and one FP32 second-level scale; value = e2m1 * block scale *    */
/* second-level scale.  Guardrail [NVS "The third change"]: the dynamic      */
/* scale is clamped to [smallest positive of the scale type, largest].       */
/* Readings: encode scale s_enc = 2688/amax_t (6 * 448, so the largest block  */
/* scale lands at E4M3 max), s_enc = 1 when amax_t is 0 or the quotient is   */
/* not finite; stored decode scale ts = 1/s_enc; block scale                 */
/* s_b = (amax_b/6) * s_enc clamped to [2^-9, 448], cast to E4M3 (RNE);      */
/* element multiplier r_b = s_enc / decode(code_b).  All binary32.           */
/* ------------------------------------------------------------------------ */

float orc_nv_encode_scale(float amax_t) {
  float s = 2688.0f / amax_t;
  if (amax_t == 0.0f || !isfinite(s)) s = 1.0f;
  return s;
}

float orc_nv_decode_scale(float s_enc) { return 1.0f / s_enc; }

/* returns the E4M3 code of the block scale; *mult receives r_b */
int orc_nv_block_scale(float amax_b, float s_enc, float *mult) {
#ifdef PLANT_NV_NO_SENC
  float sb = amax_b / 6.0f;
#else
  float sb = amax_b / 6.0f;
  sb = sb * s_enc;
#endif
  const float lo = 0.001953125f; /* 2^-9, smallest positive E4M3 */
  if (!(sb >= lo)) sb = lo;
  if (sb > 448.0f) sb = 448.0f;
  int code = orc_e4m3_rne(sb);
  float sv = (float)orc_e4m3_decode(code);
  *mult = s_enc / sv;
  return code;
}

/* ------------------------------------------------------------------------ */
/* Counter-based random numbers: Philox4x32 (Salmon, Moraes, Dror, Shaw,     */
/* "Parallel random numbers: as easy as 1, 2, 3", SC'11).  The pages name no */
/* generator; this choice and the element-to-bits mapping are readings.      */
/* ------------------------------------------------------------------------ */

static void mulhilo32(uint32_t a, uint32_t b, uint32_t *hi, uint32_t *lo) {
  uint64_t p = (uint64_t)a * (uint64_t)b;
  *hi = (uint32_t)(p >> 32);
  *lo = (uint32_t)p;
}

void orc_philox4x32(const uint32_t ctr_in[4], const uint32_t key_in[2], int rounds,
                    uint32_t out[4]) {
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int r = 0; r < rounds; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u; /* Weyl key schedule */
      k1 += 0xBB67AE85u;
    }
    uint32_t hi0, lo0, hi1, lo1;
    mulhilo32(0xD2511F53u, c0, &hi0, &lo0);
    mulhilo32(0xCD9E8D57u, c2, &hi1, &lo1);
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    uint32_t n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Rounds of the Philox block behind the stochastic-rounding bits.  The
 * pages fix no generator, only that the rounding is unbiased; Philox4x32 is
 * the published counter-based family, and its authors report 7 rounds
 * already passing their full statistical test batteries (10 is their
 * default with a safety margin).  7 rounds: the bits are uniform, so the
 * rounding stays unbiased, at 70% of the ten-round cost. */
#define ORC_SR_ROUNDS 7
int orc_sr_rounds(void) { return ORC_SR_ROUNDS; }

/* 16 random bits for element i (linear index in the quantized orientation):
 * one Philox4x32 block (ORC_SR_ROUNDS rounds) per 8 elements, counter =
 * (i>>3) as a 64-bit value in words 0-1, key = the 64-bit seed; word
 * (i>>1)&3, low half for even i and high half for odd i. */
uint32_t orc_sr_bits(uint64_t seed, uint64_t i) {
  uint32_t ctr[4] = {(uint32_t)(i >> 3), (uint32_t)(i >> 35), 0u, 0u};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  orc_philox4x32(ctr, key, ORC_SR_ROUNDS, out);
  uint32_t w = out[(i >> 1) & 3];
  return (i & 1) ? (w >> 16) : (w & 0xFFFFu);
}

/* ------------------------------------------------------------------------ */
/* Scale-factor storage in the layout the block-scaled tensor-core GEMM      */
/* reads ([NVS "The second change"]: "logical rows in swizzled storage";     */
/* [FAF "The Design Philosophy..."]: consumer layout).  Reading: 128-row x   */
/* 4-block atoms of 512 bytes; atoms ordered along the block (K) dimension   */
/* first; inside an atom row r sits at (r%32)*16 + ((r%128)/32)*4 and block  */
/* kb at kb%4.                                                               */
/* ------------------------------------------------------------------------ */

int64_t orc_sf_offset(int64_t r, int64_t kb, int64_t kb_total) {
  int64_t kb_pad = (kb_total + 3) / 4 * 4;
  int64_t atom = (r / 128) * (kb_pad / 4) + kb / 4;
#ifdef PLANT_SWIZZLE
  return atom * 512 + (r % 32) * 4 + ((r % 128) / 32) * 128 + (kb % 4);
#else
  return atom * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (kb % 4);
#endif
}

int64_t orc_sf_bytes(int64_t rows, int64_t kb_total) {
  return (rows + 127) / 128 * 128 * ((kb_total + 3) / 4 * 4);
}

/* ------------------------------------------------------------------------ */
/* Fixed-sign 32-point Hadamard [FAF "Two Key Numerical Techniques"]:        */
/* a 32x32 Hadamard with a fixed sign pattern, applied to weight-gradient    */
/* operands.  Readings: Sylvester matrix H[i][j] = (-1)^popcount(i&j),       */
/* unnormalised (H H^T = 32 I); y = H (s .* x) with s_j = -1 iff bit j of    */
/* sign_mask; computed as the in-place butterfly with strides 1,2,4,8,16,    */
/* (a, b) -> (a + b, a - b), one binary32 add per output.                    */
/* ------------------------------------------------------------------------ */

void orc_hadamard32(const float *x, uint32_t sign_mask, float *y) {
  float v[32];
#ifdef PLANT_HAD_SIGN_AFTER
  for (int j = 0; j < 32; ++j) v[j] = x[j];
#else
  for (int j = 0; j < 32; ++j) v[j] = ((sign_mask >> j) & 1u) ? -x[j] : x[j];
#endif
  for (int h = 1; h < 32; h <<= 1) {
    for (int i = 0; i < 32; ++i) {
      if (i & h) continue;
      float a = v[i], b = v[i + h];
      v[i] = a + b;
      v[i + h] = a - b;
    }
  }
#ifdef PLANT_HAD_SIGN_AFTER
  for (int j = 0; j < 32; ++j) y[j] = ((sign_mask >> j) & 1u) ? -v[j] : v[j];
#else
  for (int j = 0; j < 32; ++j) y[j] = v[j];
#endif
}

/* ------------------------------------------------------------------------ */
/* Quantization [NVS "The first change"]: block amax -> scale -> divide by    */
/* the scale -> E2M1 -> two values per byte.                                 */
/*                                                                          */
/* The quantized operand Q[R, K] is read from the bf16 input x (leading      */
/* dimension ld elements):                                                  */
/*   orient 0 (row-wise):    Q[r][k] = x[r*ld + k],  R = rows, K = cols      */
/*   orient 1 (column-wise): Q[r][k] = x[k*ld + r],  R = cols, K = rows      */
/* Outputs: payload[R][K/2] with byte = code(2j) | code(2j+1) << 4 (reading: */
/* the even element in the low nibble; [NVS "The first change"] pairs even   */
/* and odd elements); scale bytes at orc_sf_offset; ts = FP32 decode scales  */
/* (1 for NVFP4-global, [R/128][K/128] for NVFP4-CTA-local, none for MX).    */
/* NVFP4-CTA-local [FAF "The Design Philosophy..."] takes the second-level   */
/* amax over the 128x128 tile of Q that holds the block (reading; the pages  */
/* name only "CTA-local nvfp"); tiles at a ragged edge (R or K not a        */
/* multiple of 128) hold fewer values and take the amax of those, so ts is  */
/* [ceil(R/128)][ceil(K/128)].  R may be any positive count; K must be a    */
/* multiple of the block size (32 MX, 16 NV).                               */
/* hadamard: apply orc_hadamard32 to each 32-value block before the scale    */
/* (MXFP4 only).  SR bits use i = r*K + k.  Only rows [r_begin, r_end) of Q  */
/* are produced (all when r_end <= 0), for sampled checks of large tensors.  */
/* Returns 0 on success, -1 on an unsupported combination.                   */
/* ------------------------------------------------------------------------ */

static float q_elem(const uint16_t *x, int64_t ld, int orient, int64_t r, int64_t k) {
  return orient == 0 ? bf16_to_float(x[r * ld + k]) : bf16_to_float(x[k * ld + r]);
}

static void put_code(uint8_t *payload, int64_t K, int64_t r, int64_t k, int code) {
  uint8_t *b = &payload[r * (K / 2) + k / 2];
#ifdef PLANT_NIBBLE_SWAP
  k ^= 1;
#endif
  if ((k & 1) == 0) *b = (uint8_t)((*b & 0xF0) | (code & 0xF));
  else *b = (uint8_t)((*b & 0x0F) | ((code & 0xF) << 4));
}

int orc_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int fmt, int rnd,
                 int orient, uint64_t seed, int hadamard, uint32_t sign_mask, uint8_t *payload,
                 uint8_t *scales, float *ts, int64_t r_begin, int64_t r_end) {
  int64_t R = orient == 0 ? rows : cols;
  int64_t K = orient == 0 ? cols : rows;
  int bs = ORC_IS_MX(fmt) ? 32 : 16;
  if (hadamard && fmt != ORC_MXFP4) return -1;
  if (K % bs != 0 || (K & 1)) return -1;
  int64_t kb_total = K / bs;
  memset(scales, 0, (size_t)orc_sf_bytes(R, kb_total));
  memset(payload, 0, (size_t)(R * (K / 2)));

  /* second-level amax for NVFP4: one encode scale for the tensor (global) or
     one per 128x128 tile of Q (CTA-local) */
  int64_t n_tk = (K + 127) / 128;
  int64_t n_tiles = (fmt == ORC_NVFP4_CTA) ? (R + 127) / 128 * n_tk : 1;
  float *s_enc = (float *)malloc(sizeof(float) * (size_t)n_tiles);
  if (!s_enc) return -2;
  s_enc[0] = 1.0f;
  if (fmt == ORC_NVFP4_GLOBAL) {
    float amax_t = 0.0f;
    for (int64_t r = 0; r < R; ++r)
      for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(q_elem(x, ld, orient, r, k));
        if (a > amax_t) amax_t = a;
      }
    s_enc[0] = orc_nv_encode_scale(amax_t);
    ts[0] = orc_nv_decode_scale(s_enc[0]);
  }
  if (fmt == ORC_NVFP4_CTA) {
    for (int64_t tr = 0; tr < (R + 127) / 128; ++tr)
      for (int64_t tk = 0; tk < n_tk; ++tk) {
        float amax_t = 0.0f;
        for (int64_t r = tr * 128; r < tr * 128 + 128 && r < R; ++r)
          for (int64_t k = tk * 128; k < tk * 128 + 128 && k < K; ++k) {
            float a = fabsf(q_elem(x, ld, orient, r, k));
            if (a > amax_t) amax_t = a;
          }
        s_enc[tr * n_tk + tk] = orc_nv_encode_scale(amax_t);
        ts[tr * n_tk + tk] = orc_nv_decode_scale(s_enc[tr * n_tk + tk]);
      }
  }

  /* rows of Q to produce: [r_begin, r_end) (all rows when r_end <= 0); the
     second-level scales above always cover the whole operand */
  if (r_end <= 0 || r_end > R) r_end = R;
  if (r_begin < 0) r_begin = 0;
  float v[32];
  for (int64_t r = r_begin; r < r_end; ++r) {
    for (int64_t kb = 0; kb < kb_total; ++kb) {
      for (int j = 0; j < bs; ++j) v[j] = q_elem(x, ld, orient, r, kb * bs + j);
      if (hadamard) {
        float h[32];
        orc_hadamard32(v, sign_mask, h);
        for (int j = 0; j < 32; ++j) v[j] = h[j];
      }
      /* block amax (max is exact) */
      float amax_b = 0.0f;
      for (int j = 0; j < bs; ++j)
        if (fabsf(v[j]) > amax_b) amax_b = fabsf(v[j]);
      uint8_t sbyte;
      int mx_e = 0;
      float mult = 1.0f; /* NVFP4: y = v * mult */
      if (ORC_IS_MX(fmt)) {
        mx_e = (fmt == ORC_MXFP4) ? orc_mx_exponent(amax_b) : orc_mx_exponent_noclip(amax_b);
        sbyte = (uint8_t)(mx_e + 127);
      } else {
        float se = (fmt == ORC_NVFP4_CTA) ? s_enc[(r / 128) * n_tk + (kb * bs) / 128] : s_enc[0];
        sbyte = (uint8_t)orc_nv_block_scale(amax_b, se, &mult);
      }
      scales[orc_sf_offset(r, kb, kb_total)] = sbyte;
      for (int j = 0; j < bs; ++j) {
        int64_t k = kb * bs + j;
        /* MXFP4: exact multiplication by 2^-e; NVFP4: one binary32 multiply */
        float y = ORC_IS_MX(fmt) ? ldexpf(v[j], -mx_e) : v[j] * mult;
        int code;
        if (rnd == ORC_SR) code = orc_e2m1_sr(y, orc_sr_bits(seed, (uint64_t)(r * K + k)));
        else code = orc_e2m1_rne(y);
        put_code(payload, K, r, k, code);
      }
    }
  }
  free(s_enc);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Dequantization: value = e2m1(code) * block scale [* second-level scale].  */
/* Writes binary64 q[R][K] WITHOUT the second-level scale (that factor is    */
/* applied by the GEMM per tile, so that the block sums stay exact).         */
/* ------------------------------------------------------------------------ */

int orc_dequantize_blocks(const uint8_t *payload, const uint8_t *scales, int64_t R, int64_t K,
                          int fmt, const int64_t *row_idx, int64_t n_rows, double *out) {
  int bs = ORC_IS_MX(fmt) ? 32 : 16;
  int64_t kb_total = K / bs;
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t r = row_idx ? row_idx[i] : i;
    if (r < 0 || r >= R) return -1;
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = payload[r * (K / 2) + k / 2];
      int code = (k & 1) ? (byte >> 4) : (byte & 0xF);
      uint8_t sb = scales[orc_sf_offset(r, k / bs, kb_total)];
      double scale = ORC_IS_MX(fmt) ? ldexp(1.0, (int)sb - 127) : orc_e4m3_decode(sb);
      out[i * K + k] = orc_e2m1_decode(code) * scale;
    }
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Block-scaled GEMM: D[m][n] = alpha * sum_k A[m][k] * B[n][k], A and B     */
/* given as quantized operands (both K-major).  binary64 accumulation:       */
/* with E2M1 codes and E8M0/E4M3 block scales every product has at most 12   */
/* significant bits, so the block sums are exact.  NVFP4-global multiplies    */
/* by ts_A*ts_B; NVFP4-CTA-local multiplies each 128-wide K chunk by         */
/* ts_A[m/128][kc] * ts_B[n/128][kc] (the last chunk ends at K when K is    */
/* not a multiple of 128).  Computes the rows/columns listed in              */
/* m_idx/n_idx (all when NULL); out is [n_m][n_n] row-major.                 */
/* ------------------------------------------------------------------------ */

int orc_gemm(const uint8_t *pa, const uint8_t *sa, const float *tsa, const uint8_t *pb,
             const uint8_t *sb, const float *tsb, int64_t M, int64_t N, int64_t K, int fmt,
             double alpha, const int64_t *m_idx, int64_t n_m, const int64_t *n_idx, int64_t n_n,
             double *out) {
  double *arow = (double *)malloc(sizeof(double) * (size_t)K);
  double *brow = (double *)malloc(sizeof(double) * (size_t)K);
  if (!arow || !brow) {
    free(arow);
    free(brow);
    return -2;
  }
  int64_t nk = (K + 127) / 128;
  for (int64_t i = 0; i < n_m; ++i) {
    int64_t m = m_idx ? m_idx[i] : i;
    if (m < 0 || m >= M || orc_dequantize_blocks(pa, sa, M, K, fmt, &m, 1, arow) != 0) {
      free(arow);
      free(brow);
      return -1;
    }
    for (int64_t j = 0; j < n_n; ++j) {
      int64_t n = n_idx ? n_idx[j] : j;
      if (n < 0 || n >= N || orc_dequantize_blocks(pb, sb, N, K, fmt, &n, 1, brow) != 0) {
        free(arow);
        free(brow);
        return -1;
      }
      double d;
      if (fmt == ORC_NVFP4_CTA) {
        d = 0.0;
        for (int64_t kc = 0; kc < nk; ++kc) {
          double s = 0.0;
          for (int64_t k = kc * 128; k < kc * 128 + 128 && k < K; ++k) s += arow[k] * brow[k];
#ifdef PLANT_CTA_TILE_INDEX
          d += (double)tsa[(m / 128) * nk + kc] * (double)tsb[(m / 128) * nk + kc] * s;
#else
          d += (double)tsa[(m / 128) * nk + kc] * (double)tsb[(n / 128) * nk + kc] * s;
#endif
        }
      } else {
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k) s += arow[k] * brow[k];
#ifdef PLANT_GEMM_DROP_TS
        (void)tsb;
#else
        if (fmt == ORC_NVFP4_GLOBAL) s = s * ((double)tsa[0] * (double)tsb[0]);
#endif
        d = s;
      }
      out[i * n_n + j] = alpha * d;
    }
  }
  free(arow);
  free(brow);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* SwiGLU producer of the down projection's input.  [FAF] "The Design        */
/* Philosophy of Format-Aware Fusion" binds each quantization producer to    */
/* its consumer; the activation h = silu(g) * u of a gated MLP is the        */
/* producer of the down projection's input.  The pages give no numerics for  */
/* it.  Reading: binary32 arithmetic, one rounding to bf16 at the end (the   */
/* activation an unfused pipeline stores), silu(g) = g / (1 + exp(-g)), and  */
/* exp written out step by step so that every implementation of the path     */
/* computes the same bits:                                                    */
/*   clamp x to [-87, 88] (so 2^n below stays a normal scale);              */
/*   n = rint(x * RN(log2 e));                                                */
/*   r = x - n ln2 in two fused steps with ln2 = LN2_HI + LN2_LO, LN2_HI     */
/*       having 15 significant bits (Cody and Waite, "Software Manual for    */
/*       the Elementary Functions", 1980: the additive range reduction);    */
/*   p = the degree-6 Taylor polynomial of e^r (|r| <= ln2 / 2), Horner      */
/*       with fused multiply-adds from 1/720 down;                            */
/*   exp(x) = p * 2^n.                                                         */
/* Every step is one IEEE binary32 operation (fmaf: one rounding).           */
/* ------------------------------------------------------------------------ */

float orc_exp_f32(float x) {
  if (x < -87.0f) x = -87.0f;
  if (x > 88.0f) x = 88.0f;
  const float n = rintf(x * 1.44269502162933349609375f); /* RN(log2 e) */
  float r = fmaf(-n, 0.693145751953125f, x);             /* LN2_HI */
  r = fmaf(-n, 1.42860677e-6f, r);                       /* LN2_LO = RN(ln2 - LN2_HI) */
  float p = 1.38888892e-3f;                              /* RN(1/720) */
  p = fmaf(p, r, 8.33333377e-3f);                        /* RN(1/120) */
  p = fmaf(p, r, 4.16666679e-2f);                        /* RN(1/24) */
  p = fmaf(p, r, 1.66666672e-1f);                        /* RN(1/6) */
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  const uint32_t sbits = (uint32_t)((int)n + 127) << 23;
  float scale;
  memcpy(&scale, &sbits, sizeof(scale));
  return p * scale;
}

float orc_silu_f32(float g) { return g / (1.0f + orc_exp_f32(-g)); }

/* binary32 -> bf16, round to nearest even (finite values) */
static uint16_t float_to_bf16_rne(float v) {
  uint32_t b;
  memcpy(&b, &v, sizeof(b));
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

/* h[T, F] (bf16 bits) from z[T, 2F] (bf16 bits, row stride ld): gate =
 * z[t][f], up = z[t][F + f]; h = bf16(silu(gate) * up). */
#ifdef PLANT_SWIGLU_SWAP
#define ORC_GATE(z, t, f) bf16_to_float(z[(t) * ld + F + (f)])
#define ORC_UP(z, t, f) bf16_to_float(z[(t) * ld + (f)])
#else
#define ORC_GATE(z, t, f) bf16_to_float(z[(t) * ld + (f)])
#define ORC_UP(z, t, f) bf16_to_float(z[(t) * ld + F + (f)])
#endif
void orc_swiglu_bf16(const uint16_t *z, int64_t T, int64_t F, int64_t ld, uint16_t *h) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t f = 0; f < F; ++f)
      h[t * F + f] = float_to_bf16_rne(orc_silu_f32(ORC_GATE(z, t, f)) * ORC_UP(z, t, f));
}

void orc_exp_f32_batch(const float *x, int64_t n, float *y) {
  for (int64_t i = 0; i < n; ++i) y[i] = orc_exp_f32(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Batch helpers for the tests (plain loops over the scalar rules above).    */
/* ------------------------------------------------------------------------ */

void orc_e2m1_rne_batch(const float *y, int64_t n, uint8_t *codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)orc_e2m1_rne(y[i]);
}

void orc_e2m1_sr_batch(const float *y, const uint32_t *u16, int64_t n, uint8_t *codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)orc_e2m1_sr(y[i], u16[i]);
}

void orc_e4m3_rne_batch(const float *v, int64_t n, uint8_t *codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)orc_e4m3_rne(v[i]);
}

void orc_sr_bits_batch(uint64_t seed, const uint64_t *idx, int64_t n, uint32_t *bits) {
  for (int64_t i = 0; i < n; ++i) bits[i] = orc_sr_bits(seed, idx[i]);
}
