/*
 * tf4_oracle.c -- plain, slow, obviously-correct CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY (see tf4_oracle.h for who may use it and for
 * the pages each definition follows).  Built with -O2 -ffp-contract=off so
 * that every float expression below is one IEEE binary32 operation with
 * round-to-nearest-even, exactly as written.
 *
 * Exactness notes used throughout:
 *  - a bf16 value has at most 8 significant bits, an fp32 scale S at most
 *    24, and every codeword or midpoint of either grid (E2M1, uniform) is
 *    k/4 with k < 32, so a product (codeword or midpoint) * S is exact in
 *    double (<= 29 bits);
 *  - every decision below is a comparison between two such exact doubles,
 *    never a comparison of a rounded quotient; "y = |x| / S" is the real
 *    quotient, compared through |x| vs c*S.
 */
#include "tf4_oracle.h"

#include <math.h>
#include <string.h>

/* E2M1 magnitudes indexed by m3 = exponent(2 bits)<<1 | mantissa(1 bit).
 * [FQT] section 3: E2M1 = 2-bit exponent, 1-bit mantissa. */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Uniform 4-bit grid ([UFP4] design section: E1M2 / INT4): magnitudes
 * 0..7 in steps of one, indexed by the same 3-bit magnitude code.  (E1M2's
 * grid is this one divided by 4; with the tensor scale defined from the
 * grid maximum the two give the same codes and scale bytes.) */
static const double kUniform[8] = {0.0, 1.0, 2.0, 3.0, 4.0, 5.0, 6.0, 7.0};

static const double* grid_of(int fmt) { return fmt == ORC_UFP4 ? kUniform : kE2M1; }
static int block_of(int fmt) { return fmt == ORC_MXFP4 ? 32 : 16; }
static int has_tensor_scale(int fmt) { return fmt != ORC_MXFP4; }

float orc_bf16_to_float(uint16_t h) {
  uint32_t u = (uint32_t)h << 16; /* bf16 is the top half of an fp32 */
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

static int bf16_is_finite(uint16_t h) { return (h & 0x7F80u) != 0x7F80u; }
static int bf16_sign(uint16_t h) { return (h >> 15) & 1; }
static double bf16_abs(uint16_t h) { return (double)orc_bf16_to_float((uint16_t)(h & 0x7FFFu)); }

double orc_e2m1_value(int m3) { return kE2M1[m3 & 7]; }
double orc_grid_value(int fmt, int m3) { return grid_of(fmt)[m3 & 7]; }

/* E4M3 ("fn" variant: no infinities, 0x7F/0xFF are NaN): bias 7,
 * subnormals m * 2^-9, largest finite 448 (0x7E).  [FQT] section 3 names
 * E4M3 as the NVFP4 block-scale format. */
double orc_e4m3_value(uint8_t code) {
  int sign = code >> 7, e = (code >> 3) & 0xF, m = code & 7;
  double v;
  if (e == 0xF && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -v : v;
}

/* Round a non-negative finite fp32 to E4M3: the nearest of the 127
 * non-negative finite codes, ties to the even code (even mantissa),
 * anything above 448 saturates to 448.  Plain search over all codes. */
uint8_t orc_e4m3_encode(float r) {
  double rv = (double)r;
  int best = 0;
  for (int c = 1; c <= 0x7E; ++c) {
    double vb = orc_e4m3_value((uint8_t)best), vc = orc_e4m3_value((uint8_t)c);
    double db = fabs(rv - vb), dc = fabs(rv - vc); /* exact: both near rv, few bits */
    if (dc < db || (dc == db && (c & 1) == 0)) best = c;
  }
  return (uint8_t)best;
}

/* MXFP4 shared exponent: floor(log2(bamax)) - 2, clamped to the E8M0
 * range [-127, 127]; an all-zero block takes -127.  [TETRAJET] section 3
 * (per-group scale).  floor(log2) is read exactly from frexp. */
int orc_e8m0_exponent(float bamax) {
  int ex;
  if (bamax == 0.0f) return -127;
  (void)frexp((double)bamax, &ex); /* bamax = f * 2^ex, f in [0.5, 1) */
  int e = (ex - 1) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* Per-tensor scale s_t = amax / (grid max * 448) in fp32: 2688 = 6 * 448
 * for NVFP4, 3136 = 7 * 448 for the uniform grid.  A result below the
 * smallest normal fp32 (including amax == 0) makes the whole segment
 * quantize to signed zeros with s_t = 0. */
float orc_tensor_scale(int fmt, float amax) {
  float s = amax / (fmt == ORC_UFP4 ? 3136.0f : 2688.0f);
  if (!(s >= 0x1p-126f)) s = 0.0f;
  return s;
}

float orc_nvfp4_tensor_scale(float amax) { return orc_tensor_scale(ORC_NVFP4, amax); }

/* E4M3 block scale code: b = E4M3( (bamax / grid max) / s_t ), two fp32
 * divides in that order (grid max 6 for NVFP4, 7 for the uniform grid);
 * s_t == 0 gives 0. */
uint8_t orc_block_scale_code(int fmt, float bamax, float s_t) {
  if (s_t == 0.0f) return 0;
  float q = bamax / (fmt == ORC_UFP4 ? 7.0f : 6.0f);
  float r = q / s_t;
  return orc_e4m3_encode(r);
}

uint8_t orc_nvfp4_block_scale_code(float bamax, float s_t) { return orc_block_scale_code(ORC_NVFP4, bamax, s_t); }

/* Effective block scale S = s_t * dec(b), one fp32 multiply. */
float orc_nvfp4_block_scale(uint8_t code, float s_t) {
  float d = (float)orc_e4m3_value(code);
  return s_t * d;
}

float orc_mxfp4_block_scale(uint8_t code) { return (float)ldexp(1.0, (int)code - 127); }

/* Round-to-nearest: the codeword nearest to y = ax / S (real quotient),
 * ties to the even m3; saturation at the grid maximum is the
 * nearest-codeword rule itself.  [TRACE-JA] mismatch section: plain
 * nearest rounding is what the rollout does; [FQT] section 3:
 * round-to-nearest in the forward pass.
 * Scan the sorted grid; codeword j beats the current best b (< j) iff y is
 * above their midpoint, i.e. 2*ax > (V_b + V_j) * S (both sides exact). */
static int rtn_on(const double* V, double ax, double S) {
  if (S == 0.0) return 0;
  int best = 0;
  for (int j = 1; j < 8; ++j) {
    double lhs = 2.0 * ax, rhs = (V[best] + V[j]) * S;
    if (lhs > rhs || (lhs == rhs && (j % 2) == 0)) best = j;
  }
  return best;
}

/* Neighbours of y = ax / S on the grid (S > 0, y below the grid maximum,
 * y not a codeword): lo = the largest j with V_j * S < ax. */
static int grid_floor(const double* V, double ax, double S) {
  int lo = 0;
  for (int j = 1; j < 8; ++j)
    if (V[j] * S < ax) lo = j;
  return lo;
}

/* Index of the codeword equal to y, or -1. */
static int grid_exact(const double* V, double ax, double S) {
  for (int j = 0; j < 8; ++j)
    if (V[j] * S == ax) return j;
  return -1;
}

/* Stochastic rounding with a 24-bit uniform integer r: between the two
 * neighbours lo < y < hi round up iff r < 2^24 (y - lo) / (hi - lo), i.e.
 * r * (V_hi - V_lo) * S < 2^24 * (ax - V_lo * S).  Left side: <= 48 bits;
 * right side: ax and V_lo*S within a factor 2 (or V_lo = 0; on the uniform
 * grid ax - V_lo*S is a multiple of ulp(S) below S), so the difference is
 * exact -- both sides exact in double.
 * y >= grid max saturates; a codeword keeps itself.  [FQT] section 3. */
static int sr_on(const double* V, double ax, double S, uint32_t r24) {
  if (S == 0.0) return 0;
  if (ax >= V[7] * S) return 7;
  int ex = grid_exact(V, ax, S);
  if (ex >= 0) return ex;
  int lo = grid_floor(V, ax, S), hi = lo + 1;
  double lhs = (double)r24 * (V[hi] - V[lo]) * S;
  double rhs = 16777216.0 * (ax - V[lo] * S);
  return lhs < rhs ? hi : lo;
}

/* Rollout-guided rounding: of the two grid neighbours of y, take the one
 * whose mantissa bit (m3 & 1) equals the recorded bit g.  Adjacent
 * codewords always differ in that bit (on E2M1 and on the uniform grid), so
 * exactly one qualifies.  A value that is a codeword keeps it; y at or
 * above the grid maximum gives the maximum (both neighbours are it).
 * [TRACE-JA] mechanism section (the candidates are the two adjacent
 * codewords, chosen by a light comparison) and quantization-info cache
 * section (mantissa bit + scale identify the codeword). */
static int guided_on(const double* V, double ax, double S, int g) {
  if (S == 0.0) return 0;
  if (ax >= V[7] * S) return 7;
  int ex = grid_exact(V, ax, S);
  if (ex >= 0) return ex;
  int lo = grid_floor(V, ax, S), hi = lo + 1;
  return ((lo & 1) == (g & 1)) ? lo : hi;
}

int orc_rtn_m3(double ax, double S) { return rtn_on(kE2M1, ax, S); }
int orc_sr_m3(double ax, double S, uint32_t r24) { return sr_on(kE2M1, ax, S, r24); }
int orc_guided_m3(double ax, double S, int g) { return guided_on(kE2M1, ax, S, g); }
int orc_rtn_code(int fmt, double ax, double S) { return rtn_on(grid_of(fmt), ax, S); }
int orc_sr_code(int fmt, double ax, double S, uint32_t r24) { return sr_on(grid_of(fmt), ax, S, r24); }
int orc_guided_code(int fmt, double ax, double S, int g) { return guided_on(grid_of(fmt), ax, S, g); }

/* Philox4x32-10 [PHILOX]: 10 rounds of the 4x32 Philox S-box; between
 * rounds the 2-word key is bumped by the Weyl constants.  One round:
 *   (hi0, lo0) = M0 * c0,  (hi1, lo1) = M1 * c2   (full 64-bit products)
 *   c' = (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0)                        */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += W0;
      k1 += W1;
    }
    uint64_t p0 = (uint64_t)M0 * c0, p1 = (uint64_t)M1 * c2;
    uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    uint32_t n1 = (uint32_t)p1;
    uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    uint32_t n3 = (uint32_t)p0;
    c0 = n0;
    c1 = n1;
    c2 = n2;
    c3 = n3;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

/* The uniform used by stochastic rounding of element idx: word 0 of
 * Philox4x32-10 at counter (idx_lo, idx_hi, 0, 0), key (seed_lo, seed_hi),
 * top 24 bits. */
uint32_t orc_sr_uniform24(uint64_t idx, uint64_t seed) {
  uint32_t ctr[4] = {(uint32_t)idx, (uint32_t)(idx >> 32), 0u, 0u};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  orc_philox4x32_10(ctr, key, out);
  return out[0] >> 8;
}

/* ---------------------------------------------------------------------- */
/* tensor level                                                            */

static int64_t seg_begin(const int64_t* off, int32_t s, int64_t rows) {
  (void)rows;
  return off ? off[s] : 0;
}
static int64_t seg_end(const int64_t* off, int32_t s, int64_t rows) { return off ? off[s + 1] : rows; }

static int32_t segment_of_row(const int64_t* off, int32_t nseg, int64_t row) {
  if (!off) return 0;
  for (int32_t s = 0; s < nseg; ++s)
    if (row >= off[s] && row < off[s + 1]) return s;
  return nseg - 1;
}

/* Per-segment max |x|.  Non-finite inputs set ORC_NONFINITE and make that
 * segment's amax NaN. */
int orc_segment_amax(const uint16_t* x, int64_t rows, int64_t cols, int32_t nseg,
                     const int64_t* seg_off, float* amax_out) {
  int status = 0;
  for (int32_t s = 0; s < nseg; ++s) {
    float m = 0.0f;
    int bad = 0;
    for (int64_t r = seg_begin(seg_off, s, rows); r < seg_end(seg_off, s, rows); ++r)
      for (int64_t c = 0; c < cols; ++c) {
        uint16_t h = x[r * cols + c];
        if (!bf16_is_finite(h)) {
          bad = 1;
          continue;
        }
        float a = (float)bf16_abs(h);
        if (a > m) m = a;
      }
    amax_out[s] = bad ? NAN : m;
    if (bad) status |= ORC_NONFINITE;
  }
  return status;
}

int orc_segment_scales(int fmt, const uint16_t* x, int64_t rows, int64_t cols, int32_t nseg,
                       const int64_t* seg_off, float* s_t_out) {
  int status = orc_segment_amax(x, rows, cols, nseg, seg_off, s_t_out);
  for (int32_t s = 0; s < nseg; ++s)
    s_t_out[s] = isnan(s_t_out[s]) ? NAN : orc_tensor_scale(fmt, s_t_out[s]);
  return status;
}

/* Effective block scale of scale byte sc: s_t * dec(b) for the E4M3
 * formats, 2^(sc - 127) for MXFP4. */
static double block_scale(int fmt, uint8_t sc, float st) {
  return has_tensor_scale(fmt) ? (double)orc_nvfp4_block_scale(sc, st) : (double)orc_mxfp4_block_scale(sc);
}

static void put_code(uint8_t* codes, int64_t i, int nib) {
  uint8_t* p = &codes[i >> 1];
  if (i & 1)
    *p = (uint8_t)((*p & 0x0F) | (nib << 4));
  else
    *p = (uint8_t)((*p & 0xF0) | nib);
}
static int get_code(const uint8_t* codes, int64_t i) { return (codes[i >> 1] >> ((i & 1) * 4)) & 0xF; }
static void put_bit(uint8_t* bits, int64_t i, int b) {
  uint8_t* p = &bits[i >> 3];
  *p = (uint8_t)((*p & ~(1u << (i & 7))) | ((b & 1u) << (i & 7)));
}
static int get_bit(const uint8_t* bits, int64_t i) { return (bits[i >> 3] >> (i & 7)) & 1; }

/* Quantize rows [row_begin, row_end) with RTN (mode 0) or SR (mode 1).
 * NVFP4 and the uniform grid take the per-segment s_t (from
 * orc_segment_scales); MXFP4 ignores s_t.  Writes the codes, the scale bytes and, if bits != NULL, the
 * guidance bits of those rows (arrays are full-tensor sized). */
int orc_quantize_rows(int fmt, int mode, const uint16_t* x, int64_t rows, int64_t cols,
                      int32_t nseg, const int64_t* seg_off, const float* s_t, uint64_t seed,
                      int64_t row_begin, int64_t row_end, uint8_t* codes, uint8_t* scales,
                      uint8_t* bits) {
  const int block = block_of(fmt);
  const double* V = grid_of(fmt);
  const int64_t nblk_row = cols / block;
  int status = 0;
  (void)rows;
  for (int64_t r = row_begin; r < row_end; ++r) {
    float st = has_tensor_scale(fmt) ? s_t[segment_of_row(seg_off, nseg, r)] : 0.0f;
    if (has_tensor_scale(fmt) && isnan(st)) status |= ORC_NONFINITE;
    for (int64_t b = 0; b < nblk_row; ++b) {
      const int64_t base = r * cols + b * block;
      float bamax = 0.0f;
      int bad = 0;
      for (int k = 0; k < block; ++k) {
        uint16_t h = x[base + k];
        if (!bf16_is_finite(h)) bad = 1;
        else if ((float)bf16_abs(h) > bamax) bamax = (float)bf16_abs(h);
      }
      if (bad) status |= ORC_NONFINITE;
      uint8_t sc;
      double S;
      if (has_tensor_scale(fmt)) {
        sc = (isnan(st) || bad) ? 0 : orc_block_scale_code(fmt, bamax, st);
        S = (isnan(st) || bad) ? 0.0 : block_scale(fmt, sc, st);
      } else {
        int e = orc_e8m0_exponent(bamax);
        sc = (uint8_t)(e + 127);
        S = (double)orc_mxfp4_block_scale(sc);
      }
      scales[r * nblk_row + b] = sc;
      for (int k = 0; k < block; ++k) {
        const int64_t i = base + k;
        uint16_t h = x[i];
        int m3 = 0;
        if (!bad) {
          double ax = bf16_abs(h);
          m3 = mode == ORC_SR ? sr_on(V, ax, S, orc_sr_uniform24((uint64_t)i, seed)) : rtn_on(V, ax, S);
        }
        put_code(codes, i, (bf16_sign(h) << 3) | m3);
        if (bits) put_bit(bits, i, m3 & 1);
      }
    }
  }
  return status;
}

/* Train-side guided quantization of rows [row_begin, row_end): S comes
 * from the recorded scale byte (and recorded s_t for NVFP4) exactly as on
 * the rollout side; the sign is the train value's own. */
int orc_quantize_guided_rows(int fmt, const uint16_t* x, int64_t rows, int64_t cols,
                             int32_t nseg, const int64_t* seg_off, const uint8_t* rec_scales,
                             const float* rec_s_t, const uint8_t* rec_bits, int64_t row_begin,
                             int64_t row_end, uint8_t* codes) {
  const int block = block_of(fmt);
  const double* V = grid_of(fmt);
  const int64_t nblk_row = cols / block;
  int status = 0;
  (void)rows;
  for (int64_t r = row_begin; r < row_end; ++r) {
    float st = has_tensor_scale(fmt) ? rec_s_t[segment_of_row(seg_off, nseg, r)] : 0.0f;
    for (int64_t b = 0; b < nblk_row; ++b) {
      const int64_t base = r * cols + b * block;
      uint8_t sc = rec_scales[r * nblk_row + b];
      double S = block_scale(fmt, sc, st);
      int bad = 0;
      for (int k = 0; k < block; ++k)
        if (!bf16_is_finite(x[base + k])) bad = 1;
      if (bad) status |= ORC_NONFINITE;
      for (int k = 0; k < block; ++k) {
        const int64_t i = base + k;
        uint16_t h = x[i];
        int m3 = bad ? 0 : guided_on(V, bf16_abs(h), S, get_bit(rec_bits, i));
        put_code(codes, i, (bf16_sign(h) << 3) | m3);
      }
    }
  }
  return status;
}

/* Dequantize rows: out = (-1)^sign * RN_fp32(V[m3] * S); V*S is exact in
 * double, so the cast is the single rounding. */
void orc_dequantize_rows(int fmt, const uint8_t* codes, const uint8_t* scales, const float* s_t,
                         int64_t rows, int64_t cols, int32_t nseg, const int64_t* seg_off,
                         int64_t row_begin, int64_t row_end, float* out) {
  const int block = block_of(fmt);
  const double* V = grid_of(fmt);
  const int64_t nblk_row = cols / block;
  (void)rows;
  for (int64_t r = row_begin; r < row_end; ++r) {
    float st = has_tensor_scale(fmt) ? s_t[segment_of_row(seg_off, nseg, r)] : 0.0f;
    for (int64_t c = 0; c < cols; ++c) {
      const int64_t i = r * cols + c;
      uint8_t sc = scales[r * nblk_row + c / block];
      double S = block_scale(fmt, sc, st);
      int nib = get_code(codes, i);
      float mag = (float)(V[nib & 7] * S);
      out[i] = (nib & 8) ? -mag : mag;
    }
  }
}

/* Guidance extraction from codes ([TRACE-JA] quantization-info cache:
 * the mantissa bit is what is kept). */
void orc_pack_guidance(const uint8_t* codes, int64_t n, uint8_t* bits) {
  for (int64_t i = 0; i < n; ++i) put_bit(bits, i, get_code(codes, i) & 1);
}

void orc_unpack_guidance(const uint8_t* bits, int64_t n, uint8_t* mant) {
  for (int64_t i = 0; i < n; ++i) mant[i] = (uint8_t)get_bit(bits, i);
}

/* bf16 of a finite fp32 by round-to-nearest-even on the 16 dropped bits:
 * the plain definition of the bf16 output of the train-side fake
 * quantization (the fp32 dequantized value converted to bf16). */
uint16_t orc_f32_to_bf16(float v) {
  uint32_t b;
  memcpy(&b, &v, sizeof b);
  uint32_t lo = b & 0xFFFFu, hi = b >> 16;
  if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;
  return (uint16_t)hi;
}

void orc_f32_to_bf16_array(const float* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(v[i]);
}

/* Nearest rounding of x under GIVEN scale bytes (and s_t for NVFP4): the
 * train value rounded on the rollout's grid (used by the mismatch
 * diagnostics; [TRACE-JA] quantization-info cache section). */
void orc_rtn_with_scales_rows(int fmt, const uint16_t* x, int64_t rows, int64_t cols, int32_t nseg,
                              const int64_t* seg_off, const uint8_t* scales, const float* s_t,
                              int64_t row_begin, int64_t row_end, uint8_t* codes) {
  const int block = block_of(fmt);
  const double* V = grid_of(fmt);
  const int64_t nblk_row = cols / block;
  (void)rows;
  for (int64_t r = row_begin; r < row_end; ++r) {
    float st = has_tensor_scale(fmt) ? s_t[segment_of_row(seg_off, nseg, r)] : 0.0f;
    for (int64_t c = 0; c < cols; ++c) {
      const int64_t i = r * cols + c;
      uint8_t sc = scales[r * nblk_row + c / block];
      double S = block_scale(fmt, sc, st);
      uint16_t h = x[i];
      put_code(codes, i, (bf16_sign(h) << 3) | rtn_on(V, bf16_abs(h), S));
    }
  }
}

/* Block scales in the tiled layout block-scaled FP4 GEMMs read (NVIDIA cuBLAS
 * documentation, "1D Block Scaling Factors Layout"): the [rows, nb] scale
 * matrix, zero-padded to a multiple of 128 rows and 4 columns, is cut into
 * 128 x 4 tiles stored one after another in row-major tile order, 512 bytes
 * each; inside a tile, entry (r, c) sits at byte (r % 32) * 16 + (r / 32) * 4
 * + c. */
void orc_swizzle_scales(const uint8_t* scales, int64_t rows, int64_t nb, uint8_t* out) {
  const int64_t prow = (rows + 127) / 128 * 128, pcol = (nb + 3) / 4 * 4;
  const int64_t ntc = pcol / 4;
  for (int64_t r = 0; r < prow; ++r)
    for (int64_t c = 0; c < pcol; ++c) {
      const int64_t tile = (r / 128) * ntc + c / 4;
      const int64_t rr = r % 128, cc = c % 4;
      const int64_t off = tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + cc;
      out[off] = (r < rows && c < nb) ? scales[r * nb + c] : 0;
    }
}
