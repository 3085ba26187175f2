/*
 * trace_oracle.c -- CPU oracle for TRACE rollout-guided NVFP4 rounding.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the GPU path computes.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg load it.  It shares no code, header,
 * table or helper with the CUDA library, and it never calls it.
 *
 * Source of the method: the rcap.io post "TRACE: Rollout-Guided
 * Quantization-Aware Training for FP4" (2026-10-06):
 *   - section "rollout-guided rounding": pick, of the two FP4 codewords
 *     around the training value, the one that agrees with what the rollout
 *     produced;
 *   - section "compact cache": keep one mantissa bit per element plus the
 *     scale metadata;
 *   - the pseudocode listing: capture (fp4_quantize, low_bits) and the QAT
 *     forward (z = clip(x/s,-6,6), reconstruct_from_mantissa, fp4_bracket,
 *     argmin, straight_through_estimator).
 * The NVFP4 arithmetic (16-element blocks, E4M3 block scales, an fp32
 * per-tensor scale amax/(6*448), the E2M1 grid {0,.5,1,1.5,2,3,4,6}) is the
 * format the post's rollout runs in; the pages name NVFP4 but do not spell
 * it out, so the readings taken here are listed at each step.
 *
 * The MXFP4 variant near the end of the file (the post's results list: the
 * method carries over to MXFP4 W4A4) swaps the scale step for the OCP
 * Microscaling one; the rounding rules on the E2M1 grid are unchanged.  The
 * W4A8 variant after it applies the same rules to E4M3 (FP8) activations.
 *
 * Every floating-point operation below is ONE IEEE-754 binary32 operation
 * with round-to-nearest-even.  Build with -ffp-contract=off and without
 * -ffast-math so that the compiler fuses nothing.
 *
 * Parity pins: every function here is pinned by tests in tests/ against
 * brute force (exhaustive nearest-codeword and nearest-E4M3 searches in exact
 * rationals), library routines (torch bf16 and float8_e4m3fn conversion,
 * numpy float32 arithmetic), closed forms and the worked straddle example.
 */
#include <assert.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* E2M1 magnitudes, indexed by the 3-bit magnitude code. */
static const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

/* ------------------------------------------------------------------ */
/* Scalar format helpers                                               */
/* ------------------------------------------------------------------ */

/* bf16 -> fp32: the bf16 bits are the top half of the fp32 bits (exact). */
float oracle_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* fp32 -> bf16, round to nearest, ties to even, on the 16 dropped bits of
 * the significand (sign-magnitude, so the same rule holds for negatives;
 * overflow rounds to infinity as IEEE does).  Finite inputs only. */
uint16_t oracle_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint32_t sign = u & 0x80000000u;
  uint32_t mag = u & 0x7FFFFFFFu;
  assert(mag <= 0x7F7FFFFFu); /* finite */
  uint32_t keep = mag >> 16;
  uint32_t dropped = mag & 0xFFFFu;
  if (dropped > 0x8000u || (dropped == 0x8000u && (keep & 1u))) keep += 1u;
  return (uint16_t)((sign >> 16) | keep);
}

/* E4M3 (the "fn" variant: bias 7, no infinities, 0x7F/0xFF are NaN) -> fp32. */
float oracle_e4m3_to_f32(uint8_t b) {
  int s = (b >> 7) & 1;
  int e = (b >> 3) & 0xF;
  int m = b & 7;
  float v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexpf((float)m, -9);          /* subnormal: m * 2^-9 */
  else
    v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return s ? -v : v;
}

/* Non-negative fp32 -> E4M3, round to nearest with ties to the even
 * mantissa, saturating: anything that rounds above 448 becomes 448 (0x7E).
 * Textbook route: split t = f * 2^E with f in [1,2), round (f-1)*8 to an
 * integer (a carry bumps the exponent); below 2^-6 the grid is m * 2^-9. */
uint8_t oracle_f32_to_e4m3(float t) {
  assert(!(t < 0.0f) && !isnan(t));
  if (t >= 448.0f) return 0x7E;
  if (t < ldexpf(1.0f, -6)) {
    double q = nearbyint((double)t * 512.0); /* exact scaling, RNE */
    return (uint8_t)q;                       /* q == 8 is 2^-6 = 0x08 */
  }
  int E;
  double f = frexp((double)t, &E); /* t = f * 2^E, f in [0.5,1) */
  f *= 2.0;
  E -= 1;                          /* f in [1,2) */
  double q = nearbyint((f - 1.0) * 8.0); /* exact: f has 24 bits */
  if (q == 8.0) {
    q = 0.0;
    E += 1;
  }
  int code = ((E + 7) << 3) | (int)q;
  if (code > 0x7E) code = 0x7E;
  return (uint8_t)code;
}

/* Round a clipped magnitude a in [0,6] to the E2M1 grid, ties toward the
 * code whose mantissa bit (its least significant bit) is 0.  The midpoints
 * 0.25, 1.25, 2.5 and 5 therefore go down (to codes 0,2,4,6), and 0.75, 1.75
 * and 3.5 go up (to codes 2,4,6). */
int oracle_e2m1_rtn(float a) {
  assert(a >= 0.0f && a <= 6.0f);
  if (a <= 0.25f) return 0;
  if (a < 0.75f) return 1;
  if (a <= 1.25f) return 2;
  if (a < 1.75f) return 3;
  if (a <= 2.5f) return 4;
  if (a < 3.5f) return 5;
  if (a <= 5.0f) return 6;
  return 7;
}

/* fp4_bracket for a clipped magnitude a in [0,6]: the largest codeword <= a
 * and the smallest >= a.  They coincide when a is itself a codeword. */
void oracle_e2m1_bracket(float a, int* lo, int* hi) {
  assert(a >= 0.0f && a <= 6.0f);
  int l = 0;
  for (int k = 0; k < 8; ++k)
    if (kE2M1[k] <= a) l = k;
  int h = 7;
  for (int k = 7; k >= 0; --k)
    if (kE2M1[k] >= a) h = k;
  *lo = l;
  *hi = h;
}

/* The guided choice for one site (QAT forward in the pseudocode listing).
 * a: |z| after clipping; bit: the cached mantissa bit of the rollout code.
 * reconstruct_from_mantissa: read as "the bracket member whose mantissa bit
 * equals the cached bit" -- on the E2M1 code ladder neighbours alternate
 * that bit, so exactly one member qualifies; when the bracket collapses it
 * is its single member.  The argmin over the bracket is then taken as the
 * listing writes it.  Returns the magnitude code of q*. */
int oracle_guided_code(float a, int bit) {
  int lo, hi;
  oracle_e2m1_bracket(a, &lo, &hi);
  if (lo == hi) return lo;
  int q_hat = ((lo & 1) == (bit & 1)) ? lo : hi;
  float d_lo = fabsf(kE2M1[lo] - kE2M1[q_hat]);
  float d_hi = fabsf(kE2M1[hi] - kE2M1[q_hat]);
  return (d_lo <= d_hi) ? lo : hi;
}

/* Full-information guidance (the upper bound the post's layer ablation
 * compares the 1-bit cache against): the cache holds the whole rollout code,
 * and q* is the argmin of the listing taken with the exact rollout codeword:
 * of the two codewords bracketing z (one when z is a codeword), the one
 * nearest to q_roll.  z: the unclipped scaled value; roll_code: sign<<3 |
 * magnitude.  Returns the magnitude code of q*; its sign is that of z (both
 * bracket members lie on z's side of zero).  No tie is possible: q_roll is a
 * codeword, so it is either a bracket member or strictly nearer one end. */
int oracle_full_guided_code(float z, int roll_code) {
  float a = fabsf(z);
  if (a > 6.0f) a = 6.0f;
  int lo, hi;
  oracle_e2m1_bracket(a, &lo, &hi);
  /* the bracket of z on the signed grid */
  const float s = signbit(z) ? -1.0f : 1.0f;
  const float q_lo = s * kE2M1[lo], q_hi = s * kE2M1[hi];
  const float q_roll = ((roll_code & 8) ? -1.0f : 1.0f) * kE2M1[roll_code & 7];
  const float d_lo = fabsf(q_lo - q_roll), d_hi = fabsf(q_hi - q_roll);
  return (d_hi < d_lo) ? hi : lo;
}

/* Dequantised output for a signed code: bf16( (VAL[c] * sbv) * s_g ).
 * VAL[c] * sbv is exact (at most 2 x 4 significant bits), so the only
 * roundings are one fp32 multiply and the fp32 -> bf16 step. */
uint16_t oracle_dequant_bf16(int code, int negative, float sbv, float s_g) {
  float m = kE2M1[code] * sbv;
  float v = m * s_g;
  if (negative) v = -v;
  return oracle_f32_to_bf16(v);
}

/* ------------------------------------------------------------------ */
/* Scale computation shared by capture (rollout) and the comparators    */
/* ------------------------------------------------------------------ */

/* Global scale of one group: s_g = amax / (6*448), or 1 when amax is 0. */
float oracle_global_scale(float amax) {
  if (amax == 0.0f) return 1.0f;
  return amax / 2688.0f;
}

/* Block scale: t = bmax / (6 * s_g), then E4M3 with RNE and saturation. */
uint8_t oracle_block_scale(float bmax, float s_g) {
  float den6 = 6.0f * s_g;
  float t = bmax / den6;
  return oracle_f32_to_e4m3(t);
}

/* z for one element: x / (s_g * sbv); a zero denominator makes the whole
 * block a zero block, where z keeps only the sign of x. */
static float scaled_z(float x, float s_g, float sbv) {
  float d = s_g * sbv;
  if (d == 0.0f) return copysignf(0.0f, x);
  return x / d;
}

/* Group of a row: offsets[g] <= row < offsets[g+1] (linear search). */
static int group_of_row(int64_t row, int32_t G, const int64_t* offs) {
  if (G == 1 || offs == 0) return 0;
  for (int g = 0; g < G; ++g)
    if (row >= offs[g] && row < offs[g + 1]) return g;
  assert(0 && "row outside the group offsets");
  return -1;
}

static void check_offsets(int64_t rows, int32_t G, const int64_t* offs) {
  if (G == 1 || offs == 0) return;
  assert(offs[0] == 0 && offs[G] == rows);
  for (int g = 0; g < G; ++g) assert(offs[g] <= offs[g + 1]);
}

/* The global scale of every row, from the per-group scales. */
static float* expand_row_scales(int64_t rows, int32_t G, const int64_t* offs,
                                const float* gscale) {
  float* r = (float*)malloc((size_t)(rows > 0 ? rows : 1) * sizeof(float));
  assert(r);
  for (int64_t i = 0; i < rows; ++i) r[i] = gscale[group_of_row(i, G, offs)];
  return r;
}

/* ------------------------------------------------------------------ */
/* The four operations of the hot path                                 */
/* ------------------------------------------------------------------ */

/* Steps 1-2 of capture: amax = max |x| over the rows of each group. */
void oracle_group_amax(const uint16_t* x, int64_t rows, int64_t cols,
                       int32_t G, const int64_t* offs, float* amax) {
  assert(G >= 1);
  check_offsets(rows, G, offs);
  for (int g = 0; g < G; ++g) {
    int64_t r0 = (G == 1 || !offs) ? 0 : offs[g];
    int64_t r1 = (G == 1 || !offs) ? rows : offs[g + 1];
    float m = 0.0f;
    for (int64_t i = r0 * cols; i < r1 * cols; ++i) {
      float a = fabsf(oracle_bf16_to_f32(x[i]));
      assert(isfinite(a));
      if (a > m) m = a;
    }
    amax[g] = m;
  }
}

/* Steps 3-6 of capture for rows whose global scales are known:
 *   codes : N/2 bytes, element 2k in the low nibble of byte k, 2k+1 high;
 *           a code is sign<<3 | magnitude code.
 *   mbits : N/32 words, element i at bit (i & 31) of word (i >> 5).
 *   scales: N/16 E4M3 bytes, row-major [rows, cols/16]. */
void oracle_capture_rows(const uint16_t* x, int64_t rows, int64_t cols,
                         const float* row_gscale, uint8_t* codes,
                         uint32_t* mbits, uint8_t* scales) {
  assert(cols % 32 == 0);
  int64_t n = rows * cols;
  memset(codes, 0, (size_t)(n / 2));
  memset(mbits, 0, (size_t)(n / 32) * sizeof(uint32_t));
  for (int64_t b = 0; b < n / 16; ++b) {
    float s_g = row_gscale[(b * 16) / cols];
    float bmax = 0.0f;
    for (int j = 0; j < 16; ++j) {
      float a = fabsf(oracle_bf16_to_f32(x[b * 16 + j]));
      if (a > bmax) bmax = a;
    }
    uint8_t sb = oracle_block_scale(bmax, s_g);
    scales[b] = sb;
    float sbv = oracle_e4m3_to_f32(sb);
    for (int j = 0; j < 16; ++j) {
      int64_t i = b * 16 + j;
      float z = scaled_z(oracle_bf16_to_f32(x[i]), s_g, sbv);
      float a = fabsf(z);
      if (a > 6.0f) a = 6.0f; /* clip(z, -6, 6) */
      int c = oracle_e2m1_rtn(a);
      int code = (signbit(z) ? 8 : 0) | c;
      codes[i / 2] |= (uint8_t)(code << (4 * (i & 1)));
      mbits[i / 32] |= (uint32_t)(c & 1) << (i & 31); /* low_bits(q_roll, 1) */
    }
  }
}

/* Rollout capture (pseudocode: q_roll = fp4_quantize(x_rollout, scale_roll);
 * cache = (low_bits(q_roll, b=1), scale_roll)).  gscale: G fp32 scales. */
void oracle_capture(const uint16_t* x, int64_t rows, int64_t cols, int32_t G,
                    const int64_t* offs, uint8_t* codes, uint32_t* mbits,
                    uint8_t* scales, float* gscale) {
  assert(cols % 32 == 0 && G >= 1);
  float* amax = (float*)malloc((size_t)G * sizeof(float));
  assert(amax);
  oracle_group_amax(x, rows, cols, G, offs, amax);
  for (int g = 0; g < G; ++g) gscale[g] = oracle_global_scale(amax[g]);
  free(amax);
  float* rs = expand_row_scales(rows, G, offs, gscale);
  oracle_capture_rows(x, rows, cols, rs, codes, mbits, scales);
  free(rs);
}

/* One fake-quant forward over rows with given scales.  guided != 0 uses the
 * cached mantissa bits (TRACE); guided == 0 is plain round-to-nearest (the
 * vanilla QAT comparator).  mask: bit i set when |z_i| <= 6, z taken before
 * clipping (straight-through estimator support).  sites: optional signed
 * code per element. */
enum { FQ_RTN = 0, FQ_GUIDED = 1, FQ_FULL = 2 };

static void fake_quant(const uint16_t* x, int64_t rows, int64_t cols,
                       const float* row_gscale, const uint32_t* mbits,
                       const uint8_t* rcodes, const uint8_t* scales,
                       uint16_t* out, uint32_t* mask, uint8_t* sites,
                       int mode) {
  assert(cols % 32 == 0);
  int64_t n = rows * cols;
  if (mask) memset(mask, 0, (size_t)(n / 32) * sizeof(uint32_t));
  for (int64_t b = 0; b < n / 16; ++b) {
    float s_g = row_gscale[(b * 16) / cols];
    float sbv = oracle_e4m3_to_f32(scales[b]);
    for (int j = 0; j < 16; ++j) {
      int64_t i = b * 16 + j;
      float xv = oracle_bf16_to_f32(x[i]);
      assert(isfinite(xv));
      float z = scaled_z(xv, s_g, sbv);
      float a = fabsf(z);
      if (mask && a <= 6.0f) mask[i / 32] |= 1u << (i & 31);
      if (a > 6.0f) a = 6.0f;
      int c;
      if (mode == FQ_GUIDED)
        c = oracle_guided_code(a, (int)((mbits[i / 32] >> (i & 31)) & 1u));
      else if (mode == FQ_FULL)
        c = oracle_full_guided_code(z, (rcodes[i / 2] >> (4 * (i & 1))) & 0xF);
      else
        c = oracle_e2m1_rtn(a);
      if (out) out[i] = oracle_dequant_bf16(c, signbit(z) != 0, sbv, s_g);
      if (sites) sites[i] = (uint8_t)((signbit(z) ? 8 : 0) | c);
    }
  }
}

/* Guided QAT forward for rows with known global scales (row_gscale[r]);
 * mbits == NULL gives the round-to-nearest comparator instead. */
void oracle_fake_quant_rows(const uint16_t* x, int64_t rows, int64_t cols,
                            const float* row_gscale, const uint32_t* mbits,
                            const uint8_t* scales, uint16_t* out,
                            uint32_t* mask) {
  fake_quant(x, rows, cols, row_gscale, mbits, 0, scales, out, mask, 0,
             mbits != 0 ? FQ_GUIDED : FQ_RTN);
}

/* Guided QAT forward on x_train with the rollout's cache (pseudocode:
 * z = clip(x_train/s); bracket; pick by the cached bit; s * q_star). */
void oracle_guided_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                       int32_t G, const int64_t* offs, const uint32_t* mbits,
                       const uint8_t* scales, const float* gscale,
                       uint16_t* out, uint32_t* mask) {
  check_offsets(rows, G, offs);
  float* rs = expand_row_scales(rows, G, offs, gscale);
  fake_quant(x_train, rows, cols, rs, mbits, 0, scales, out, mask, 0, FQ_GUIDED);
  free(rs);
}

/* Plain round-to-nearest fake-quant with the given scales (comparator). */
void oracle_rtn_fwd(const uint16_t* x, int64_t rows, int64_t cols, int32_t G,
                    const int64_t* offs, const uint8_t* scales,
                    const float* gscale, uint16_t* out, uint32_t* mask) {
  check_offsets(rows, G, offs);
  float* rs = expand_row_scales(rows, G, offs, gscale);
  fake_quant(x, rows, cols, rs, 0, 0, scales, out, mask, 0, FQ_RTN);
  free(rs);
}

/* Diagnostic: the signed code (sign<<3 | magnitude code) that the guided
 * forward (mbits != NULL) or the round-to-nearest forward (mbits == NULL)
 * picks at every site, one byte per element.  Used to check the per-site
 * properties the post states for rollout-guided rounding. */
void oracle_fake_quant_codes(const uint16_t* x, int64_t rows, int64_t cols,
                             int32_t G, const int64_t* offs,
                             const uint32_t* mbits, const uint8_t* scales,
                             const float* gscale, uint8_t* sites) {
  check_offsets(rows, G, offs);
  float* rs = expand_row_scales(rows, G, offs, gscale);
  fake_quant(x, rows, cols, rs, mbits, 0, scales, 0, 0, sites,
             mbits != 0 ? FQ_GUIDED : FQ_RTN);
  free(rs);
}

/* Full-information guided forward on x_train with the rollout's full codes
 * (capture's `codes` output) and scales. */
void oracle_full_guided_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                            int32_t G, const int64_t* offs, const uint8_t* rcodes,
                            const uint8_t* scales, const float* gscale,
                            uint16_t* out, uint32_t* mask) {
  check_offsets(rows, G, offs);
  float* rs = expand_row_scales(rows, G, offs, gscale);
  fake_quant(x_train, rows, cols, rs, 0, rcodes, scales, out, mask, 0, FQ_FULL);
  free(rs);
}

/* Signed code picked at every site by full-information guidance. */
void oracle_full_guided_codes(const uint16_t* x, int64_t rows, int64_t cols,
                              int32_t G, const int64_t* offs,
                              const uint8_t* rcodes, const uint8_t* scales,
                              const float* gscale, uint8_t* sites) {
  check_offsets(rows, G, offs);
  float* rs = expand_row_scales(rows, G, offs, gscale);
  fake_quant(x, rows, cols, rs, 0, rcodes, scales, 0, 0, sites, FQ_FULL);
  free(rs);
}

/* Full-information guided forward for rows with known global scales. */
void oracle_full_guided_rows(const uint16_t* x, int64_t rows, int64_t cols,
                             const float* row_gscale, const uint8_t* rcodes,
                             const uint8_t* scales, uint16_t* out,
                             uint32_t* mask) {
  fake_quant(x, rows, cols, row_gscale, 0, rcodes, scales, out, mask, 0, FQ_FULL);
}

/* Position of a signed code on the signed E2M1 ladder: -7..7 (+0 and -0
 * are one point). */
static int ladder(int code) {
  const int mag = code & 7;
  return (code & 8) ? -mag : mag;
}

/* Mismatch diagnostic (the compact-cache paragraph: most sites where the two
 * paths disagree differ by one adjacent codebook entry).  For every element
 * of x_train, with the rollout's scales, three training-side codes are
 * compared with the rollout's code q_roll (capture's `codes`): round to
 * nearest, 1-bit guided (the bit is q_roll's mantissa bit), and
 * full-information guided.  hist[k*15 + d] counts the elements whose code k
 * (0 RTN, 1 guided, 2 full) sits d ladder steps from q_roll.  The counts are
 * added to hist. */
void oracle_mismatch_histogram(const uint16_t* x, int64_t rows, int64_t cols,
                               int32_t G, const int64_t* offs,
                               const uint8_t* rcodes, const uint8_t* scales,
                               const float* gscale, uint64_t* hist) {
  assert(cols % 32 == 0);
  check_offsets(rows, G, offs);
  float* rs = expand_row_scales(rows, G, offs, gscale);
  const int64_t n = rows * cols;
  for (int64_t b = 0; b < n / 16; ++b) {
    const float s_g = rs[(b * 16) / cols];
    const float sbv = oracle_e4m3_to_f32(scales[b]);
    for (int j = 0; j < 16; ++j) {
      const int64_t i = b * 16 + j;
      const float z = scaled_z(oracle_bf16_to_f32(x[i]), s_g, sbv);
      float a = fabsf(z);
      if (a > 6.0f) a = 6.0f;
      const int rc = (rcodes[i / 2] >> (4 * (i & 1))) & 0xF;
      const int sz = signbit(z) ? 8 : 0;
      const int c_rtn = sz | oracle_e2m1_rtn(a);
      const int c_gd = sz | oracle_guided_code(a, rc & 1);
      const int c_full = sz | oracle_full_guided_code(z, rc);
      const int lr = ladder(rc);
      hist[0 * 15 + abs(ladder(c_rtn) - lr)] += 1;
      hist[1 * 15 + abs(ladder(c_gd) - lr)] += 1;
      hist[2 * 15 + abs(ladder(c_full) - lr)] += 1;
    }
  }
  free(rs);
}

/* Masked straight-through estimator backward: the gradient passes where the
 * mask bit is set and is +0.0 elsewhere. */
void oracle_fq_bwd(const uint16_t* grad_out, const uint32_t* mask, int64_t n,
                   uint16_t* grad_in) {
  for (int64_t i = 0; i < n; ++i)
    grad_in[i] = ((mask[i / 32] >> (i & 31)) & 1u) ? grad_out[i] : (uint16_t)0;
}

/* ------------------------------------------------------------------ */
/* MXFP4 variant                                                        */
/*                                                                      */
/* The pages say only that the method carries over to MXFP4 and that    */
/* MX scales are powers of two.  The format is the OCP Microscaling one: */
/* 32-element blocks along a row, one E8M0 scale X = 2^e per block with  */
/* e = floor(log2(max|x|)) - 2 (2 is the exponent of E2M1's largest      */
/* value 6 = 1.5 * 2^2), clamped to E8M0's range [-127, 127]; an         */
/* all-zero block takes e = -127; there is no per-tensor scale.  Then    */
/* z = x / X, and clipping, rounding, the cached bit, the STE mask and   */
/* dequantisation q * X are those of the NVFP4 path.                     */
/* ------------------------------------------------------------------ */

/* E8M0 byte -> 2^(b - 127) (exact; 2^-127 is an fp32 subnormal). */
float oracle_e8m0_to_f32(uint8_t b) {
  assert(b != 0xFF); /* the NaN encoding is never produced */
  return ldexpf(1.0f, (int)b - 127);
}

/* E8M0 scale byte of a block whose largest magnitude is amax. */
uint8_t oracle_mx_scale(float amax) {
  int e = -127;
  if (amax != 0.0f) {
    int k;
    (void)frexpf(amax, &k); /* amax = m * 2^k, m in [0.5, 1): floor(log2) = k-1 */
    e = (k - 1) - 2;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
  }
  return (uint8_t)(e + 127);
}

/* MX capture: codes, mantissa bits (layouts as oracle_capture_rows) and one
 * E8M0 byte per 32 elements, row-major [rows, cols/32]. */
void oracle_mx_capture(const uint16_t* x, int64_t rows, int64_t cols,
                       uint8_t* codes, uint32_t* mbits, uint8_t* scales) {
  assert(cols % 32 == 0);
  const int64_t n = rows * cols;
  memset(codes, 0, (size_t)(n / 2));
  memset(mbits, 0, (size_t)(n / 32) * sizeof(uint32_t));
  for (int64_t b = 0; b < n / 32; ++b) {
    float bmax = 0.0f;
    for (int j = 0; j < 32; ++j) {
      const float a = fabsf(oracle_bf16_to_f32(x[b * 32 + j]));
      if (a > bmax) bmax = a;
    }
    scales[b] = oracle_mx_scale(bmax);
    const float X = oracle_e8m0_to_f32(scales[b]);
    for (int j = 0; j < 32; ++j) {
      const int64_t i = b * 32 + j;
      const float z = oracle_bf16_to_f32(x[i]) / X;
      float a = fabsf(z);
      if (a > 6.0f) a = 6.0f;
      const int c = oracle_e2m1_rtn(a);
      codes[i / 2] |= (uint8_t)(((signbit(z) ? 8 : 0) | c) << (4 * (i & 1)));
      mbits[i / 32] |= (uint32_t)(c & 1) << (i & 31);
    }
  }
}

/* MX fake-quant forward with given E8M0 scales; mode as fake_quant(). */
static void mx_fake_quant(const uint16_t* x, int64_t rows, int64_t cols,
                          const uint32_t* mbits, const uint8_t* rcodes,
                          const uint8_t* scales, uint16_t* out, uint32_t* mask,
                          uint8_t* sites, int mode) {
  assert(cols % 32 == 0);
  const int64_t n = rows * cols;
  if (mask) memset(mask, 0, (size_t)(n / 32) * sizeof(uint32_t));
  for (int64_t b = 0; b < n / 32; ++b) {
    const float X = oracle_e8m0_to_f32(scales[b]);
    for (int j = 0; j < 32; ++j) {
      const int64_t i = b * 32 + j;
      const float xv = oracle_bf16_to_f32(x[i]);
      assert(isfinite(xv));
      const float z = xv / X;
      float a = fabsf(z);
      if (mask && a <= 6.0f) mask[i / 32] |= 1u << (i & 31);
      if (a > 6.0f) a = 6.0f;
      int c;
      if (mode == FQ_GUIDED)
        c = oracle_guided_code(a, (int)((mbits[i / 32] >> (i & 31)) & 1u));
      else if (mode == FQ_FULL)
        c = oracle_full_guided_code(z, (rcodes[i / 2] >> (4 * (i & 1))) & 0xF);
      else
        c = oracle_e2m1_rtn(a);
      if (out) {
        float v = kE2M1[c] * X; /* exact: at most 2 significant bits */
        if (signbit(z)) v = -v;
        out[i] = oracle_f32_to_bf16(v);
      }
      if (sites) sites[i] = (uint8_t)((signbit(z) ? 8 : 0) | c);
    }
  }
}

void oracle_mx_guided_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                          const uint32_t* mbits, const uint8_t* scales,
                          uint16_t* out, uint32_t* mask) {
  mx_fake_quant(x_train, rows, cols, mbits, 0, scales, out, mask, 0, FQ_GUIDED);
}

void oracle_mx_rtn_fwd(const uint16_t* x, int64_t rows, int64_t cols,
                       const uint8_t* scales, uint16_t* out, uint32_t* mask) {
  mx_fake_quant(x, rows, cols, 0, 0, scales, out, mask, 0, FQ_RTN);
}

void oracle_mx_full_guided_fwd(const uint16_t* x_train, int64_t rows,
                               int64_t cols, const uint8_t* rcodes,
                               const uint8_t* scales, uint16_t* out,
                               uint32_t* mask) {
  mx_fake_quant(x_train, rows, cols, 0, rcodes, scales, out, mask, 0, FQ_FULL);
}

/* Per-element signed codes of an MX fake-quant (mode as fake_quant()). */
void oracle_mx_fake_quant_codes(const uint16_t* x, int64_t rows, int64_t cols,
                                const uint32_t* mbits, const uint8_t* rcodes,
                                const uint8_t* scales, uint8_t* sites, int mode) {
  mx_fake_quant(x, rows, cols, mbits, rcodes, scales, 0, 0, sites, mode);
}

/* ------------------------------------------------------------------ */
/* Block-scale layout of a block-scaled FP4 GEMM                        */
/*                                                                      */
/* The abstract on the thelatestinai.com TRACE page credits NVFP4 with  */
/* FP4 GEMMs that run W4A4 natively.  A tcgen05 block-scaled FP4 GEMM    */
/* reads its block scales not                                            */
/* row-major but in 128 x 4 tiles: the [rows, scols] scale matrix is     */
/* padded to whole tiles (rows to a multiple of 128, scale columns to a  */
/* multiple of 4), the tiles are stored one after another in row-major   */
/* tile order, and inside a 512-byte tile the entry of row r and column  */
/* c sits at 16 * (r mod 32) + 4 * (r div 32) + c.  The layout is the     */
/* same for E4M3 scales of 16-element blocks and E8M0 scales of          */
/* 32-element blocks.                                                    */
/* ------------------------------------------------------------------ */

/* Bytes of the tiled layout of a [rows, scols] scale matrix. */
int64_t oracle_swizzled_scale_bytes(int64_t rows, int64_t scols) {
  const int64_t rt = (rows + 127) / 128, ct = (scols + 3) / 4;
  return rt * ct * 512;
}

/* Row-major scales [rows, scols] -> the tiled layout (padding bytes 0). */
void oracle_swizzle_scales(const uint8_t* lin, int64_t rows, int64_t scols,
                           uint8_t* out) {
  const int64_t ct = (scols + 3) / 4;
  memset(out, 0, (size_t)oracle_swizzled_scale_bytes(rows, scols));
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < scols; ++c) {
      const int64_t tile = (r / 128) * ct + c / 4;
      const int64_t rr = r % 128, cc = c % 4;
      out[tile * 512 + 16 * (rr % 32) + 4 * (rr / 32) + cc] = lin[r * scols + c];
    }
  }
}

/* ------------------------------------------------------------------ */
/* W4A8: TRACE on FP8 activations with MX scales (MXFP8)                */
/*                                                                      */
/* The results list names the W4A8 setting beside MXFP4 W4A4.  With     */
/* 8-bit activations the elements are E4M3 (the OCP MX FP8 element that  */
/* carries mantissa bits) in 32-element blocks with an E8M0 scale        */
/* X = 2^e, e = floor(log2 max|x|) - 8 (8 is the exponent of E4M3's      */
/* largest value 448 = 1.75 * 2^8), clamped to [-127, 127] (-127 for an  */
/* all-zero block).  z = x / X, clipped to [-448, 448]; round to nearest */
/* E4M3 with ties to the even mantissa; the code is one byte (sign bit 7, */
/* magnitude 0..0x7E); the cached bit is the lowest bit of the magnitude */
/* code (its mantissa's last bit); the STE mask is |z| <= 448.  The      */
/* bracket and the two guided choices are those of the E2M1 path on the  */
/* E4M3 grid, whose neighbouring codes also alternate that bit.          */
/* ------------------------------------------------------------------ */

uint8_t oracle_mx8_scale(float amax) {
  int e = -127;
  if (amax != 0.0f) {
    int k;
    (void)frexpf(amax, &k);
    e = (k - 1) - 8;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
  }
  return (uint8_t)(e + 127);
}

/* The E4M3 codes around a in [0, 448]: the largest with value <= a and the
 * smallest with value >= a (by scanning the 127 finite magnitudes). */
void oracle_e4m3_bracket(float a, int* lo, int* hi) {
  assert(a >= 0.0f && a <= 448.0f);
  int l = 0, h = 0x7E;
  for (int c = 0; c <= 0x7E; ++c)
    if (oracle_e4m3_to_f32((uint8_t)c) <= a) l = c;
  for (int c = 0x7E; c >= 0; --c)
    if (oracle_e4m3_to_f32((uint8_t)c) >= a) h = c;
  *lo = l;
  *hi = h;
}

int oracle_e4m3_guided_code(float a, int bit) {
  int lo, hi;
  oracle_e4m3_bracket(a, &lo, &hi);
  if (lo == hi) return lo;
  return ((lo & 1) == (bit & 1)) ? lo : hi;
}

/* z unclipped; roll_code: the rollout's E4M3 byte (sign bit 7). */
int oracle_e4m3_full_guided_code(float z, int roll_code) {
  float a = fabsf(z);
  if (a > 448.0f) a = 448.0f;
  int lo, hi;
  oracle_e4m3_bracket(a, &lo, &hi);
  const float s = signbit(z) ? -1.0f : 1.0f;
  const float q_lo = s * oracle_e4m3_to_f32((uint8_t)lo), q_hi = s * oracle_e4m3_to_f32((uint8_t)hi);
  const float q_roll = ((roll_code & 0x80) ? -1.0f : 1.0f) *
                       oracle_e4m3_to_f32((uint8_t)(roll_code & 0x7F));
  return (fabsf(q_hi - q_roll) < fabsf(q_lo - q_roll)) ? hi : lo;
}

/* MXFP8 capture: codes uint8[N] (element i = byte i), mbits, E8M0 scales
 * [rows, cols/32]. */
void oracle_mx8_capture(const uint16_t* x, int64_t rows, int64_t cols,
                        uint8_t* codes, uint32_t* mbits, uint8_t* scales) {
  assert(cols % 32 == 0);
  const int64_t n = rows * cols;
  memset(mbits, 0, (size_t)(n / 32) * sizeof(uint32_t));
  for (int64_t b = 0; b < n / 32; ++b) {
    float bmax = 0.0f;
    for (int j = 0; j < 32; ++j) {
      const float a = fabsf(oracle_bf16_to_f32(x[b * 32 + j]));
      if (a > bmax) bmax = a;
    }
    scales[b] = oracle_mx8_scale(bmax);
    const float X = oracle_e8m0_to_f32(scales[b]);
    for (int j = 0; j < 32; ++j) {
      const int64_t i = b * 32 + j;
      const float z = oracle_bf16_to_f32(x[i]) / X;
      float a = fabsf(z);
      if (a > 448.0f) a = 448.0f;
      const int c = oracle_f32_to_e4m3(a);
      codes[i] = (uint8_t)((signbit(z) ? 0x80 : 0) | c);
      mbits[i / 32] |= (uint32_t)(c & 1) << (i & 31);
    }
  }
}

static void mx8_fake_quant(const uint16_t* x, int64_t rows, int64_t cols,
                           const uint32_t* mbits, const uint8_t* rcodes,
                           const uint8_t* scales, uint16_t* out, uint32_t* mask,
                           uint8_t* sites, int mode) {
  assert(cols % 32 == 0);
  const int64_t n = rows * cols;
  if (mask) memset(mask, 0, (size_t)(n / 32) * sizeof(uint32_t));
  for (int64_t b = 0; b < n / 32; ++b) {
    const float X = oracle_e8m0_to_f32(scales[b]);
    for (int j = 0; j < 32; ++j) {
      const int64_t i = b * 32 + j;
      const float xv = oracle_bf16_to_f32(x[i]);
      assert(isfinite(xv));
      const float z = xv / X;
      float a = fabsf(z);
      if (mask && a <= 448.0f) mask[i / 32] |= 1u << (i & 31);
      if (a > 448.0f) a = 448.0f;
      int c;
      if (mode == FQ_GUIDED)
        c = oracle_e4m3_guided_code(a, (int)((mbits[i / 32] >> (i & 31)) & 1u));
      else if (mode == FQ_FULL)
        c = oracle_e4m3_full_guided_code(z, rcodes[i]);
      else
        c = oracle_f32_to_e4m3(a);
      if (out) {
        float v = oracle_e4m3_to_f32((uint8_t)c) * X; /* exact: 4 significant bits */
        if (signbit(z)) v = -v;
        out[i] = oracle_f32_to_bf16(v);
      }
      if (sites) sites[i] = (uint8_t)((signbit(z) ? 0x80 : 0) | c);
    }
  }
}

void oracle_mx8_guided_fwd(const uint16_t* x, int64_t rows, int64_t cols,
                           const uint32_t* mbits, const uint8_t* scales,
                           uint16_t* out, uint32_t* mask) {
  mx8_fake_quant(x, rows, cols, mbits, 0, scales, out, mask, 0, FQ_GUIDED);
}

void oracle_mx8_rtn_fwd(const uint16_t* x, int64_t rows, int64_t cols,
                        const uint8_t* scales, uint16_t* out, uint32_t* mask) {
  mx8_fake_quant(x, rows, cols, 0, 0, scales, out, mask, 0, FQ_RTN);
}

void oracle_mx8_full_guided_fwd(const uint16_t* x, int64_t rows, int64_t cols,
                                const uint8_t* rcodes, const uint8_t* scales,
                                uint16_t* out, uint32_t* mask) {
  mx8_fake_quant(x, rows, cols, 0, rcodes, scales, out, mask, 0, FQ_FULL);
}

void oracle_mx8_fake_quant_codes(const uint16_t* x, int64_t rows, int64_t cols,
                                 const uint32_t* mbits, const uint8_t* rcodes,
                                 const uint8_t* scales, uint8_t* sites, int mode) {
  mx8_fake_quant(x, rows, cols, mbits, rcodes, scales, 0, 0, sites, mode);
}

/* E4M3 rounding of the fp32 values with bit patterns first .. first+count-1
 * (positive finite), for the exhaustive comparison with the device. */
void oracle_e4m3_sweep(uint32_t first, uint32_t count, uint8_t* out) {
  for (uint32_t i = 0; i < count; ++i) {
    const uint32_t u = first + i;
    float t;
    memcpy(&t, &u, sizeof t);
    out[i] = oracle_f32_to_e4m3(t);
  }
}

/* The mismatch diagnostic of oracle_mismatch_histogram for the MXFP4
 * variant: z = x / X with the rollout's E8M0 scales, the same three rules
 * and the same 15-point ladder. */
void oracle_mx_mismatch_histogram(const uint16_t* x, int64_t rows, int64_t cols,
                                  const uint8_t* rcodes, const uint8_t* scales,
                                  uint64_t* hist) {
  assert(cols % 32 == 0);
  const int64_t n = rows * cols;
  for (int64_t b = 0; b < n / 32; ++b) {
    const float X = oracle_e8m0_to_f32(scales[b]);
    for (int j = 0; j < 32; ++j) {
      const int64_t i = b * 32 + j;
      const float z = oracle_bf16_to_f32(x[i]) / X;
      float a = fabsf(z);
      if (a > 6.0f) a = 6.0f;
      const int rc = (rcodes[i / 2] >> (4 * (i & 1))) & 0xF;
      const int sz = signbit(z) ? 8 : 0;
      const int lr = ladder(rc);
      hist[0 * 15 + abs(ladder(sz | oracle_e2m1_rtn(a)) - lr)] += 1;
      hist[1 * 15 + abs(ladder(sz | oracle_guided_code(a, rc & 1)) - lr)] += 1;
      hist[2 * 15 + abs(ladder(sz | oracle_full_guided_code(z, rc)) - lr)] += 1;
    }
  }
}
