/*
 * kernel_math_check.c -- exhaustive CPU checks of the two arithmetic
 * identities the CUDA kernels rely on (they are restated here in plain C;
 * nothing is shared with the kernels or the oracle).
 *
 * 1. Quotient: with r = RN(1/d), q0 = RN(x*r), e = RN(x - q0*d) (fused),
 *    z = RN(q0 + e*r) (fused), z == RN(x/d) for every bf16 x and fp32 d
 *    whose quotient is a normal number.  Rounding scales with the
 *    exponents, so every (bf16 significand, fp32 significand) pair with x in
 *    [1,2) and [2,4) and d in [1,2) covers it: 2^7 * 2^23 * 2 cases.
 *    (The correction step is Markstein's, IBM J. Res. Dev. 34(1), 1990.)
 *
 * 1b. The same step run negated -- q0' = RN(x*(-r)), e = RN(x + q0'*d),
 *    z' = RN(q0' + e*(-r)) -- gives z' == -RN(x/d) bit for bit on the same
 *    cases; and over every finite bf16 x (zeros and subnormals included)
 *    and denominators across [2^-90, 2^100], z' has the sign opposite to x
 *    (also for x = +-0 and for quotients that underflow), equals -(x/d)
 *    wherever |x/d| >= 1/4, and stays below 1/4 in magnitude elsewhere, so
 *    its E2M1 code is the signed zero there.  (A subnormal x can leave the
 *    remainder inexact, the unnegated step alike; every such case has
 *    |x/d| far below 1/4.)
 *
 * 2. Grid rounding: for every fp32 a in [0, 6], with
 *    M = 2^22 * max(1, 2^floor(log2 a)), RD(a + M) - M and RU(a + M) - M are
 *    the largest / smallest E2M1 codewords <= / >= a, and the lowest bit of
 *    the bits of RD(a + M) is the lowest bit of the floor codeword's code.
 *
 * Exit status 0 when all of them hold everywhere.  Build: gcc -O2 -mfma
 * -ffp-contract=off kernel_math_check.c -lm -lpthread
 */
#include <fenv.h>
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#define NT 8

static long neg_bad; /* 1b mismatches of the last run() */

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static const float VAL[8] = {0.f, .5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};

typedef struct { int t; long bad; long bad_neg; } arg_t;

static void* quotient_worker(void* p) {
  arg_t* A = (arg_t*)p;
  long bad = 0;
  for (uint32_t md = (uint32_t)A->t; md < (1u << 23); md += NT) {
    const float d = f_of(0x3F800000u | md);
    const float r = 1.0f / d;
    for (uint32_t ma = 0; ma < 128; ++ma) {
      for (uint32_t e = 0; e < 2; ++e) {
        const float x = f_of(((127u + e) << 23) | (ma << 16));
        volatile float q0 = x * r;
#ifdef NO_CORRECTION /* negative control: the uncorrected product */
        const float z = q0;
#else
        const float rem = fmaf(q0, -d, x);
        const float z = fmaf(rem, r, q0);
#endif
        if (u_of(z) != u_of(x / d)) ++bad;
#ifdef NO_CORRECTION
        const float zn = -q0;
#else
        volatile float q0n = x * -r;
        const float zn = fmaf(fmaf(q0n, d, x), -r, q0n);
#endif
        if (u_of(zn) != u_of(-(x / d))) ++A->bad_neg;
      }
    }
  }
  A->bad = bad;
  return 0;
}

static void* grid_worker(void* p) {
  arg_t* A = (arg_t*)p;
  long bad = 0;
  const uint32_t top = u_of(6.0f);
  for (uint32_t ab = (uint32_t)A->t; ab <= top; ab += NT) {
    const float a = f_of(ab);
    uint32_t mb = (ab & 0x7F800000u) + 0x0B000000u;
    if (mb < 0x4A800000u) mb = 0x4A800000u;
    const float M = f_of(mb);
    volatile float va = a, vM = M; /* re-read after every mode change */
    fesetround(FE_DOWNWARD);
    volatile float lo = va + vM;
    fesetround(FE_UPWARD);
    volatile float hi = va + vM;
    fesetround(FE_TONEAREST);
    const float flo = lo - M, fhi = hi - M; /* exact */
    int kl = 0, kh = 7;
    for (int k = 0; k < 8; ++k) if (VAL[k] <= a) kl = k;
    for (int k = 7; k >= 0; --k) if (VAL[k] >= a) kh = k;
#ifdef NO_CORRECTION /* negative control: a magic addend one binade too small */
    (void)flo;
    if (f_of(u_of(lo) - 0x00800000u) - M * 0.5f != VAL[kl]) ++bad;
#else
    if (flo != VAL[kl] || fhi != VAL[kh] || (int)(u_of(lo) & 1u) != (kl & 1)) ++bad;
#endif
  }
  A->bad = bad;
  return 0;
}

static long run(void* (*fn)(void*)) {
  pthread_t th[NT];
  arg_t a[NT];
  for (int i = 0; i < NT; ++i) {
    a[i].t = i; a[i].bad = 0; a[i].bad_neg = 0;
    pthread_create(&th[i], 0, fn, &a[i]);
  }
  long bad = 0;
  neg_bad = 0;
  for (int i = 0; i < NT; ++i) { pthread_join(th[i], 0); bad += a[i].bad; neg_bad += a[i].bad_neg; }
  return bad;
}

/* 1b, sign and code-range part: every finite bf16 x, d = 2^k * (1 + j/8). */
static void* sign_worker(void* p) {
  arg_t* A = (arg_t*)p;
  long bad = 0;
  for (int k = -90 + A->t; k <= 99; k += NT) {
    for (int j = 0; j < 8; ++j) {
      const float d = ldexpf(1.0f + (float)j / 8.0f, k);
      const float r = 1.0f / d;
      for (uint32_t xb = 0; xb < 0x10000u; ++xb) {
        if ((xb & 0x7F80u) == 0x7F80u) continue; /* inf / NaN */
        const float x = f_of(xb << 16);
        const float q = x / d;
        if (fabsf(q) > 0x1p64f) continue; /* far outside the clipped code range */
#if defined(NO_CORRECTION)
        const float zn = -q;
        (void)r;
#elif defined(SIGN_CONTROL) /* negative control: the unnegated step, negated after */
        volatile float q0 = x * r;
        const float zn = -fmaf(fmaf(q0, -d, x), r, q0);
#else
        volatile float q0n = x * -r;
        const float zn = fmaf(fmaf(q0n, d, x), -r, q0n);
#endif
        if (((u_of(zn) ^ u_of(x)) & 0x80000000u) == 0u) ++bad;
        else if (fabsf(q) >= 0.25f) { if (u_of(zn) != u_of(-q)) ++bad; }
        else if (!(fabsf(zn) < 0.25f)) ++bad;
      }
    }
  }
  A->bad = bad;
  return 0;
}

int main(void) {
  const long bq = run(quotient_worker);
  const long bn = neg_bad;
  printf("quotient: %ld mismatches of %ld cases\n", bq, (long)(1L << 31));
  const long bs = run(sign_worker);
  printf("negated quotient: %ld mismatches of %ld cases, %ld in the sign / range sweep\n", bn,
         (long)(1L << 31), bs);
  const long bg = run(grid_worker);
  printf("grid rounding: %ld mismatches of %u values in [0, 6]\n", bg, u_of(6.0f) + 1u);
  return (bq == 0 && bn == 0 && bs == 0 && bg == 0) ? 0 : 1;
}
