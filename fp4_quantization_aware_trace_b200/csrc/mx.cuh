// mx.cuh -- the MX-scaled variants: MXFP4 (W4A4, E2M1 elements) and W4A8
// (E4M3 activations), capture and fake-quant forwards.  Included by
// trace_fp4.cu inside its anonymous namespace.
#pragma once

// ---------------------------------------------------------------------------
// Kernels 8-9: the MXFP4 variant (the post's results list: the method carries
// over to MXFP4).  OCP Microscaling scales: one E8M0 byte per 32 elements of
// a row, X = 2^e with e = floor(log2 max|x|) - 2 clamped at -127, and no
// global scale.  A thread's pair of 16-element blocks is exactly one MX
// block.  Dividing by a power of two is exact up to the one rounding of the
// result, so z = x * 2^-e matches z = fl(x / X) with no correction step and
// no exact path; the E2M1 decisions are those of the NVFP4 kernels.
// ---------------------------------------------------------------------------

// E8M0 exponent of a block whose max|x| has the bf16 bits amax (sign
// cleared): floor(log2 amax) - 2, at least -127 (a bf16 amax stays below
// 2^128, so the top of the range is never reached); -127 for an all-zero
// block.
__device__ __forceinline__ int mx_exp(uint32_t amax) {
  if (amax == 0u) return -127;
  const int e = (int)(amax >> 7);
  const int fl = e != 0 ? e - 127 : (31 - __clz((int)amax)) - 133;  // bf16 subnormal: m * 2^-133
  return max(fl - 2, -127);
}

// Codes of one 16-element block: c0 elements 0-7, c1 elements 8-15.
__device__ __forceinline__ void mx_codes_block(const V8& v, u64 inv2, uint32_t& c0, uint32_t& c1) {
  // |z| < 8 from the block's own maximum; the conversion saturates past 6
  // and keeps the sign of x, also on zeros
  float z[16];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t w = v.w[k];
    upk(mul2(pk(bf16_lo(w), bf16_hi(w)), inv2), z[2 * k], z[2 * k + 1]);
  }
  c0 = cvt_e2m1x8(z[0], z[1], z[2], z[3], z[4], z[5], z[6], z[7]);
  c1 = cvt_e2m1x8(z[8], z[9], z[10], z[11], z[12], z[13], z[14], z[15]);
}

template <bool SW>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_mx_capture(const V8* __restrict__ x, Shape sh, uint4* __restrict__ codes,
                 uint32_t* __restrict__ mbits, uint8_t* __restrict__ scales) {
  pdl_begin();
  for (uint32_t t = blockIdx.x; t < sh.ntiles; t += gridDim.x) {
    const uint32_t b = t * kTileBlks + 2u * threadIdx.x;  // even; nblk is even
    if (b >= sh.nblk) continue;
    const V8 v0 = ld_block_stream(x + b), v1 = ld_block_stream(x + b + 1);
    const int e = mx_exp(max(absmax_block(v0), absmax_block(v1)));
    const float inv = pow2f(-e);
    const u64 inv2 = pk(inv, inv);
    uint4 c;
    mx_codes_block(v0, inv2, c.x, c.y);
    mx_codes_block(v1, inv2, c.z, c.w);
    codes[b >> 1] = c;
    mbits[b >> 1] = nibble_lsbs4(c);
    if (SW) {
      const uint32_t row = fastdiv(b, sh.bpr);
      scales[tiled_scale_offset(row, (b - row * sh.bpr.d) >> 1, sh.sw_ct)] = (uint8_t)(e + 127);
    } else {
      scales[b >> 1] = (uint8_t)(e + 127);
    }
  }
}

// Round to nearest over one 16-element half of an MX block (scale 2^e given
// as inv2 = 2^-e and X2 = 2^e): bf16 outputs, mask bits at pos0..pos0+15 of
// m, and the codes as rtn_block (KIND 0 none, 1 magnitudes, 2 signed with
// x's sign).
template <int KIND>
__device__ __forceinline__ void mx_rtn_block(const V8& v, u64 inv2, u64 X2, V8& o, uint32_t& m,
                                             int pos0, uint32_t& c0, uint32_t& c1) {
  // z = |x| * 2^-e (the sign is put back on the output); the mask bits are
  // accumulated on the FMA pipe as rtn_block does
  u64 mf = pk(0.0f, 0.0f);
  const u64 four = pk(4.0f, 4.0f);
  c0 = 0u;
  c1 = 0u;
#pragma unroll
  for (int p = 7; p >= 0; --p) {
    const uint32_t w = v.w[p];
    float zl, zh;
    upk(mul2(pk(__uint_as_float((w & 0x7FFFu) << 16), __uint_as_float(w & 0x7FFF0000u)), inv2),
        zl, zh);  // exact z >= 0 (inf only past 6)
    mf = fma2(mf, four, pk(le6_step(zl), le6_step(zh)));
    float al = fminf(zl, 6.0f), ah = fminf(zh, 6.0f);
    uint32_t h2;
    if (KIND == 0) {
      h2 = rtn_e2m1x2_f16x2(al, ah);
    } else {
      if (KIND == 2) {
        al = __uint_as_float(__float_as_uint(al) | ((w << 16) & 0x80000000u));
        ah = __uint_as_float(__float_as_uint(ah) | (w & 0x80000000u));
      }
      uint32_t code;
      h2 = rtn_e2m1x2_f16x2_code(al, ah, code);
      if (p < 4) c0 += code << (8 * p); else c1 += code << (8 * (p - 4));
    }
    const float tl = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
    const float th = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
    float ql, qh;
    upk(mul2(pk(tl, th), X2), ql, qh);  // exact
    o.w[p] = cvt_bf16x2(ql, qh) | (w & 0x80008000u);
  }
  float ml, mh;
  upk(mf, ml, mh);
  m |= __float2uint_rn(__fmaf_rn(mh, 2.0f, ml)) << pos0;
}

// Two elements of an MX guided rule: z = x * 2^-e exact, floor and ceiling
// by directed rounding with the unscaled grid addend, the rule's choice
// (side as guided_pair), scaled back by X = 2^e.
template <int MODE>
__device__ __forceinline__ uint32_t mx_guided_pair(uint32_t w, uint32_t side, u64 inv2, u64 X2) {
  float zl, zh;
  upk(mul2(pk(bf16_lo(w), bf16_hi(w)), inv2), zl, zh);  // exact z (inf only past 6)
  const float al = fminf(fabsf(zl), 6.0f), ah = fminf(fabsf(zh), 6.0f);
  const u64 MM = pk(grid_magic(al), grid_magic(ah));
  const u64 aa = pk(al, ah);
  float lol, loh, hil, hih;
  upk(add_rm2(aa, MM), lol, loh);
  upk(add_rp2(aa, MM), hil, hih);
  float tl, th;
  if (MODE == kGuided) {
    const uint32_t lb = __float_as_uint(lol), hb = __float_as_uint(loh);
    const float sl = __uint_as_float(lb + ((lb ^ side) & (__float_as_uint(hil) - lb)));
    const float sh = __uint_as_float(hb + ((hb ^ (side >> 1)) & (__float_as_uint(hih) - hb)));
    upk(sub2(pk(sl, sh), MM), tl, th);
  } else {
    float fl, fh, cl, ch;
    upk(sub2(pk(lol, loh), MM), fl, fh);
    upk(sub2(pk(hil, hih), MM), cl, ch);
    const uint32_t h2 = e2m1x2_to_f16x2(side & 0xFFu);
    float rl = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
    float rh = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
    rl = __uint_as_float(__float_as_uint(rl) ^ ((w << 16) & 0x80000000u));
    rh = __uint_as_float(__float_as_uint(rh) ^ (w & 0x80000000u));
    tl = rl > fl ? cl : fl;
    th = rh > fh ? ch : fh;
  }
  float ql, qh;
  upk(mul2(pk(tl, th), X2), ql, qh);  // exact
  return cvt_bf16x2(ql, qh) | (w & 0x80008000u);
}

// One 16-element half of the MX fake-quant forward: round to nearest, then
// (guided rules) the pairs holding a site where the rule disagrees with it
// recomputed with the rule's pair routine, as fq_block_fast.
template <int MODE>
__device__ __forceinline__ void mx_fq_half(const V8& v, uint32_t bits16, uint32_t r0, uint32_t r1,
                                           u64 inv2, u64 X2, V8& o, uint32_t& m, int pos0) {
  uint32_t c0, c1;
  mx_rtn_block<MODE == kRtn ? 0 : MODE == kGuided ? 1 : 2>(v, inv2, X2, o, m, pos0, c0, c1);
  if (MODE == kRtn) return;
  const uint32_t bad = MODE == kGuided ? (nibble_lsbs2(c0, c1) ^ bits16) & 0xFFFFu
                                       : nibble_any2(c0 ^ r0, c1 ^ r1);
  uint32_t pairs = (bad | (bad >> 1)) & 0x5555u;
  while (pairs != 0u) {
    const int p = (__ffs(pairs) - 1) >> 1;
    pairs &= pairs - 1u;
    const uint32_t side = MODE == kGuided ? bits16 >> (2 * p) : (p < 4 ? r0 : r1) >> (8 * (p & 3));
    put_word(o, p, mx_guided_pair<MODE>(pick_word(v, p), side, inv2, X2));
  }
}

template <int MODE, bool SW>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_mx_fake_quant(const V8* __restrict__ x, Shape sh, const uint32_t* __restrict__ mbits,
                    const uint4* __restrict__ rcodes, const uint8_t* __restrict__ scales,
                    V8* __restrict__ out, uint32_t* __restrict__ mask) {
  pdl_begin();
  for (uint32_t t = blockIdx.x; t < sh.ntiles; t += gridDim.x) {
    const uint32_t b = t * kTileBlks + 2u * threadIdx.x;  // even; nblk is even
    if (b >= sh.nblk) continue;
    const V8 v0 = ld_block_stream(x + b), v1 = ld_block_stream(x + b + 1);
    const uint32_t bits = MODE == kGuided ? __ldcs(mbits + (b >> 1)) : 0u;
    const uint4 rc = MODE == kFull ? __ldcs(rcodes + (b >> 1)) : make_uint4(0u, 0u, 0u, 0u);
    size_t so = b >> 1;
    if (SW) {
      const uint32_t row = fastdiv(b, sh.bpr);
      so = tiled_scale_offset(row, (b - row * sh.bpr.d) >> 1, sh.sw_ct);
    }
    const int e = (int)__ldcs(scales + so) - 127;
    const float inv = pow2f(-e), X = pow2f(e);
    const u64 inv2 = pk(inv, inv), X2 = pk(X, X);  // 2^-e and 2^e
    uint32_t m = 0u;
    V8 o;
    mx_fq_half<MODE>(v0, bits & 0xFFFFu, rc.x, rc.y, inv2, X2, o, m, 0);
    st_block(out + b, o);
    mx_fq_half<MODE>(v1, bits >> 16, rc.z, rc.w, inv2, X2, o, m, 16);
    st_block(out + b + 1, o);
    mask[b >> 1] = m;
  }
}

// ---------------------------------------------------------------------------
// Kernels 10-11: W4A8 -- TRACE on FP8 (E4M3) activations with MX scales (the
// post's results list names the W4A8 setting).  32-element blocks with an
// E8M0 scale X = 2^e, e = floor(log2 max|x|) - 8 (448 = 1.75 * 2^8), clamped
// at -127; z = x * 2^-e exactly as for MXFP4; round to nearest E4M3 (ties to
// the even mantissa) saturating at 448; one byte per code (sign in bit 7);
// the cached bit is the lowest bit of the magnitude code; STE mask |z| <= 448.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int mx8_exp(uint32_t amax) {
  if (amax == 0u) return -127;
  const int e = (int)(amax >> 7);
  const int fl = e != 0 ? e - 127 : (31 - __clz((int)amax)) - 133;
  return max(fl - 8, -127);
}

// Two fp32 -> two E4M3 bytes (round to nearest even, satfinite), lo in bits
// 0-7; the sign of each input is kept, also on zeros.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 bytes (lo in bits 0-7) -> f16x2 (exact, signed).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t h2;
  uint16_t in = (uint16_t)two;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return h2;
}

// Grid addend for the E4M3 grid: M = 2^20 * max(2^-6, 2^E) (E the binade
// of a <= 448), so that a + M keeps 3 fraction bits of a's binade (2^-9
// steps below 2^-6, E4M3's subnormal spacing).
__device__ __forceinline__ float grid_magic8(float a) {
  return __uint_as_float(max((__float_as_uint(a) & 0x7F800000u) + 0x0A000000u, 0x46800000u));
}

// Lowest bit of each of 4 code bytes -> 4 bits.
__device__ __forceinline__ uint32_t byte_lsbs(uint32_t w) {
  return ((w & 0x01010101u) * 0x01020408u) >> 24;
}

template <bool SW>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_mx8_capture(const V8* __restrict__ x, Shape sh, V8* __restrict__ codes,
                  uint32_t* __restrict__ mbits, uint8_t* __restrict__ scales) {
  pdl_begin();
  for (uint32_t t = blockIdx.x; t < sh.ntiles; t += gridDim.x) {
    const uint32_t b = t * kTileBlks + 2u * threadIdx.x;  // even; nblk is even
    if (b >= sh.nblk) continue;
    const V8 v0 = ld_block_stream(x + b), v1 = ld_block_stream(x + b + 1);
    const int e = mx8_exp(max(absmax_block(v0), absmax_block(v1)));
    const float inv = pow2f(-e);
    const u64 inv2 = pk(inv, inv);
    V8 c;
    uint32_t bits = 0u;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t w = k < 8 ? v0.w[k] : v1.w[k - 8];
      float zl, zh;
      upk(mul2(pk(bf16_lo(w), bf16_hi(w)), inv2), zl, zh);
      // |z| < 512 from the block's own maximum; the conversion saturates
      // past 448 and keeps the sign of x
      const uint32_t two = cvt_e4m3x2(zl, zh);
      if (k & 1) c.w[k >> 1] |= two << 16; else c.w[k >> 1] = two;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) bits |= byte_lsbs(c.w[k]) << (4 * k);
    st_block(codes + (b >> 1), c);  // one 32-byte store (a struct copy would split it)
    mbits[b >> 1] = bits;
    size_t so = b >> 1;
    if (SW) {
      const uint32_t row = fastdiv(b, sh.bpr);
      so = tiled_scale_offset(row, (b - row * sh.bpr.d) >> 1, sh.sw_ct);
    }
    scales[so] = (uint8_t)(e + 127);
  }
}

// Two elements of a W4A8 guided rule: z = x * 2^-e exact, floor and ceiling
// on the E4M3 grid by directed rounding with the grid addend, the rule's
// choice (side: kGuided -- the two cached bits; kFull -- the rollout's two
// code bytes, low first), scaled back by X = 2^e.
template <int MODE>
__device__ __forceinline__ uint32_t mx8_guided_pair(uint32_t w, uint32_t side, u64 inv2, u64 X2) {
  float zl, zh;
  upk(mul2(pk(bf16_lo(w), bf16_hi(w)), inv2), zl, zh);
  const float al = fminf(fabsf(zl), 448.0f), ah = fminf(fabsf(zh), 448.0f);
  const u64 MM = pk(grid_magic8(al), grid_magic8(ah));
  const u64 aa = pk(al, ah);
  float lol, loh, hil, hih;
  upk(add_rm2(aa, MM), lol, loh);
  upk(add_rp2(aa, MM), hil, hih);
  float tl, th;
  if (MODE == kGuided) {
    const uint32_t lb = __float_as_uint(lol), hb = __float_as_uint(loh);
    const float sl = __uint_as_float(lb + ((lb ^ side) & (__float_as_uint(hil) - lb)));
    const float sh = __uint_as_float(hb + ((hb ^ (side >> 1)) & (__float_as_uint(hih) - hb)));
    upk(sub2(pk(sl, sh), MM), tl, th);
  } else {
    float fl, fh, cl, ch;
    upk(sub2(pk(lol, loh), MM), fl, fh);
    upk(sub2(pk(hil, hih), MM), cl, ch);
    const uint32_t h2 = e4m3x2_to_f16x2(side & 0xFFFFu);
    float rl = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
    float rh = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
    rl = __uint_as_float(__float_as_uint(rl) ^ ((w << 16) & 0x80000000u));
    rh = __uint_as_float(__float_as_uint(rh) ^ (w & 0x80000000u));
    tl = rl > fl ? cl : fl;
    th = rh > fh ? ch : fh;
  }
  float ql, qh;
  upk(mul2(pk(tl, th), X2), ql, qh);  // exact
  return cvt_bf16x2(ql, qh) | (w & 0x80008000u);
}

// One 16-element half of the W4A8 fake-quant forward: round to nearest on
// the E4M3 grid (hardware conversion, ties to the even mantissa,
// saturating at 448) with the STE mask, then, for the guided rules, the
// sites whose rule disagrees with it recomputed and patched in, as
// fq_block_fast: the 1-bit rule wherever the code's lowest bit is not the
// cached bit, the full rule wherever the code (signed with x's sign) is not
// the rollout's; the pairs holding such a site are recomputed with the
// rule's pair routine.  bits16: the cached bits; r: the rollout's 16 code
// bytes of this half (4 words, element j in byte j).
template <int MODE>
__device__ __forceinline__ uint32_t mx8_rtn_half(const V8& v, uint32_t bits16, uint4 r, u64 inv2,
                                                 u64 X2, V8& o, uint32_t& m, int pos0) {
  uint32_t bad = 0u;
  u64 mf = pk(0.0f, 0.0f);
  const u64 four = pk(4.0f, 4.0f);
#pragma unroll
  for (int p = 7; p >= 0; --p) {
    const uint32_t w = v.w[p];
    float zl, zh;
    upk(mul2(pk(__uint_as_float((w & 0x7FFFu) << 16), __uint_as_float(w & 0x7FFF0000u)), inv2),
        zl, zh);  // exact z >= 0 (inf only past 448)
    mf = fma2(mf, four, pk(le448_step(zl), le448_step(zh)));
    float al = fminf(zl, 448.0f), ah = fminf(zh, 448.0f);
    if (MODE == kFull) {
      al = __uint_as_float(__float_as_uint(al) | ((w << 16) & 0x80000000u));
      ah = __uint_as_float(__float_as_uint(ah) | (w & 0x80000000u));
    }
    const uint32_t two = cvt_e4m3x2(al, ah);
    if (MODE == kGuided) {
      // lowest bits of the two codes (compared with the cached bits below)
      bad |= ((two & 1u) | ((two >> 7) & 2u)) << (2 * p);
    } else if (MODE == kFull) {
      const uint32_t rw = (p & 2) ? (p & 4 ? r.w : r.y) : (p & 4 ? r.z : r.x);
      const uint32_t dx = two ^ ((rw >> (16 * (p & 1))) & 0xFFFFu);
      bad |= (((dx & 0xFFu) != 0u) | (((dx >> 8) != 0u) << 1)) << (2 * p);
    }
    const uint32_t h2 = e4m3x2_to_f16x2(two);
    const float tl = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
    const float th = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
    float ql, qh;
    upk(mul2(pk(tl, th), X2), ql, qh);  // exact
    o.w[p] = cvt_bf16x2(ql, qh) | (w & 0x80008000u);
  }
  float ml, mh;
  upk(mf, ml, mh);
  m |= __float2uint_rn(__fmaf_rn(mh, 2.0f, ml)) << pos0;
  if (MODE == kRtn) return 0u;
  return MODE == kGuided ? (bad ^ bits16) & 0xFFFFu : bad;
}

template <int MODE>
__device__ __forceinline__ void mx8_fq_half(const V8& v, uint32_t bits16, uint4 r, u64 inv2,
                                            u64 X2, V8& o, uint32_t& m, int pos0) {
  const uint32_t bad = mx8_rtn_half<MODE>(v, bits16, r, inv2, X2, o, m, pos0);
  if (MODE == kRtn) return;
  uint32_t pairs = (bad | (bad >> 1)) & 0x5555u;
  while (pairs != 0u) {
    const int p = (__ffs(pairs) - 1) >> 1;
    pairs &= pairs - 1u;
    const uint32_t rw = p < 2 ? r.x : p < 4 ? r.y : p < 6 ? r.z : r.w;
    const uint32_t side = MODE == kGuided ? bits16 >> (2 * p) : rw >> (16 * (p & 1));
    put_word(o, p, mx8_guided_pair<MODE>(pick_word(v, p), side, inv2, X2));
  }
}

// SEP: out does not alias x; the guided rules then store both halves'
// round-to-nearest outputs and recompute the pairs that need it in one loop
// per thread, their inputs and rollout codes read back from memory, as
// k_fake_quant does.
template <int MODE, bool SW, bool SEP = false>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_mx8_fake_quant(const V8* __restrict__ x, Shape sh, const uint32_t* __restrict__ mbits,
                     const V8* __restrict__ rcodes, const uint8_t* __restrict__ scales,
                     V8* __restrict__ out, uint32_t* __restrict__ mask) {
  pdl_begin();
  for (uint32_t t = blockIdx.x; t < sh.ntiles; t += gridDim.x) {
    const uint32_t b = t * kTileBlks + 2u * threadIdx.x;  // even; nblk is even
    if (b >= sh.nblk) continue;
    // with separate outputs the guided rules read words of x (and halfwords
    // of the rollout codes) back for the pairs they recompute: keep them in L1
    constexpr bool kKeepL1 = SEP && MODE != kRtn;
    const V8 v0 = kKeepL1 ? ld_block_l1(x + b) : ld_block_stream(x + b);
    const V8 v1 = kKeepL1 ? ld_block_l1(x + b + 1) : ld_block_stream(x + b + 1);
    const uint32_t bits = MODE == kGuided ? __ldcs(mbits + (b >> 1)) : 0u;
    const V8 rc = MODE != kFull ? zero_block()
                  : kKeepL1     ? ld_block_l1(rcodes + (b >> 1))
                                : ld_block_stream(rcodes + (b >> 1));
    size_t so = b >> 1;
    if (SW) {
      const uint32_t row = fastdiv(b, sh.bpr);
      so = tiled_scale_offset(row, (b - row * sh.bpr.d) >> 1, sh.sw_ct);
    }
    const int e = (int)__ldcs(scales + so) - 127;
    const float inv = pow2f(-e), X = pow2f(e);
    const u64 inv2 = pk(inv, inv), X2 = pk(X, X);  // 2^-e and 2^e
    uint32_t m = 0u;
    V8 o;
    if (SEP && MODE != kRtn) {
      const uint32_t bad0 = mx8_rtn_half<MODE>(
          v0, bits & 0xFFFFu, make_uint4(rc.w[0], rc.w[1], rc.w[2], rc.w[3]), inv2, X2, o, m, 0);
      st_block(out + b, o);
      const uint32_t bad1 = mx8_rtn_half<MODE>(
          v1, bits >> 16, make_uint4(rc.w[4], rc.w[5], rc.w[6], rc.w[7]), inv2, X2, o, m, 16);
      st_block(out + b + 1, o);
      uint32_t pairs = ((bad0 | (bad0 >> 1)) & 0x5555u) | (((bad1 | (bad1 >> 1)) & 0x5555u) << 16);
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(x + b);
      const unsigned short* rh = reinterpret_cast<const unsigned short*>(rcodes + (b >> 1));
      uint32_t* ow = reinterpret_cast<uint32_t*>(out + b);
      while (pairs != 0u) {
        const int q = (__ffs(pairs) - 1) >> 1;  // pair q of the thread's 32 elements
        pairs &= pairs - 1u;
        const uint32_t side = MODE == kGuided ? bits >> (2 * q) : (uint32_t)__ldg(rh + q);
        ow[q] = mx8_guided_pair<MODE>(__ldg(xw + q), side, inv2, X2);
      }
    } else {
      mx8_fq_half<MODE>(v0, bits & 0xFFFFu, make_uint4(rc.w[0], rc.w[1], rc.w[2], rc.w[3]), inv2,
                        X2, o, m, 0);
      st_block(out + b, o);
      mx8_fq_half<MODE>(v1, bits >> 16, make_uint4(rc.w[4], rc.w[5], rc.w[6], rc.w[7]), inv2, X2,
                        o, m, 16);
      st_block(out + b + 1, o);
    }
    mask[b >> 1] = m;
  }
}
