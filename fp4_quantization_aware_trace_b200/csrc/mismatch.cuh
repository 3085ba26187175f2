// mismatch.cuh -- the mismatch-distance histogram kernel (ladder distance of
// the round-to-nearest, 1-bit guided and full-information guided codes from
// the rollout's).  Included by trace_fp4.cu inside its anonymous namespace.
#pragma once

// ---------------------------------------------------------------------------
// Kernel 7: mismatch diagnostic.  For each element of x_train, with the
// rollout's scales, the distance on the signed E2M1 ladder (-6 .. -0.5, 0,
// 0.5 .. 6: 15 points) between the rollout's code and the code each of three
// training-side rules picks -- round to nearest, 1-bit guided, full-
// information guided -- counted into 3 x 15 bins (compact-cache paragraph:
// sites where the two sides disagree are nearly all one codeword apart).
//
// The codes of 8 elements travel as 8 nibbles of one 32-bit word, and the
// three rules, the distances and the counting run on whole words: every
// per-nibble sum or difference below stays inside 0..15, so no carry or
// borrow crosses into the next nibble.
// ---------------------------------------------------------------------------
constexpr int kHistBins = 15;  // distances 0..14
constexpr int kHistModes = 3;  // round to nearest, 1-bit guided, full-information guided

// The codes of one block, elements 0-7 in word 0 and 8-15 in word 1: floor
// and ceiling magnitude codes of clip(|z|) on the grid (equal when it is a
// codeword) and the round-to-nearest code with the sign of z.
struct BlockCodes {
  uint32_t f[2], c[2], r[2];
};

// One pair on the fast path: as the guided forward, z * 2^64 from |x|, the
// floor and ceiling by directed rounding on the grid, each scaled back and
// converted exactly to its code; round to nearest through the hardware
// conversion (ties to the even code) of min(|z|, 6) with the sign of x.
__device__ __forceinline__ void codes_pair(uint32_t w, const BlkK& k, float* f, float* c, float* r) {
  const uint32_t wa = w & 0x7FFF7FFFu;
  const u64 xx = pk(__uint_as_float(wa << 16), __uint_as_float(wa & 0xFFFF0000u));
  float zl, zh;
  upk(quot2(mul2(xx, pk(kXs, kXs)), k), zl, zh);
  const float al = fminf(zl, kSixS), ah = fminf(zh, kSixS);  // NaN (|x| * 2^64 = inf) -> 6 * 2^64
  const u64 MM = pk(grid_magic_s(al), grid_magic_s(ah));
  const u64 aa = pk(al, ah);
  const u64 un = pk(0x1p-64f, 0x1p-64f);
  float rl, rh;
  upk(mul2(sub2(add_rm2(aa, MM), MM), un), f[0], f[1]);
  upk(mul2(sub2(add_rp2(aa, MM), MM), un), c[0], c[1]);
  upk(mul2(aa, un), rl, rh);
  r[0] = __uint_as_float(__float_as_uint(rl) | ((w << 16) & 0x80000000u));
  r[1] = __uint_as_float(__float_as_uint(rh) | (w & 0x80000000u));
}

// The same codes on the exact path (d outside the fast range).
__device__ __noinline__ BlockCodes codes_block_exact(const V8* src, float d) {
  const V8 v = ld_block_ro(src);
  uint32_t f[2] = {0u, 0u}, c[2] = {0u, 0u}, r[2] = {0u, 0u};
  for (int j = 0; j < 16; ++j) {
    const uint32_t w = v.w[j >> 1];
    const float xf = (j & 1) ? bf16_hi(w) : bf16_lo(w);
    const Exact e = exact_site(xf, d);
    const uint32_t sg = (j & 1) ? (w >> 31) : ((w >> 15) & 1u);
    const int sh = 4 * (j & 7);
    f[j >> 3] |= (uint32_t)e.floor << sh;
    c[j >> 3] |= (uint32_t)(e.exact ? e.floor : e.floor + 1) << sh;
    r[j >> 3] |= ((sg << 3) | (uint32_t)e.rtn) << sh;
  }
  BlockCodes bc;
  for (int h = 0; h < 2; ++h) {
    bc.f[h] = f[h];
    bc.c[h] = c[h];
    bc.r[h] = r[h];
  }
  return bc;
}

// Codes of a block whose scale d is on the guided fast path.
__device__ __forceinline__ BlockCodes block_codes_fast(const V8& v, float d) {
  BlockCodes bc;
  const BlkK bk = make_blk(d, 0.0f, 0.0f);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float f[8], c[8], r[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) codes_pair(v.w[4 * h + k], bk, f + 2 * k, c + 2 * k, r + 2 * k);
    bc.f[h] = cvt_e2m1x8(f);
    bc.c[h] = cvt_e2m1x8(c);
    bc.r[h] = cvt_e2m1x8(r);
  }
  return bc;
}

// Codes of a block with any scale d: zero block, fast path or exact path.
__device__ __forceinline__ BlockCodes block_codes(const V8& v, const V8* src, float d) {
  BlockCodes bc;
  if (d == 0.0f) {
    // zero block: z = +-0, every code is zero with the sign of x
    bc.f[0] = bc.f[1] = bc.c[0] = bc.c[1] = 0u;
    bc.r[0] = bc.r[1] = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t w = v.w[k];
      bc.r[k >> 2] |= ((((w >> 15) & 1u) << 3) | ((w >> 31) << 7)) << (8 * (k & 3));
    }
  } else if (fast_scale(d, kDMaxExactZ)) {
    bc = block_codes_fast(v, d);
  } else {
    bc = codes_block_exact(src, d);
  }
  return bc;
}

// Ladder distances of 8 nibbles: training magnitude codes t against the
// rollout magnitudes qm (both 0..7); s15 is 0xF on nibbles where the two
// signs agree.  Same sign: |t - qm|; opposite signs: t + qm.
__device__ __forceinline__ uint32_t ladder_dist8(uint32_t t, uint32_t qm, uint32_t s15) {
  const uint32_t diff = t + 0x88888888u - qm;  // 8 + t - qm, in 1..15
  const uint32_t ge = diff & 0x88888888u;      // t >= qm
  const uint32_t m15 = ge | (ge - (ge >> 3));  // 0xF where t >= qm
  // t >= qm: diff - 8;  t < qm: 8 - diff = (7 - diff) + 1
  const uint32_t ad = (diff ^ 0x77777777u ^ m15) + 0x11111111u - (ge >> 3);
  return (ad & s15) | ((t + qm) & ~s15);
}

// Count 8 distances: ones in a register, two and above (rare) in shared
// memory; zeros are what is left over at the end.
__device__ __forceinline__ void count8(uint32_t d, uint32_t& ones, uint32_t* bins) {
  const uint32_t ge2 = (((d >> 1) & 0x77777777u) + 0x77777777u) & 0x88888888u;  // d >= 2
  ones += __popc(d & 0x11111111u & ~(ge2 >> 3));
  for (uint32_t g = ge2; g != 0u; g &= g - 1u) {
    const int j = (__ffs((int)g) - 1) >> 2;
    // a distance is at most 14; the clamp only keeps the index in bounds
    atomicAdd(&bins[min((d >> (4 * j)) & 0xFu, 14u)], 1u);
  }
}

// The three rules on 8 elements: f, c, r as in BlockCodes, q the rollout's
// signed codes.
__device__ __forceinline__ void hist_word(uint32_t f, uint32_t c, uint32_t r, uint32_t q,
                                          uint32_t (&ones)[kHistModes], uint32_t* bins) {
  const uint32_t ne = c - f;  // 1 where the bracket holds two codewords
  const uint32_t qm = q & 0x77777777u;
  const uint32_t s8 = ~(q ^ r) & 0x88888888u;  // signs of z and q_roll agree
  const uint32_t s15 = s8 | (s8 - (s8 >> 3));
  // round to nearest
  count8(ladder_dist8(r & 0x77777777u, qm, s15), ones[0], bins);
  // 1-bit guided: the ceiling where the floor's mantissa bit is not q_roll's
  count8(ladder_dist8(f + ((f ^ q) & ne), qm, s15), ones[1], bins + kHistBins);
  // full information: the ceiling where q_roll, on z's side, lies above the
  // floor (8 + qm - f - 1 has bit 3 set exactly when qm > f)
  const uint32_t up = ((qm + 0x88888888u - f - 0x11111111u) >> 3) & (s8 >> 3) & ne;
  count8(ladder_dist8(f + up, qm, s15), ones[2], bins + 2 * kHistBins);
}

// Floor, ceiling and signed round-to-nearest codes of one site on the exact
// path, packed as f | c << 4 | r << 8: z = x / d (NVFP4) or x * 2^-e given
// as inv (MX, exact).  Reads the site's bf16 input at src.
__device__ __noinline__ uint32_t site_codes_exact(const uint16_t* src, float d, float inv, int mx) {
  const uint32_t xb = (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(src));
  const float xf = __uint_as_float(xb << 16);
  const Exact e = mx ? exact_of_z(__fmul_rn(xf, inv)) : exact_site(xf, d);
  const uint32_t c = (uint32_t)(e.exact ? e.floor : e.floor + 1);
  const uint32_t r = (((xb >> 15) & 1u) << 3) | (uint32_t)e.rtn;
  return (uint32_t)e.floor | (c << 4) | (r << 8);
}

// Signed round-to-nearest codes of one fast-path block (c0: elements 0-7,
// c1: 8-15), each with the sign of x: the exact quotient, min(|z|, 6) --
// which also maps the NaN of an overflowing quotient (a training value far
// beyond the rollout's scale) to 6 -- and the hardware conversion.
__device__ __forceinline__ void rtn_codes_signed(const V8& v, float d, uint32_t& c0,
                                                 uint32_t& c1) {
  const BlkK k = make_blk(d, 0.0f, 0.0f);
  float a[16];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const uint32_t w = v.w[p];
    float zl, zh;
    upk(quot2(pk(bf16_lo(w), bf16_hi(w)), k), zl, zh);
    a[2 * p] = __uint_as_float(__float_as_uint(fminf(fabsf(zl), 6.0f)) | ((w << 16) & 0x80000000u));
    a[2 * p + 1] = __uint_as_float(__float_as_uint(fminf(fabsf(zh), 6.0f)) | (w & 0x80000000u));
  }
  c0 = cvt_e2m1x8(a);
  c1 = cvt_e2m1x8(a + 8);
}

// Floor, ceiling and signed round-to-nearest codes of one pair (word w) as
// three bytes (lo element in the low nibble), by the grid rounding of
// codes_pair (NVFP4, constants k) or on z = |x| * 2^-e (MX, inv2).
__device__ __forceinline__ void pair_codes(uint32_t w, const BlkK& k, uint32_t& f, uint32_t& c,
                                           uint32_t& r) {
  float ff[2], cc[2], rr[2];
  codes_pair(w, k, ff, cc, rr);
  f = cvt_e2m1x8(ff[0], ff[1], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f);
  c = cvt_e2m1x8(cc[0], cc[1], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f);
  r = cvt_e2m1x8(rr[0], rr[1], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f);
}
__device__ __forceinline__ void mx_pair_codes(uint32_t w, u64 inv2, uint32_t& f, uint32_t& c,
                                              uint32_t& r) {
  const uint32_t wa = w & 0x7FFF7FFFu;
  float zl, zh;
  upk(mul2(pk(bf16_lo(wa), bf16_hi(wa)), inv2), zl, zh);  // inf only past 6
  const float al = fminf(zl, 6.0f), ah = fminf(zh, 6.0f);
  const u64 MM = pk(grid_magic(al), grid_magic(ah));
  const u64 aa = pk(al, ah);
  float fl, fh, cl, ch;
  upk(sub2(add_rm2(aa, MM), MM), fl, fh);
  upk(sub2(add_rp2(aa, MM), MM), cl, ch);
  f = cvt_e2m1x8(fl, fh, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f);
  c = cvt_e2m1x8(cl, ch, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f);
  r = cvt_e2m1x8(__uint_as_float(__float_as_uint(al) | ((w << 16) & 0x80000000u)),
                 __uint_as_float(__float_as_uint(ah) | (w & 0x80000000u)), 0.f, 0.f, 0.f, 0.f,
                 0.f, 0.f);
}

// Bit j (0-31) set where nibble j of the four words differs from zero.
__device__ __forceinline__ uint32_t nibble_any4(uint4 w) {
  w.x |= w.x >> 1; w.y |= w.y >> 1; w.z |= w.z >> 1; w.w |= w.w >> 1;
  return nibble_lsbs4(make_uint4(w.x | (w.x >> 2), w.y | (w.y >> 2), w.z | (w.z >> 2),
                                 w.w | (w.w >> 2)));
}

// MX: MXFP4 scales (one E8M0 byte per thread's pair of blocks, no groups)
// instead of E4M3 block scales with global scales.
//
// Where the training side's round-to-nearest code (signed) equals the
// rollout's, all three rules sit at distance 0: round to nearest by
// definition, the 1-bit rule because that code's mantissa bit is the cached
// bit (it keeps the bracket member carrying it), the full rule because the
// rollout codeword is then in the bracket.  So the pass computes the signed
// round-to-nearest codes as capture does, and only the sites whose code
// differs from the rollout's -- rare for a drifted pair -- go through the
// exact per-site codes and the three rules.  Zero blocks and blocks outside
// the fast range take the whole-block path.
template <bool MX>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_mismatch_hist(const V8* __restrict__ x, Shape sh, const int64_t* __restrict__ offs,
                    const uint4* __restrict__ rcodes, const uint8_t* __restrict__ scales,
                    const float* __restrict__ gscale, unsigned long long* __restrict__ hist) {
  __shared__ uint32_t bins[kHistModes * kHistBins];
  __shared__ uint32_t seen;
  if (threadIdx.x < kHistModes * kHistBins) bins[threadIdx.x] = 0u;
  if (threadIdx.x == 0) seen = 0u;
  __syncthreads();
  pdl_begin();
  GroupCursor gc;
  gc.init(offs, sh.G);
  float s_g = 1.0f;
  uint32_t ones[kHistModes] = {0u, 0u, 0u}, n = 0u;

  for (uint32_t t = blockIdx.x; t < sh.ntiles; t += gridDim.x) {
    const uint32_t b = t * kTileBlks + 2u * threadIdx.x;  // even; nblk is even
    if (b >= sh.nblk) continue;
    const V8 v0 = ld_block_stream(x + b), v1 = ld_block_stream(x + b + 1);
    const uint4 rc = __ldcs(rcodes + (b >> 1));
    const uint16_t* src = reinterpret_cast<const uint16_t*>(x + b);
    n += 32u;
    float d0 = 0.0f, d1 = 0.0f, inv = 0.0f;
    uint4 r;
    if (MX) {
      inv = pow2f(127 - (int)__ldcs(scales + (b >> 1)));
      const u64 inv2 = pk(inv, inv);
      mx_codes_block(v0, inv2, r.x, r.y);
      mx_codes_block(v1, inv2, r.z, r.w);
    } else {
      const uint32_t sb2 = __ldcs(reinterpret_cast<const unsigned short*>(scales) + (b >> 1));
      if (gc.seek(sh.G > 1 ? fastdiv(b, sh.bpr) : 0u)) s_g = __ldg(gscale + gc.g);
      float sbv0, sbv1;
      e4m3x2_to_f32(sb2, sbv0, sbv1);
      d0 = __fmul_rn(s_g, sbv0);
      d1 = __fmul_rn(s_g, sbv1);
      if (!(fast_scale(d0) && fast_scale(d1))) {
        // zero block or a scale outside the fast range: whole blocks
        const BlockCodes k0 = block_codes(v0, x + b, d0), k1 = block_codes(v1, x + b + 1, d1);
        hist_word(k0.f[0], k0.c[0], k0.r[0], rc.x, ones, bins);
        hist_word(k0.f[1], k0.c[1], k0.r[1], rc.y, ones, bins);
        hist_word(k1.f[0], k1.c[0], k1.r[0], rc.z, ones, bins);
        hist_word(k1.f[1], k1.c[1], k1.r[1], rc.w, ones, bins);
        continue;
      }
      rtn_codes_signed(v0, d0, r.x, r.y);
      rtn_codes_signed(v1, d1, r.z, r.w);
    }
    const uint32_t bad = nibble_any4(make_uint4(r.x ^ rc.x, r.y ^ rc.y, r.z ^ rc.z, r.w ^ rc.w));
    // the pairs holding such a site, each counted whole: a site of the pair
    // whose code agrees sits at distance 0 under every rule, which is what
    // the count leaves to the remainder anyway
    uint32_t pairs = (bad | (bad >> 1)) & 0x55555555u;
    while (pairs != 0u) {
      const int p = (__ffs(pairs) - 1) >> 1;  // 0..15: pair p & 7 of block p >> 3
      pairs &= pairs - 1u;
      const uint32_t q = ((p < 4 ? rc.x : p < 8 ? rc.y : p < 12 ? rc.z : rc.w) >> (8 * (p & 3))) & 0xFFu;
      const uint32_t w = p < 8 ? pick_word(v0, p) : pick_word(v1, p & 7);
      const float d = p < 8 ? d0 : d1;
      uint32_t f, c, rr;
      if (MX) {
        mx_pair_codes(w, pk(inv, inv), f, c, rr);
      } else if (fast_scale(d, kDMaxExactZ)) {
        pair_codes(w, make_blk(d, 0.0f, 0.0f), f, c, rr);
      } else {
        const uint32_t lo = site_codes_exact(src + 2 * p, d, inv, 0);
        const uint32_t hi = site_codes_exact(src + 2 * p + 1, d, inv, 0);
        f = (lo & 0xFu) | ((hi & 0xFu) << 4);
        c = ((lo >> 4) & 0xFu) | (hi & 0xF0u);
        rr = (lo >> 8) | ((hi >> 8) << 4);
      }
      // the pair in the lowest byte; the other six nibbles are all zero and
      // count as distance 0
      hist_word(f, c, rr, q, ones, bins);
    }
  }
#pragma unroll
  for (int k = 0; k < kHistModes; ++k) ones[k] = __reduce_add_sync(0xFFFFFFFFu, ones[k]);
  n = __reduce_add_sync(0xFFFFFFFFu, n);
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int k = 0; k < kHistModes; ++k) atomicAdd(&bins[k * kHistBins + 1], ones[k]);
    atomicAdd(&seen, n);
  }
  __syncthreads();
  if (threadIdx.x < kHistModes * kHistBins) {
    const int k = threadIdx.x / kHistBins, dist = threadIdx.x % kHistBins;
    uint32_t v = bins[threadIdx.x];
    if (dist == 0) {
      uint32_t other = 0u;
      for (int j = 1; j < kHistBins; ++j) other += bins[k * kHistBins + j];
      v = seen - other;
    }
    if (v != 0u) atomicAdd(hist + threadIdx.x, (unsigned long long)v);
  }
}
