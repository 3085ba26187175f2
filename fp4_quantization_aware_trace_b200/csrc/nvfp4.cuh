// nvfp4.cuh -- the NVFP4 kernels of the path: zeroing of the amax
// accumulators, the grid amax, rollout capture, the fake-quant forward (round
// to nearest, 1-bit guided, full-information guided) and the masked
// straight-through backward, plus their exact per-element path.  Included by
// trace_fp4.cu inside its anonymous namespace.
#pragma once

// ---- exact path: the format's steps with an IEEE division -----------------

struct Exact {
  int rtn;     // round-to-nearest magnitude code of clip(|z|)
  int floor;   // largest code with value <= clip(|z|)
  bool exact;  // clip(|z|) is a codeword (bracket collapses)
  bool in;     // |z| <= 6 (STE mask)
};

// The decisions of a site from its exact quotient z.
__device__ __forceinline__ Exact exact_of_z(float z) {
  const float a = fabsf(z);
  Exact e;
  e.in = a <= 6.0f;
  const float c = fminf(a, 6.0f);
  e.rtn = (c <= 0.25f) ? 0 : (c < 0.75f) ? 1 : (c <= 1.25f) ? 2 : (c < 1.75f) ? 3
        : (c <= 2.5f) ? 4 : (c < 3.5f) ? 5 : (c <= 5.0f) ? 6 : 7;
  e.floor = (c < 0.5f) ? 0 : (c < 1.0f) ? 1 : (c < 1.5f) ? 2 : (c < 2.0f) ? 3
          : (c < 3.0f) ? 4 : (c < 4.0f) ? 5 : (c < 6.0f) ? 6 : 7;
  const float v = (e.floor == 0) ? 0.0f : (e.floor == 1) ? 0.5f : (e.floor == 2) ? 1.0f
                : (e.floor == 3) ? 1.5f : (e.floor == 4) ? 2.0f : (e.floor == 5) ? 3.0f
                : (e.floor == 6) ? 4.0f : 6.0f;
  e.exact = (c == v);
  return e;
}

// The decisions of a site x with scale d (IEEE division; d = 0 gives +-0).
__device__ __forceinline__ Exact exact_site(float xf, float d) {
  return exact_of_z((d == 0.0f) ? copysignf(0.0f, xf) : __fdiv_rn(xf, d));
}

// E2M1 magnitude (as fp32) of a code 0..7.
__device__ __forceinline__ float e2m1_value(int c) {
  return c >= 2 ? __uint_as_float((uint32_t)(c + 252) << 22) : (c == 1 ? 0.5f : 0.0f);
}

// Capture of one block on the exact path: 16 codes (sign<<3 | rtn).
// The out-of-line exact-path functions read their block back from global
// memory and return their results by value (or store them themselves):
// passing the block's registers in or taking the address of the caller's
// outputs put those locals in local memory on every path, the fast one
// included.
__device__ __noinline__ uint2 capture_block_exact(const V8* src, float d) {
  const V8 v = ld_block_ro(src);
  uint32_t c[2] = {0u, 0u};
  for (int j = 0; j < 16; ++j) {
    const uint32_t w = v.w[j >> 1];
    const float xf = (j & 1) ? bf16_hi(w) : bf16_lo(w);
    const Exact e = exact_site(xf, d);
    const uint32_t sg = (j & 1) ? (w >> 31) : ((w >> 15) & 1u);
    c[j >> 3] |= ((sg << 3) | (uint32_t)e.rtn) << (4 * (j & 7));
  }
  return make_uint2(c[0], c[1]);
}

// Output bits (bf16 with x's sign) of one site on the exact path, for
// `mode` 0 round to nearest, 1 guided by the cached bit `side`, 2 guided by
// the rollout's signed 4-bit code `side` (full information: of floor and
// ceiling, the one nearest the rollout value reflected to z's side of zero;
// no codeword lies between them, so that is the ceiling exactly when the
// value lies above the floor).  `in` receives the STE mask bit.
// The code a rule picks at a site with decisions e (mode and side as
// site_exact below; xb: the site's bf16 bits, for its sign).
__device__ __forceinline__ int rule_code(const Exact& e, uint32_t xb, uint32_t side, int mode) {
  int c = e.rtn;
  if (mode == 1) {
    c = e.exact ? e.floor : e.floor + ((e.floor ^ (int)(side & 1u)) & 1);
  } else if (mode == 2) {
    float q = e2m1_value((int)(side & 7u));
    if (((side >> 3) & 1u) != ((xb >> 15) & 1u)) q = -q;
    const int hi = e.exact ? e.floor : e.floor + 1;
    c = (q > e2m1_value(e.floor)) ? hi : e.floor;
  }
  return c;
}

__device__ __forceinline__ uint32_t site_exact(uint32_t xb, float d, float sbv, float s_g,
                                               uint32_t side, int mode, bool& in) {
  const Exact e = exact_site(__uint_as_float(xb << 16), d);
  const int c = rule_code(e, xb, side, mode);
  in = e.in;
  const uint32_t mag = (uint32_t)__bfloat16_as_ushort(
      __float2bfloat16_rn(__fmul_rn(__fmul_rn(e2m1_value(c), sbv), s_g)));
  return (xb & 0x8000u) | mag;
}

// Fake-quant of one block on the exact path: bf16 outputs and STE mask.
// mode as site_exact; bits16: the cached bits (mode 1); c0, c1: the rollout
// codes of elements 0-7 and 8-15 (mode 2).
__device__ __noinline__ uint32_t fake_quant_block_exact(const V8* src, float d, float sbv, float s_g,
                                                    uint32_t bits16, uint32_t c0, uint32_t c1,
                                                    int mode, V8* dst) {
  const V8 v = ld_block_ro(src);
  uint32_t m = 0u;
  V8 o;
  for (int k = 0; k < 8; ++k) o.w[k] = 0u;
  for (int j = 0; j < 16; ++j) {
    const uint32_t w = v.w[j >> 1];
    const uint32_t xb = (j & 1) ? (w >> 16) : (w & 0xFFFFu);
    const uint32_t side = mode == 1 ? (bits16 >> j) & 1u
                        : ((j < 8 ? c0 : c1) >> (4 * (j & 7))) & 0xFu;
    bool in;
    o.w[j >> 1] |= site_exact(xb, d, sbv, s_g, side, mode, in) << (16 * (j & 1));
    m |= (uint32_t)in << j;
  }
  st_block_plain(dst, o);
  return m;
}

// One site of a guided forward recomputed on the exact path (the fast pass
// rounded it to nearest, and the site's rule may choose the other
// neighbour): reads the site's bf16 input at src, returns its output bits.
__device__ __noinline__ uint32_t guided_site_fix(const uint16_t* src, float d, float sbv,
                                                 float s_g, uint32_t side, int mode) {
  bool in;
  return site_exact((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(src)), d, sbv, s_g,
                    side, mode, in);
}

// ---------------------------------------------------------------------------
// Kernel 0: zero the per-group amax accumulators.
// ---------------------------------------------------------------------------
__global__ void k_zero_u32(uint32_t* p, int n) {
  pdl_begin();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = 0u;
}

// Per-group constants of capture.
struct GroupK {
  float s_g;    // amax / 2688, or 1
  float den6;   // RN(6 * s_g)
  float r6;     // RN(1 / den6)
  bool fast6;   // den6 in the range where bmax/den6 may use the FMA quotient
};

__device__ __forceinline__ GroupK group_consts(uint32_t amax_bits) {
  GroupK k;
  const float a = __uint_as_float(amax_bits << 16);
  k.s_g = amax_bits == 0u ? 1.0f : __fdiv_rn(a, 2688.0f);
  k.den6 = __fmul_rn(6.0f, k.s_g);
  k.fast6 = fast_scale(k.den6);
  k.r6 = k.fast6 ? __frcp_rn(k.den6) : 0.0f;
  return k;
}

// The same constants from s_g (as the amax pass leaves it in gscale).
__device__ __forceinline__ GroupK group_consts_of_sg(float s_g) {
  GroupK k;
  k.s_g = s_g;
  k.den6 = __fmul_rn(6.0f, s_g);
  k.fast6 = fast_scale(k.den6);
  k.r6 = k.fast6 ? __frcp_rn(k.den6) : 0.0f;
  return k;
}

// ---------------------------------------------------------------------------
// Kernel 1: per-group amax (bits of max|x| as bf16, kept as u32 so that
// atomicMax orders them as magnitudes), max-accumulated into amax[0, G):
// the first pass of a capture whose tensor is split into row shards or
// chunks (the one-launch capture below reduces inside its own grid).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_amax(const V8* __restrict__ x, Shape sh, const int64_t* __restrict__ offs,
           uint32_t* __restrict__ amax) {
  __shared__ uint32_t table[kAmaxTable];
  __shared__ int g_first_s;
  pdl_begin();
  if (blockIdx.x >= sh.ntiles) return;

  // the first tile's loads go out before the CTA's set-up barrier
  V8 v[kBlkPerThread];
  {
    const uint32_t base = blockIdx.x * kTileBlks + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kBlkPerThread; ++u) {
      const uint32_t b = base + u * kThreads;
      v[u] = b < sh.nblk ? ld_block_stream(x + b) : zero_block();
    }
  }
  GroupCursor gc;
  gc.init(offs, sh.G);
  if (sh.G > 1) {
    if (threadIdx.x == 0) {
      gc.seek(fastdiv(blockIdx.x * kTileBlks, sh.bpr));
      g_first_s = gc.g;
    }
    for (int i = threadIdx.x; i < kAmaxTable; i += kThreads) table[i] = 0u;
  } else if (threadIdx.x == 0) {
    table[0] = 0u;
    g_first_s = 0;
  }
  __syncthreads();
  const int g_first = g_first_s;
  gc.init(offs, sh.G);

  uint32_t run = 0u;
  int run_g = -1;
  auto flush = [&](int g, uint32_t val) {
    if (g < 0 || val == 0u) return;
    const int slot = g - g_first;
    if (slot >= 0 && slot < kAmaxTable) atomicMax(&table[slot], val);
    else atomicMax(&amax[g], val);
  };

  for (uint32_t t = blockIdx.x; t < sh.ntiles;) {
    const uint32_t base = t * kTileBlks + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kBlkPerThread; ++u) {
      const uint32_t b = base + u * kThreads;
      if (b >= sh.nblk) continue;
      if (sh.G > 1) {
        gc.seek(fastdiv(b, sh.bpr));
        if (gc.g != run_g) {
          flush(run_g, run);
          run = 0u;
          run_g = gc.g;
        }
      } else {
        run_g = 0;
      }
      run = max(run, absmax_block(v[u]));
    }
    t += gridDim.x;
    if (t >= sh.ntiles) break;
    const uint32_t nb = t * kTileBlks + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kBlkPerThread; ++u) {
      const uint32_t b = nb + u * kThreads;
      v[u] = b < sh.nblk ? ld_block_stream(x + b) : zero_block();
    }
  }
  if (sh.G == 1) {
    run = __reduce_max_sync(0xFFFFFFFFu, run);
    if ((threadIdx.x & 31) == 0 && run) atomicMax(&table[0], run);
  } else {
    flush(run_g, run);
  }
  __syncthreads();
  if (sh.G == 1) {
    if (threadIdx.x == 0 && table[0]) atomicMax(&amax[0], table[0]);
    return;
  }
  for (int i = threadIdx.x; i < kAmaxTable; i += kThreads) {
    const uint32_t val = table[i];
    if (val && g_first + i < sh.G) atomicMax(&amax[g_first + i], val);
  }
}

// ---------------------------------------------------------------------------
// Kernel 2: capture.  Per 16-element block: E4M3 scale; per element: the
// round-to-nearest code and its mantissa bit.
// ---------------------------------------------------------------------------
// Scale bytes of a pair of blocks: t = bmax / RN(6 s_g), E4M3
// round-to-nearest-even, satfinite.  Returns s0 | s1 << 8.
__device__ __forceinline__ uint32_t pair_scale_bytes(const V8& v0, const V8& v1, const GroupK& gk) {
  const float b0 = __uint_as_float(absmax_block(v0) << 16);
  const float b1 = __uint_as_float(absmax_block(v1) << 16);
  float t0, t1;
  if (gk.fast6) {
    const u64 bb = pk(b0, b1), rr = pk(gk.r6, gk.r6);
    const u64 q0 = mul2(bb, rr);
    upk(fma2(fma2(q0, pk(-gk.den6, -gk.den6), bb), rr, q0), t0, t1);
  } else {
    t0 = __fdiv_rn(b0, gk.den6);
    t1 = __fdiv_rn(b1, gk.den6);
  }
  return cvt_e4m3(t0) | (cvt_e4m3(t1) << 8);
}

// Codes of one block whose scale d is on the fast path: c0 elements 0-7,
// c1 8-15.
// The quotient runs negated: with q0' = RN(x * -r), e = x + q0' d (exact)
// and z' = RN(q0' + e * -r), z' = -RN(x / d) by the symmetry of
// round-to-nearest, and a zero quotient keeps the opposite of x's sign
// (x = +-0 and underflows alike), which the unnegated step loses for
// x = -0.  The codes of z' with every sign bit flipped are the codes of
// RN(x / d) with x's sign (cvt ... satfinite is odd in its input).
__device__ __forceinline__ void codes_fast(const V8& v, float d, uint32_t& c0, uint32_t& c1) {
  const float r = __frcp_rn(d);
  const u64 nrr = pk(-r, -r), dd = pk(d, d);
  float z[16];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t w = v.w[k];
    const u64 xx = pk(bf16_lo(w), bf16_hi(w));
    const u64 q0 = mul2(xx, nrr);
    upk(fma2(fma2(q0, dd, xx), nrr, q0), z[2 * k], z[2 * k + 1]);
  }
  c0 = cvt_e2m1x8(z) ^ 0x88888888u;
  c1 = cvt_e2m1x8(z + 8) ^ 0x88888888u;
}

// Codes of one block with any scale d: zero block, fast path or exact path.
__device__ __forceinline__ void codes_block(const V8& v, const V8* src, float d, uint32_t& c0,
                                            uint32_t& c1) {
  if (d == 0.0f) {
    // zero block: z = +-0, code = sign only
    c0 = c1 = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t w = v.w[k];
      const uint32_t nib = (((w >> 15) & 1u) << 3) | ((w >> 31) << 7);
      if (k < 4) c0 |= nib << (8 * k); else c1 |= nib << (8 * (k - 4));
    }
  } else if (fast_scale(d)) {
    codes_fast(v, d, c0, c1);
  } else {
    const uint2 c = capture_block_exact(src, d);
    c0 = c.x;
    c1 = c.y;
  }
}

// Each thread owns two adjacent blocks: one 16-byte store of codes, one
// 32-bit store of mantissa bits, one 16-bit store of scales.
// SW: scales in the tiled layout of a block-scaled GEMM instead of row-major.
// The quantising pass given the per-group amax words (of a sharded or
// chunk-streamed tensor): the group constants are computed from them, and
// this pass writes gscale.
template <bool SW>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_capture(const V8* __restrict__ x, Shape sh, const int64_t* __restrict__ offs,
              const uint32_t* __restrict__ amax, uint4* __restrict__ codes,
              uint32_t* __restrict__ mbits, uint8_t* __restrict__ scales,
              float* __restrict__ gscale) {
  pdl_begin();
  GroupCursor gc;
  gc.init(offs, sh.G);
  GroupK gk = {1.0f, 6.0f, 0.0f, false};  // set at the first block (seek)
  // tiles in reverse order: an amax pass just before read the high tiles
  // last, so they are the most likely to be still in L2.  The first tile's
  // loads go out before anything else.
  uint32_t i = blockIdx.x;
  auto tile_base = [&](uint32_t k) { return (sh.ntiles - 1u - k) * kTileBlks + 2u * threadIdx.x; };
  V8 v0 = zero_block(), v1 = zero_block();
  if (i < sh.ntiles && tile_base(i) < sh.nblk) {
    v0 = ld_block_stream(x + tile_base(i));
    v1 = ld_block_stream(x + tile_base(i) + 1);
  }
  // global scales of all groups (any CTA may write them; all write the same)
  for (int g = blockIdx.x * kThreads + threadIdx.x; g < sh.G; g += gridDim.x * kThreads)
    gscale[g] = group_consts(__ldcg(amax + g)).s_g;

  for (; i < sh.ntiles; i += gridDim.x) {
    const uint32_t b = tile_base(i);  // even; nblk is even
    const uint32_t inext = i + gridDim.x;
    if (b < sh.nblk) {
      // both blocks of the pair are in the same row (cols is a multiple of 32)
      const uint32_t row = (SW || sh.G > 1) ? fastdiv(b, sh.bpr) : 0u;
      if (gc.seek(row)) gk = group_consts(__ldcg(amax + gc.g));
      const uint32_t s2 = pair_scale_bytes(v0, v1, gk);
      float sb0, sb1;
      e4m3x2_to_f32(s2, sb0, sb1);
      const float d0 = __fmul_rn(gk.s_g, sb0), d1 = __fmul_rn(gk.s_g, sb1);
      uint4 c;
      if (fast_scale(d0) && fast_scale(d1)) {  // the common case, without per-block branches
        codes_fast(v0, d0, c.x, c.y);
        codes_fast(v1, d1, c.z, c.w);
      } else {
        codes_block(v0, x + b, d0, c.x, c.y);
        codes_block(v1, x + b + 1, d1, c.z, c.w);
      }
      codes[b >> 1] = c;
      mbits[b >> 1] = nibble_lsbs4(c);
      const uint16_t sv = (uint16_t)s2;
      if (SW)  // the pair's two columns are neighbours inside one tile
        *reinterpret_cast<uint16_t*>(scales + tiled_scale_offset(row, b - row * sh.bpr.d, sh.sw_ct)) = sv;
      else
        reinterpret_cast<uint16_t*>(scales)[b >> 1] = sv;
    }
    if (inext < sh.ntiles && tile_base(inext) < sh.nblk) {
      v0 = ld_block_stream(x + tile_base(inext));
      v1 = ld_block_stream(x + tile_base(inext) + 1);
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 2': capture in one launch.  A cooperative grid (every CTA resident
// at once, at most a few per SM): each CTA reduces the amax of its tiles --
// one contiguous range of tiles per CTA, so that a CTA meets few groups --
// into the accumulators, the CTAs meet at a grid barrier, and each CTA then
// quantises the same tiles in reverse order, so that it starts on what it
// read last (in L2 on tensors that fit there).  The barrier's last arriving
// CTA takes each group's final amax, zeroes its accumulator, writes s_g to
// gscale and releases the others, which read their constants from gscale.
// Workspace (u32): [0] arrival count (zero between calls), [1] generation
// (counts calls), [2] error flag (set if a CTA gave up waiting), [3] unused,
// [4, 4 + G) the accumulators (zero between calls).
// ---------------------------------------------------------------------------
template <bool SW>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_capture_coop(const V8* __restrict__ x, Shape sh, const int64_t* __restrict__ offs,
                   uint32_t* __restrict__ ws, uint4* __restrict__ codes,
                   uint32_t* __restrict__ mbits, uint8_t* __restrict__ scales,
                   float* __restrict__ gscale) {
  __shared__ uint32_t table[kAmaxTable];
  __shared__ int g_first_s;
  __shared__ uint32_t gen_s, last_s, ok_s;
  pdl_begin();
  uint32_t* const cnt = ws;
  uint32_t* const gen = ws + 1;
  uint32_t* const err = ws + 2;
  uint32_t* const acc = ws + 4;
  // this CTA's tiles: [t0, t1), nonempty when there are tiles (the grid has
  // at most one CTA per tile)
  const uint32_t t0 = (uint32_t)((uint64_t)blockIdx.x * sh.ntiles / gridDim.x);
  const uint32_t t1 = (uint32_t)((uint64_t)(blockIdx.x + 1u) * sh.ntiles / gridDim.x);

  // ---- phase 1: amax of the CTA's tiles, three in flight per thread (the
  // quantising phase sets the register budget, so they cost no occupancy);
  // the first loads go out before the set-up
  V8 a0, a1, b0, b1, c0, c1;
  auto load = [&](uint32_t t, V8& v0, V8& v1) {
    const uint32_t b = t * kTileBlks + threadIdx.x;
    v0 = (t < t1 && b < sh.nblk) ? ld_block_stream(x + b) : zero_block();
    v1 = (t < t1 && b + kThreads < sh.nblk) ? ld_block_stream(x + b + kThreads) : zero_block();
  };
  load(t0, a0, a1);
  load(t0 + 1u, b0, b1);
  load(t0 + 2u, c0, c1);
  GroupCursor gc;
  gc.init(offs, sh.G);
  if (threadIdx.x == 0) gen_s = ld_acquire_gpu(gen);  // before this CTA's arrival
  if (sh.G > 1) {
    if (threadIdx.x == 0) {
      gc.seek(t0 < t1 ? fastdiv(t0 * kTileBlks, sh.bpr) : 0u);
      g_first_s = gc.g;
    }
    for (int i = threadIdx.x; i < kAmaxTable; i += kThreads) table[i] = 0u;
  } else if (threadIdx.x == 0) {
    table[0] = 0u;
    g_first_s = 0;
  }
  __syncthreads();
  const int g_first = g_first_s;
  gc.init(offs, sh.G);
  uint32_t run = 0u;
  int run_g = sh.G > 1 ? -1 : 0;
  auto flush = [&](int g, uint32_t val) {
    if (g < 0 || val == 0u) return;
    const int slot = g - g_first;
    if (slot >= 0 && slot < kAmaxTable) atomicMax(&table[slot], val);
    else atomicMax(&acc[g], val);
  };
  auto take = [&](uint32_t t, const V8& v0, const V8& v1) {
    if (sh.G == 1) {  // blocks past the end were loaded as zeros
      run = max(run, max(absmax_block(v0), absmax_block(v1)));
      return;
    }
    const uint32_t b = t * kTileBlks + threadIdx.x;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t bu = b + u * kThreads;
      if (bu >= sh.nblk) continue;
      gc.seek(fastdiv(bu, sh.bpr));
      if (gc.g != run_g) {
        flush(run_g, run);
        run = 0u;
        run_g = gc.g;
      }
      run = max(run, absmax_block(u == 0 ? v0 : v1));
    }
  };
  for (uint32_t t = t0; t < t1; t += 3u) {
    take(t, a0, a1);
    load(t + 3u, a0, a1);
    if (t + 1u >= t1) break;
    take(t + 1u, b0, b1);
    load(t + 4u, b0, b1);
    if (t + 2u >= t1) break;
    take(t + 2u, c0, c1);
    load(t + 5u, c0, c1);
  }
  if (sh.G == 1) {
    run = __reduce_max_sync(0xFFFFFFFFu, run);
    if ((threadIdx.x & 31) == 0 && run) atomicMax(&table[0], run);
  } else {
    flush(run_g, run);
  }
  __syncthreads();
  if (sh.G == 1) {
    if (threadIdx.x == 0 && table[0]) atomicMax(&acc[0], table[0]);
  } else {
    for (int i = threadIdx.x; i < kAmaxTable; i += kThreads) {
      const uint32_t val = table[i];
      if (val && g_first + i < sh.G) atomicMax(&acc[g_first + i], val);
    }
  }

  // phase 2's first tile (the last one read) is loaded before the barrier,
  // so that the wait covers its latency; x is not written by this kernel
  const uint32_t ntile_cta = t1 - t0;
  auto tile_base = [&](uint32_t k) { return (t0 + k) * kTileBlks + 2u * threadIdx.x; };
  V8 v0 = zero_block(), v1 = zero_block();
  if (ntile_cta > 0u && tile_base(ntile_cta - 1u) < sh.nblk) {
    v0 = ld_block_stream(x + tile_base(ntile_cta - 1u));
    v1 = ld_block_stream(x + tile_base(ntile_cta - 1u) + 1);
  }

  // ---- grid barrier
  __threadfence();  // this thread's maxima before the CTA's arrival
  __syncthreads();
  if (threadIdx.x == 0) {
    last_s = atomicAdd(cnt, 1u) == gridDim.x - 1u;
    ok_s = 1u;
  }
  __syncthreads();
  if (last_s) {
    __threadfence();
#pragma unroll 4
    for (int g = threadIdx.x; g < sh.G; g += kThreads) {
      const uint32_t a = __ldcg(acc + g);
      acc[g] = 0u;
      gscale[g] = group_consts(a).s_g;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      *cnt = 0u;
      __threadfence();  // the global scales and the reset before the release
      st_release_gpu(gen, gen_s + 1u);
    }
  } else if (threadIdx.x == 0) {
    uint32_t polls = 0u;
    while (ld_acquire_gpu(gen) == gen_s) {
      if (++polls >= kBarrierPolls) {
        atomicExch(err, 1u);
        ok_s = 0u;
        break;
      }
      __nanosleep(256);
    }
  }
  __syncthreads();
  if (!ok_s) return;

  // ---- phase 2: quantise the same tiles, last first; two adjacent blocks
  // per thread
  gc.init(offs, sh.G);
  GroupK gk = {1.0f, 6.0f, 0.0f, false};  // set at the first block (seek)
  for (uint32_t k = ntile_cta; k-- > 0u;) {
    const uint32_t b = tile_base(k);  // even; nblk is even
    if (b < sh.nblk) {
      const uint32_t row = (SW || sh.G > 1) ? fastdiv(b, sh.bpr) : 0u;
      if (gc.seek(row)) gk = group_consts_of_sg(__ldcg(gscale + gc.g));
      const uint32_t s2 = pair_scale_bytes(v0, v1, gk);
      float sb0, sb1;
      e4m3x2_to_f32(s2, sb0, sb1);
      const float d0 = __fmul_rn(gk.s_g, sb0), d1 = __fmul_rn(gk.s_g, sb1);
      uint4 c;
      if (fast_scale(d0) && fast_scale(d1)) {
        codes_fast(v0, d0, c.x, c.y);
        codes_fast(v1, d1, c.z, c.w);
      } else {
        codes_block(v0, x + b, d0, c.x, c.y);
        codes_block(v1, x + b + 1, d1, c.z, c.w);
      }
      codes[b >> 1] = c;
      mbits[b >> 1] = nibble_lsbs4(c);
      const uint16_t sv = (uint16_t)s2;
      if (SW)
        *reinterpret_cast<uint16_t*>(scales + tiled_scale_offset(row, b - row * sh.bpr.d, sh.sw_ct)) = sv;
      else
        reinterpret_cast<uint16_t*>(scales)[b >> 1] = sv;
    }
    if (k > 0u && tile_base(k - 1u) < sh.nblk) {
      v0 = ld_block_stream(x + tile_base(k - 1u));
      v1 = ld_block_stream(x + tile_base(k - 1u) + 1);
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 3/5: fake-quant forward with given scales: bf16 q*·s and the STE
// mask, q* chosen by round-to-nearest, by the cached mantissa bit, or by the
// whole rollout code.
// ---------------------------------------------------------------------------
// Fake-quant modes: round to nearest (vanilla QAT), 1-bit guided (TRACE's
// compact cache), full-information guided (the cache keeps the whole code).
enum FqMode { kRtn = 0, kGuided = 1, kFull = 2 };

// Round to nearest over one fast-path block (d in [2^-90, 2^100], block
// constants k): bf16 outputs q*s with x's sign, the 16 STE mask bits, and
// with KIND 1 the 16
// magnitude codes, with KIND 2 the 16 codes signed with x's sign (c0:
// elements 0-7, c1: 8-15, element j in nibble j % 8); KIND 0 returns no
// codes.
template <int KIND>
__device__ __forceinline__ void rtn_block(const V8& v, const BlkK& k, V8& o, uint32_t& m,
                                          uint32_t& c0, uint32_t& c1) {
  // the quotient is taken of |x| (the sign is put back on the output), and
  // the mask bits are accumulated on the FMA pipe as a float, Horner style
  // from the last pair down: bit 2p of mf.lo, bit 2p of mf.hi (element
  // 2p + 1) -- exact, every partial sum stays below 2^16
  u64 mf = pk(0.0f, 0.0f);
  const u64 four = pk(4.0f, 4.0f);
  c0 = 0u;
  c1 = 0u;
#pragma unroll
  for (int p = 7; p >= 0; --p) {
    const uint32_t w = v.w[p];
    float zl, zh;
    upk(quot2(pk(__uint_as_float((w & 0x7FFFu) << 16), __uint_as_float(w & 0x7FFF0000u)), k),
        zl, zh);  // z >= 0; NaN where |x| / d overflows
    mf = fma2(mf, four, pk(le6_step(zl), le6_step(zh)));
    float al = fminf(zl, 6.0f), ah = fminf(zh, 6.0f);  // NaN -> 6
    uint32_t h2;
    if (KIND == 0) {
      // round to nearest on the grid (ties to the even code), decoded
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
    const float vl = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
    const float vh = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
    float ql, qh;
    upk(mul2(mul2(pk(vl, vh), k.sbv2), k.sg2), ql, qh);
    o.w[p] = cvt_bf16x2(ql, qh) | (w & 0x80008000u);
  }
  float ml, mh;
  upk(mf, ml, mh);
  m = __float2uint_rn(__fmaf_rn(mh, 2.0f, ml));
}

// Lowest bit of each of the 16 nibbles of (c0, c1) in bits 0-15 (bit j =
// nibble j); bits 16-31 are not defined.  Multiply-gather as nibble_lsbs4.
__device__ __forceinline__ uint32_t nibble_lsbs2(uint32_t c0, uint32_t c1) {
  const uint32_t kGather = (1u << 24) | (1u << 18) | (1u << 12) | (1u << 6);
  const uint32_t t0 = ((c0 & 0x01010101u) | ((c0 >> 3) & 0x02020202u)) * kGather;
  const uint32_t t1 = ((c1 & 0x01010101u) | ((c1 >> 3) & 0x02020202u)) * kGather;
  return __byte_perm(t0, t1, 0x0073u);
}

// Bit j (0-15) set where nibble j of (c0, c1) is nonzero.
__device__ __forceinline__ uint32_t nibble_any2(uint32_t c0, uint32_t c1) {
  c0 |= c0 >> 1;
  c1 |= c1 >> 1;
  return nibble_lsbs2(c0 | (c0 >> 2), c1 | (c1 >> 2)) & 0xFFFFu;
}

// Two elements (one bf16x2 word w) of a guided rule, for d in [2^-90, 2^16]:
// z * 2^64 exact (|x| * 2^64 keeps every nonzero bf16's quotient and
// remainder normal there, so "z is exactly zero" is decided exactly), floor
// and ceiling by directed rounding with the grid addend, then the rule's
// choice.  side: kGuided -- the two cached bits in bits 0 and 1; kFull -- the
// rollout's two codes (low nibble first).  k: the block's constants with
// s_b scaled by 2^-64.  Returns the pair's bf16 outputs with x's signs.
template <int MODE>
__device__ __forceinline__ uint32_t guided_pair(uint32_t w, uint32_t side, const BlkK& k) {
  const u64 xx = pk(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  float zl, zh;
  upk(quot2(mul2(xx, pk(kXs, kXs)), k), zl, zh);
  const float al = fminf(fabsf(zl), kSixS), ah = fminf(fabsf(zh), kSixS);  // NaN -> 6 * 2^64
  const u64 MM = MODE == kGuided ? grid_magic_s2(al, ah) : pk(grid_magic_s(al), grid_magic_s(ah));
  const u64 aa = pk(al, ah);
  float lol, loh, hil, hih;
  upk(add_rm2(aa, MM), lol, loh);
  upk(add_rp2(aa, MM), hil, hih);
  float ql, qh;
  if (MODE == kGuided) {
    // of floor / ceiling, the one whose mantissa bit is the cached bit: the
    // bits of the two sums differ by 0 (a on the grid) or 1, and the lowest
    // bit of the floor sum is its codeword's mantissa bit
    const uint32_t lb = __float_as_uint(lol), hb = __float_as_uint(loh);
    const float tl = __uint_as_float(lb + ((lb ^ side) & (__float_as_uint(hil) - lb)));
    const float th = __uint_as_float(hb + ((hb ^ (side >> 1)) & (__float_as_uint(hih) - hb)));
    upk(mul2(mul2(sub2(pk(tl, th), MM), k.sbv2), k.sg2), ql, qh);
  } else {
    // of floor / ceiling, the one nearest the rollout codeword: the rollout
    // value reflected to z's side of zero picks the ceiling exactly when it
    // lies above the floor (no codeword lies between)
    float fl, fh, cl, ch;
    upk(sub2(pk(lol, loh), MM), fl, fh);
    upk(sub2(pk(hil, hih), MM), cl, ch);
    const uint32_t h2 = e2m1x2_to_f16x2(side & 0xFFu);
    float rl = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
    float rh = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
    rl = __uint_as_float(__float_as_uint(rl) ^ ((w << 16) & 0x80000000u));
    rh = __uint_as_float(__float_as_uint(rh) ^ (w & 0x80000000u));
    upk(mul2(pk(rl, rh), pk(kXs, kXs)), rl, rh);
    const float tl = rl > fl ? cl : fl;
    const float th = rh > fh ? ch : fh;
    upk(mul2(mul2(pk(tl, th), k.sbv2), k.sg2), ql, qh);
  }
  return cvt_bf16x2(ql, qh) | (w & 0x80008000u);
}

// Word p (0-7) of a block, and a block with word p replaced, by selects (no
// indexed access, which would put the block in local memory).
__device__ __forceinline__ uint32_t pick_word(const V8& v, int p) {
  uint32_t w = v.w[0];
#pragma unroll
  for (int k = 1; k < 8; ++k) w = (p == k) ? v.w[k] : w;
  return w;
}
__device__ __forceinline__ void put_word(V8& v, int p, uint32_t w) {
#pragma unroll
  for (int k = 0; k < 8; ++k) v.w[k] = (p == k) ? w : v.w[k];
}

// One fast-path block of the fake-quant forward: bf16 outputs in o, the 16
// mask bits in m.  The guided rules (MODE kGuided: bits16 = the block's
// cached bits; kFull: r0, r1 = its rollout codes, elements 0-7 and 8-15)
// start from round to nearest, which is one of the two codewords around z,
// and keep it wherever the rule agrees with it: the 1-bit rule wherever its
// mantissa bit equals the cached bit (the bracket member with that bit, or
// the collapsed bracket), the full rule wherever its code equals the
// rollout's (the rollout codeword itself is then in the bracket).  The pairs
// holding a site where they disagree -- where the training and rollout sides
// round differently, rare for a drifted pair -- are recomputed with the
// rule's own pair routine, from registers; for d beyond 2^16 (outside that
// routine's range) such sites go through the exact per-site path, reading
// the block's inputs at src (o is stored by the caller afterwards, so out
// may alias x).
// The round-to-nearest pass of fq_block_fast alone: outputs and mask, and
// the returned bits of the sites where the block's rule disagrees with it.
template <int MODE>
__device__ __forceinline__ uint32_t fq_block_rtn(const V8& v, uint32_t bits16, uint32_t r0,
                                                 uint32_t r1, const BlkK& k, V8& o, uint32_t& m) {
  uint32_t c0, c1;
  rtn_block<MODE == kRtn ? 0 : MODE == kGuided ? 1 : 2>(v, k, o, m, c0, c1);
  if (MODE == kRtn) return 0u;
  return MODE == kGuided ? (nibble_lsbs2(c0, c1) ^ bits16) & 0xFFFFu : nibble_any2(c0 ^ r0, c1 ^ r1);
}

template <int MODE>
__device__ __forceinline__ void fq_block_fast(const V8& v, const uint16_t* src, uint32_t bits16,
                                              uint32_t r0, uint32_t r1, float d, float sbv,
                                              float s_g, V8& o, uint32_t& m) {
  BlkK k = make_blk(d, sbv, s_g);
  uint32_t bad = fq_block_rtn<MODE>(v, bits16, r0, r1, k, o, m);
  if (MODE == kRtn || bad == 0u) return;
  if (fast_scale(d, kDMaxExactZ)) {
    k.sbv2 = mul2(k.sbv2, pk(0x1p-64f, 0x1p-64f));  // exact
    uint32_t pairs = (bad | (bad >> 1)) & 0x5555u;
    while (pairs != 0u) {
      const int p = (__ffs(pairs) - 1) >> 1;
      pairs &= pairs - 1u;
      const uint32_t side = MODE == kGuided ? bits16 >> (2 * p)
                                            : (p < 4 ? r0 : r1) >> (8 * (p & 3));
      put_word(o, p, guided_pair<MODE>(pick_word(v, p), side, k));
    }
    return;
  }
  while (bad != 0u) {
    const int j = __ffs(bad) - 1;
    bad &= bad - 1u;
    const uint32_t side = MODE == kGuided ? (bits16 >> j) & 1u
                                          : ((j < 8 ? r0 : r1) >> (4 * (j & 7))) & 0xFu;
    const uint32_t val = guided_site_fix(src + j, d, sbv, s_g, side, MODE);
    const uint32_t sh = 16u * (uint32_t)(j & 1), keep = 0xFFFF0000u >> sh;
    const int p = j >> 1;
    put_word(o, p, (pick_word(o, p) & keep) | (val << sh));
  }
}

// Pair q (0-15) of a thread's two blocks recomputed with its guided rule
// and stored over the round-to-nearest word already written at out: the
// variant for outputs that do not alias the inputs, so the pair's input word
// is read back from x (a cache hit: the block was just read) instead of kept
// in registers.  d, sbv: the pair's block; side as guided_pair (MODE kGuided:
// the pair's two cached bits in bits 0 and 1; kFull: its two rollout codes).
// r: RN(1/d), as the round-to-nearest pass took it.
template <int MODE>
__device__ __forceinline__ void patch_pair(const uint32_t* xw, uint32_t* ow, int q, float d,
                                           float r, float sbv, float s_g, uint32_t side) {
  if (fast_scale(d, kDMaxExactZ)) {
    BlkK k;
    k.rr = pk(r, r);
    k.ndd = pk(-d, -d);
    const float sbs = __fmul_rn(sbv, 0x1p-64f);  // exact
    k.sbv2 = pk(sbs, sbs);
    k.sg2 = pk(s_g, s_g);
    ow[q] = guided_pair<MODE>(__ldg(xw + q), side, k);
  } else {
    const uint16_t* src = reinterpret_cast<const uint16_t*>(xw + q);
    const uint32_t lo = guided_site_fix(src, d, sbv, s_g, MODE == kGuided ? side & 1u : side & 0xFu,
                                        MODE);
    const uint32_t hi = guided_site_fix(src + 1, d, sbv, s_g,
                                        MODE == kGuided ? (side >> 1) & 1u : (side >> 4) & 0xFu,
                                        MODE);
    ow[q] = lo | (hi << 16);
  }
}

// One block with any scale (zero block, fast path or exact path): stores its
// output at dst and returns its 16 mask bits.
template <int MODE>
__device__ __forceinline__ uint32_t fake_quant_block(const V8& v, const V8* src, uint32_t bits16,
                                                     uint32_t c0, uint32_t c1, float sbv, float s_g,
                                                     V8* dst) {
  const float d = __fmul_rn(s_g, sbv);
  V8 o;
  uint32_t m;
  if (d == 0.0f) {
    // zero block: z = +-0, output +-0, mask set
#pragma unroll
    for (int k = 0; k < 8; ++k) o.w[k] = v.w[k] & 0x80008000u;
    m = 0xFFFFu;
  } else if (fast_scale(d)) {
    fq_block_fast<MODE>(v, reinterpret_cast<const uint16_t*>(src), bits16, c0, c1, d, sbv, s_g,
                        o, m);
  } else {
    return fake_quant_block_exact(src, d, sbv, s_g, bits16, c0, c1, MODE, dst);
  }
  st_block(dst, o);
  return m;
}

// Each thread owns two adjacent blocks, so their mantissa bits, scales and
// mask move as one 32-bit / 16-bit / 32-bit access (the full codes as one
// 16-byte access).
// MINB: resident CTAs per SM the register budget is cut for.  The
// full-information forward has a second build at 2 CTAs per SM for large
// tensors: each thread then walks several tiles, and with the larger register
// budget it ran 16% faster on B200 at 268M elements (and 13% slower at 33M,
// where a thread sees one tile).
// SEP: out does not alias x.  The guided rules then write both blocks'
// round-to-nearest outputs first and recompute the pairs that need it in one
// loop for the thread's 32 elements, reading their inputs back from x.
template <int MODE, bool SW, int MINB = kCtasPerSm, bool SEP = false>
__global__ void __launch_bounds__(kThreads, MINB)
    k_fake_quant(const V8* __restrict__ x, Shape sh, const int64_t* __restrict__ offs,
                 const uint32_t* __restrict__ mbits, const uint4* __restrict__ rcodes,
                 const uint8_t* __restrict__ scales, const float* __restrict__ gscale,
                 V8* __restrict__ out, uint32_t* __restrict__ mask) {
  pdl_begin();
  GroupCursor gc;
  gc.init(offs, sh.G);
  float s_g = 1.0f;

  for (uint32_t t = blockIdx.x; t < sh.ntiles; t += gridDim.x) {
    const uint32_t b = t * kTileBlks + 2u * threadIdx.x;  // even; nblk is even
    if (b >= sh.nblk) continue;
    // with separate outputs the guided rules read words of x back (the
    // pairs they recompute): keep the blocks in L1 for that
    constexpr bool kKeepL1 = SEP && MODE != kRtn;
    const V8 v0 = kKeepL1 ? ld_block_l1(x + b) : ld_block_stream(x + b);
    const V8 v1 = kKeepL1 ? ld_block_l1(x + b + 1) : ld_block_stream(x + b + 1);
    const uint32_t bits = MODE == kGuided ? __ldcs(mbits + (b >> 1)) : 0u;
    const uint4 rc = MODE == kFull ? __ldcs(rcodes + (b >> 1)) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t row = (SW || sh.G > 1) ? fastdiv(b, sh.bpr) : 0u;
    const uint32_t sb2 =
        SW ? __ldcs(reinterpret_cast<const unsigned short*>(
                 scales + tiled_scale_offset(row, b - row * sh.bpr.d, sh.sw_ct)))
           : __ldcs(reinterpret_cast<const unsigned short*>(scales) + (b >> 1));
    if (gc.seek(row)) s_g = __ldg(gscale + gc.g);
    uint32_t m0, m1;
    float sbv0, sbv1;
    e4m3x2_to_f32(sb2, sbv0, sbv1);
    // a row holds a whole number of 32-element words, so both blocks of the
    // pair are in the same row and group
    const float d0 = __fmul_rn(s_g, sbv0), d1 = __fmul_rn(s_g, sbv1);
    if (SEP && MODE != kRtn && fast_scale(d0) && fast_scale(d1)) {
      // the common case for separate output buffers
      V8 o;
      const BlkK k0 = make_blk(d0, sbv0, s_g);
      const uint32_t bad0 = fq_block_rtn<MODE>(v0, bits & 0xFFFFu, rc.x, rc.y, k0, o, m0);
      st_block(out + b, o);
      const BlkK k1 = make_blk(d1, sbv1, s_g);
      const uint32_t bad1 = fq_block_rtn<MODE>(v1, bits >> 16, rc.z, rc.w, k1, o, m1);
      st_block(out + b + 1, o);
      float r0, r1, unused;
      upk(k0.rr, r0, unused);
      upk(k1.rr, r1, unused);
      uint32_t pairs = ((bad0 | (bad0 >> 1)) & 0x5555u) | (((bad1 | (bad1 >> 1)) & 0x5555u) << 16);
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(x + b);
      uint32_t* ow = reinterpret_cast<uint32_t*>(out + b);
      while (pairs != 0u) {
        const int q = (__ffs(pairs) - 1) >> 1;  // pair q & 7 of block q >> 3
        pairs &= pairs - 1u;
        const uint32_t side =
            MODE == kGuided ? bits >> (2 * q)
                            : (q < 4 ? rc.x : q < 8 ? rc.y : q < 12 ? rc.z : rc.w) >> (8 * (q & 3));
        patch_pair<MODE>(xw, ow, q, q < 8 ? d0 : d1, q < 8 ? r0 : r1, q < 8 ? sbv0 : sbv1, s_g,
                         side);
      }
    } else if (fast_scale(d0) && fast_scale(d1)) {
      // the common case, without per-block branches
      V8 o;
      const uint16_t* src = reinterpret_cast<const uint16_t*>(x + b);
      fq_block_fast<MODE>(v0, src, bits & 0xFFFFu, rc.x, rc.y, d0, sbv0, s_g, o, m0);
      st_block(out + b, o);
      fq_block_fast<MODE>(v1, src + 16, bits >> 16, rc.z, rc.w, d1, sbv1, s_g, o, m1);
      st_block(out + b + 1, o);
    } else {
      m0 = fake_quant_block<MODE>(v0, x + b, bits & 0xFFFFu, rc.x, rc.y, sbv0, s_g, out + b);
      m1 = fake_quant_block<MODE>(v1, x + b + 1, bits >> 16, rc.z, rc.w, sbv1, s_g, out + b + 1);
    }
    mask[b >> 1] = m0 | (m1 << 16);
  }
}

// ---------------------------------------------------------------------------
// Kernel 4: masked straight-through backward.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_ste_bwd(const V8* __restrict__ g, Shape sh, const uint32_t* __restrict__ mask,
              V8* __restrict__ gin) {
  pdl_begin();
  for (uint32_t t = blockIdx.x; t < sh.ntiles; t += gridDim.x) {
    const uint32_t b = t * kTileBlks + 2u * threadIdx.x;  // two adjacent blocks
    if (b >= sh.nblk) continue;
    const V8 v0 = ld_block_stream(g + b), v1 = ld_block_stream(g + b + 1);
    const uint32_t m = __ldcs(mask + (b >> 1));
    V8 r0, r1;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      // bits (2k, 2k+1) -> keep masks of the two halves of word k
      r0.w[k] = v0.w[k] & ((((m >> (2 * k)) & 1u) * 0x0000FFFFu) |
                           (((m >> (2 * k + 1)) & 1u) * 0xFFFF0000u));
      r1.w[k] = v1.w[k] & ((((m >> (2 * k + 16)) & 1u) * 0x0000FFFFu) |
                           (((m >> (2 * k + 17)) & 1u) * 0xFFFF0000u));
    }
    st_block(gin + b, r0);
    st_block(gin + b + 1, r1);
  }
}
