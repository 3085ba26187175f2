// trace_fp4.cu -- B200 (sm_100a) kernels and C ABI for TRACE rollout-guided
// NVFP4 rounding: rollout capture of the compact cache, the guided QAT
// fake-quant forward, the masked straight-through backward and the
// round-to-nearest comparator.
//
// Method: rcap.io post "TRACE: Rollout-Guided Quantization-Aware Training for
// FP4" (2026-10-06), sections "rollout-guided rounding" and "compact cache"
// and its pseudocode listing (capture; QAT forward).  The number format and
// the layouts are documented in include/trace_fp4.h.
//
// Design (everything here is HBM-bound elementwise work; no tensor cores):
//   * x is streamed as 16-byte vectors of 8 bf16; a CTA of 256 threads works
//     on tiles of 1024 vectors (16 KiB), 4 vectors per thread with all loads
//     issued before any use; each CTA owns one contiguous range of tiles and
//     the grid is a multiple of the SM count.  Two neighbouring lanes hold
//     the two halves of a 16-element scale block.
//   * Capture is a two-pass grid amax: kernel 1 reduces max|x| per group
//     (shared-memory table per CTA, one global atomicMax per group per CTA
//     into a zeroed workspace); kernel 2 walks the same tiles in REVERSE
//     order, so it starts on the data kernel 1 touched last and finds much of
//     x still in the 126 MB L2.
//   * Division-free fast path.  z = fl(x / d) (d = fl(s_g * s_b)) is needed
//     only through comparisons with the codewords, the midpoints and 6, all
//     of which have their low 21 fp32 bits zero.  za = fl(|x| * fl(1/d)) is
//     within 6 units in the last place of fl(|x|/d); when za is more than 16
//     units away from every number whose low 21 bits are zero, za and
//     fl(|x|/d) fall strictly inside the same interval between critical
//     points, so every decision taken on za is the one the exact quotient
//     gives.  The rest (za near a critical point, tiny quotients, zero
//     blocks, scales outside [2^-120, 2^120]) takes the exact path, which
//     divides with IEEE round-to-nearest (__fdiv_rn), as the format states.
//   * Outputs: codes as one 32-bit store per vector, mantissa bits and STE
//     mask as one byte per vector (lane l writes byte l: a warp fills one
//     32-byte sector), block scales as one byte per block.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "trace_fp4.h"

namespace {

constexpr int kThreads = 256;
constexpr int kVecPerThread = 4;
constexpr int kTileVecs = kThreads * kVecPerThread;  // 1024 vectors = 8192 elements
constexpr int kCtasPerSm = 4;
constexpr int kAmaxTable = 256;  // groups per CTA kept in shared memory

// Critical-point window, in fp32 units in the last place (see header).
constexpr uint32_t kNearWin = 16u;
constexpr uint32_t kLow21 = 0x1FFFFFu;
constexpr uint32_t kSix = 0x40C00000u;        // 6.0f
constexpr uint32_t kTinyZ = 0x0D800000u;      // 2^-100
constexpr uint32_t kDMin = 0x03800000u;       // 2^-120
constexpr uint32_t kDMax = 0x7B800000u;       // 2^120

// ---------------------------------------------------------------------------
// Fast unsigned 32-bit division by a runtime constant (Granlund & Montgomery,
// "Division by invariant integers using multiplication", PLDI 1994, the
// round-up method with the add-back step), used to map a vector index to its
// row when there are several groups.
// ---------------------------------------------------------------------------
struct FastDiv {
  uint32_t d, m, s;  // s = ceil(log2 d); d == 1 handled separately
};

FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{d, 0u, 0u};
  if (d <= 1) return f;
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  f.s = l;
  f.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1ull);
  return f;
}

__device__ __forceinline__ uint32_t fastdiv(uint32_t n, const FastDiv& f) {
  if (f.d <= 1) return n;
  uint32_t t = __umulhi(n, f.m);
  return (t + ((n - t) >> 1)) >> (f.s - 1);
}

// ---------------------------------------------------------------------------
// Number-format helpers (hardware conversions from the public PTX ISA).
// ---------------------------------------------------------------------------

// Eight fp32 magnitudes -> eight E2M1 codes (round to nearest even, satfinite)
// packed as nibbles: element j in bits [4j, 4j+4).
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&z)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(z[0]), "f"(z[1]), "f"(z[2]), "f"(z[3]), "f"(z[4]), "f"(z[5]),
        "f"(z[6]), "f"(z[7]));
  return r;
}

// fp32 >= 0 -> E4M3 byte (round to nearest even, saturating at 448).
__device__ __forceinline__ uint32_t cvt_e4m3(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
  return (uint32_t)(r & 0xFFu);
}

// E4M3 byte -> fp32 (exact, through f16).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  uint32_t h2;
  uint16_t in = (uint16_t)b;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// |x| of the 8 elements of a vector as fp32.
__device__ __forceinline__ void abs8(const uint4& v, float (&a)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    a[2 * k] = __uint_as_float((w[k] << 16) & 0x7FFF0000u);
    a[2 * k + 1] = __uint_as_float(w[k] & 0x7FFF0000u);
  }
}

// Sign bits of the 8 elements: bit j = sign of element j.
__device__ __forceinline__ uint32_t signs8(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t s = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    s |= (((w[k] >> 15) & 1u) | ((w[k] >> 30) & 2u)) << (2 * k);
  return s;
}

// max|x| of the 8 elements as bf16 bits (integer order = magnitude order).
__device__ __forceinline__ uint32_t absmax8_bits(const uint4& v) {
  uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                        __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

// Bit j of the result = bit 4j of n (gathers the lowest bit of each nibble).
__device__ __forceinline__ uint32_t nibble_lsbs(uint32_t n) {
  uint32_t c = n & 0x11111111u;
  c = (c | (c >> 3)) & 0x03030303u;
  c = (c | (c >> 6)) & 0x000F000Fu;
  return (c | (c >> 12)) & 0xFFu;
}

// True when za (bits zb) is within kNearWin ulps of a number whose low 21
// bits are zero (every codeword, midpoint and 6 is such a number).
__device__ __forceinline__ bool near_critical(uint32_t zb) {
  return ((zb + kNearWin) & kLow21) < 2u * kNearWin;
}

// ---- exact path: the format's steps with an IEEE division -----------------

struct Exact {
  int rtn;     // round-to-nearest magnitude code of clip(|z|)
  int floor;   // largest code with value <= clip(|z|)
  bool exact;  // clip(|z|) is a codeword (bracket collapses)
  bool in;     // |z| <= 6 (STE mask)
};

__device__ __noinline__ Exact exact_site(float xf, float d) {
  float z = (d == 0.0f) ? copysignf(0.0f, xf) : __fdiv_rn(xf, d);
  float a = fabsf(z);
  Exact e;
  e.in = a <= 6.0f;
  float c = fminf(a, 6.0f);
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

// E2M1 magnitude (as fp32) of a code 0..7.
__device__ __forceinline__ float e2m1_value(int c) {
  return c >= 2 ? __uint_as_float((uint32_t)(c + 252) << 22) : (c == 1 ? 0.5f : 0.0f);
}

// bf16 magnitude of q * s for code c: bf16((VAL[c] * sbv) * s_g).
__device__ __forceinline__ uint32_t dequant_exact(int c, float sbv, float s_g) {
  return f32_to_bf16_bits(__fmul_rn(__fmul_rn(e2m1_value(c), sbv), s_g));
}

// Per-block dequant table for the fast path: for c >= 1 the magnitude is a
// power of two times bf16(s_g*sbv) (even codes and code 1) or times
// bf16((1.5*sbv)*s_g) (odd codes >= 3); both products are one fp32 rounding
// of the exact value, and scaling by 2^j commutes with both roundings while
// the result stays normal, which d in [2^-120, 2^120] guarantees.
__device__ __forceinline__ uint32_t dequant_fast(uint32_t c, uint32_t b1, uint32_t b15) {
  uint32_t base = ((c & 1u) && c >= 3u) ? b15 : b1;
  uint32_t r = base + (((c >> 1) - 1u) << 7);
  return c == 0u ? 0u : (r & 0xFFFFu);
}

// ---------------------------------------------------------------------------
// Group lookup: offsets[g] <= row < offsets[g+1], cached per thread.
// ---------------------------------------------------------------------------
struct GroupCursor {
  const int64_t* offs;
  int G;
  uint32_t lo, hi;  // cached row range of group g
  int g;

  __device__ void init(const int64_t* o, int G_) {
    offs = o;
    G = G_;
    lo = 1u;
    hi = 0u;
    g = 0;
  }
  // returns true when the group changed
  __device__ __forceinline__ bool seek(uint32_t row) {
    if (G == 1) { if (g == 0 && lo == 0u) return false; g = 0; lo = 0u; hi = 0xFFFFFFFFu; return true; }
    if (row >= lo && row < hi) return false;
    int a = 0, b = G;  // last g with offs[g] <= row
    while (b - a > 1) {
      int m = (a + b) >> 1;
      if ((uint64_t)offs[m] <= row) a = m; else b = m;
    }
    g = a;
    lo = (uint32_t)offs[a];
    hi = (uint32_t)offs[a + 1];
    return true;
  }
};

struct Shape {
  uint32_t nvec;    // N / 8
  uint32_t ntiles;  // ceil(nvec / kTileVecs)
  FastDiv vpr;      // vectors per row
  int G;
};

__device__ __forceinline__ void cta_tile_range(const Shape& sh, uint32_t& t0, uint32_t& t1) {
  uint64_t P = gridDim.x, c = blockIdx.x;
  t0 = (uint32_t)((uint64_t)sh.ntiles * c / P);
  t1 = (uint32_t)((uint64_t)sh.ntiles * (c + 1) / P);
}

// ---------------------------------------------------------------------------
// Kernel 0: zero the per-group amax accumulators.
// ---------------------------------------------------------------------------
__global__ void k_zero_u32(uint32_t* p, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = 0u;
}

// ---------------------------------------------------------------------------
// Kernel 1: per-group amax (bits of max|x| as bf16, kept as u32 so that
// atomicMax orders them as magnitudes).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, kCtasPerSm) k_amax(const uint4* __restrict__ x, Shape sh,
                                                   const int64_t* __restrict__ offs,
                                                   uint32_t* __restrict__ amax) {
  __shared__ uint32_t table[kAmaxTable];
  __shared__ int g_first_s;
  uint32_t t0, t1;
  cta_tile_range(sh, t0, t1);
  if (t0 >= t1) return;
  const uint32_t v_first = t0 * kTileVecs;
  const uint32_t v_last = min(t1 * kTileVecs, sh.nvec) - 1u;

  GroupCursor gc;
  gc.init(offs, sh.G);
  if (threadIdx.x == 0) {
    gc.seek(fastdiv(v_first, sh.vpr));
    g_first_s = gc.g;
  }
  for (int i = threadIdx.x; i < kAmaxTable; i += kThreads) table[i] = 0u;
  __syncthreads();
  const int g_first = g_first_s;
  gc.init(offs, sh.G);

  uint32_t run = 0u;
  int run_g = -1;
  auto flush = [&](int g, uint32_t val) {
    if (g < 0 || val == 0u) return;
    int slot = g - g_first;
    if (slot >= 0 && slot < kAmaxTable) atomicMax(&table[slot], val);
    else atomicMax(&amax[g], val);
  };

  for (uint32_t t = t0; t < t1; ++t) {
    uint4 v[kVecPerThread];
    const uint32_t base = t * kTileVecs + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      uint32_t vi = base + u * kThreads;
      v[u] = vi < sh.nvec ? __ldg(x + vi) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      uint32_t vi = base + u * kThreads;
      if (vi >= sh.nvec) continue;
      if (sh.G > 1) {
        gc.seek(fastdiv(vi, sh.vpr));
        if (gc.g != run_g) { flush(run_g, run); run = 0u; run_g = gc.g; }
      } else {
        run_g = 0;
      }
      run = max(run, absmax8_bits(v[u]));
    }
  }
  if (sh.G == 1) {
    // whole CTA feeds one accumulator: warp reduce, then shared, then global
    for (int o = 16; o > 0; o >>= 1) run = max(run, __shfl_xor_sync(0xFFFFFFFFu, run, o));
    if ((threadIdx.x & 31) == 0 && run) atomicMax(&table[0], run);
  } else {
    flush(run_g, run);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kAmaxTable; i += kThreads) {
    uint32_t val = table[i];
    if (val && g_first + i < sh.G) atomicMax(&amax[g_first + i], val);
  }
}

// Global scale from the amax bits: s_g = amax / 2688, or 1 for amax = 0.
__device__ __forceinline__ float global_scale_from(uint32_t amax_bits) {
  float a = __uint_as_float(amax_bits << 16);
  return amax_bits == 0u ? 1.0f : __fdiv_rn(a, 2688.0f);
}

// ---------------------------------------------------------------------------
// Kernel 2: capture.  Per 16-element block: E4M3 scale; per element: the
// round-to-nearest code and its mantissa bit.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, kCtasPerSm) k_capture(const uint4* __restrict__ x, Shape sh,
                                                      const int64_t* __restrict__ offs,
                                                      const uint32_t* __restrict__ amax,
                                                      uint32_t* __restrict__ codes,
                                                      uint8_t* __restrict__ mbits,
                                                      uint8_t* __restrict__ scales,
                                                      float* __restrict__ gscale) {
  // global scales of all groups (any CTA may write them; all write the same)
  for (int g = blockIdx.x * kThreads + threadIdx.x; g < sh.G; g += gridDim.x * kThreads)
    gscale[g] = global_scale_from(amax[g]);

  uint32_t t0, t1;
  cta_tile_range(sh, t0, t1);
  GroupCursor gc;
  gc.init(offs, sh.G);
  float s_g = 1.0f, den6 = 6.0f;
  const bool odd_lane = threadIdx.x & 1;

  for (uint32_t tt = t1; tt > t0; --tt) {  // reverse order: L2 reuse after k_amax
    const uint32_t t = tt - 1u;
    uint4 v[kVecPerThread];
    const uint32_t base = t * kTileVecs + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      uint32_t vi = base + u * kThreads;
      v[u] = vi < sh.nvec ? __ldcs(x + vi) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const uint32_t vi = base + u * kThreads;
      const bool valid = vi < sh.nvec;
      if (valid && gc.seek(sh.G > 1 ? fastdiv(vi, sh.vpr) : 0u)) {
        s_g = global_scale_from(__ldg(amax + gc.g));
        den6 = __fmul_rn(6.0f, s_g);
      }
      // block max over the lane pair holding the 16-element block
      uint32_t m = absmax8_bits(v[u]);
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      if (!valid) continue;
      const float bmax = __uint_as_float(m << 16);
      const uint32_t sb = cvt_e4m3(__fdiv_rn(bmax, den6));
      const float sbv = e4m3_to_f32(sb);
      const float d = __fmul_rn(s_g, sbv);
      const uint32_t db = __float_as_uint(d);
      const bool fast_blk = db >= kDMin && db <= kDMax;
      const float r = fast_blk ? __frcp_rn(d) : 0.0f;

      float a[8], za[8];
      abs8(v[u], a);
      uint32_t slow = fast_blk ? 0u : 0xFFu;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        za[j] = __fmul_rn(a[j], r);
        const uint32_t zb = __float_as_uint(za[j]);
        const bool hard = (a[j] != 0.0f) && (near_critical(zb) || zb < kTinyZ);
        slow |= (uint32_t)hard << j;
      }
      uint32_t code = cvt_e2m1x8(za);
      if (slow) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
          if (!((slow >> j) & 1u)) continue;
          const float xf = (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
          const Exact e = exact_site(xf, d);
          code = (code & ~(0xFu << (4 * j))) | ((uint32_t)e.rtn << (4 * j));
        }
      }
      const uint32_t mb = nibble_lsbs(code);
      // sign bit of every nibble = sign of x (z = x/d keeps it, zeros too)
      const uint32_t sg = signs8(v[u]);
      uint32_t sgn = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) sgn |= ((sg >> j) & 1u) << (4 * j + 3);
      code |= sgn;
      codes[vi] = code;
      mbits[vi] = (uint8_t)mb;
      if (!odd_lane) scales[vi >> 1] = (uint8_t)sb;
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 3/5: fake-quant forward with given scales.  GUIDED: pick, of the
// bracket around z, the member whose mantissa bit is the cached bit; else
// round to nearest.  Writes bf16 q*·s and the STE mask.
// ---------------------------------------------------------------------------
template <bool GUIDED>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) k_fake_quant(const uint4* __restrict__ x, Shape sh,
                                                         const int64_t* __restrict__ offs,
                                                         const uint8_t* __restrict__ mbits,
                                                         const uint8_t* __restrict__ scales,
                                                         const float* __restrict__ gscale,
                                                         uint4* __restrict__ out,
                                                         uint8_t* __restrict__ mask) {
  uint32_t t0, t1;
  cta_tile_range(sh, t0, t1);
  GroupCursor gc;
  gc.init(offs, sh.G);
  float s_g = 1.0f;

  for (uint32_t t = t0; t < t1; ++t) {
    uint4 v[kVecPerThread];
    uint32_t bits[kVecPerThread], sbs[kVecPerThread];
    const uint32_t base = t * kTileVecs + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const uint32_t vi = base + u * kThreads;
      const bool valid = vi < sh.nvec;
      v[u] = valid ? __ldcs(x + vi) : make_uint4(0u, 0u, 0u, 0u);
      bits[u] = (GUIDED && valid) ? (uint32_t)__ldcs(mbits + vi) : 0u;
      sbs[u] = valid ? (uint32_t)__ldcs(scales + (vi >> 1)) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const uint32_t vi = base + u * kThreads;
      if (vi >= sh.nvec) continue;
      if (gc.seek(sh.G > 1 ? fastdiv(vi, sh.vpr) : 0u)) s_g = __ldg(gscale + gc.g);
      const float sbv = e4m3_to_f32(sbs[u]);
      const float d = __fmul_rn(s_g, sbv);
      const uint32_t db = __float_as_uint(d);
      const bool fast_blk = db >= kDMin && db <= kDMax;
      const float r = fast_blk ? __frcp_rn(d) : 0.0f;
      const uint32_t b1 = f32_to_bf16_bits(d);
      const uint32_t b15 = f32_to_bf16_bits(__fmul_rn(__fmul_rn(1.5f, sbv), s_g));

      float a[8], za[8];
      abs8(v[u], a);
      uint32_t slow = fast_blk ? 0u : 0xFFu;
      uint32_t inmask = 0u;
      uint32_t c[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        za[j] = __fmul_rn(a[j], r);
        const uint32_t zb = __float_as_uint(za[j]);
        const bool hard = (a[j] != 0.0f) && (near_critical(zb) || zb < kTinyZ);
        slow |= (uint32_t)hard << j;
        inmask |= (uint32_t)(zb <= kSix) << j;
        if (GUIDED) {
          const int tq = (int)(zb >> 22) - 252;
          const uint32_t k = (uint32_t)(min(max(tq, 0), 7) + (tq == 0));
          const bool exact = (zb == 0u) || (zb > kSix);
          const uint32_t bit = (bits[u] >> j) & 1u;
          c[j] = exact ? k : k + ((k ^ bit) & 1u);
        }
      }
      if (!GUIDED) {
        const uint32_t code = cvt_e2m1x8(za);
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = (code >> (4 * j)) & 0xFu;
      }
      uint32_t o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = dequant_fast(c[j], b1, b15);
      if (slow) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
          if (!((slow >> j) & 1u)) continue;
          const float xf = (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
          const Exact e = exact_site(xf, d);
          int cs;
          if (GUIDED) {
            const int bit = (bits[u] >> j) & 1;
            cs = e.exact ? e.floor : e.floor + ((e.floor ^ bit) & 1);
          } else {
            cs = e.rtn;
          }
          inmask = (inmask & ~(1u << j)) | ((uint32_t)e.in << j);
          o[j] = dequant_exact(cs, sbv, s_g);
        }
      }
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint4 res;
      res.x = (o[0] | (o[1] << 16)) | (w[0] & 0x80008000u);
      res.y = (o[2] | (o[3] << 16)) | (w[1] & 0x80008000u);
      res.z = (o[4] | (o[5] << 16)) | (w[2] & 0x80008000u);
      res.w = (o[6] | (o[7] << 16)) | (w[3] & 0x80008000u);
      out[vi] = res;
      mask[vi] = (uint8_t)inmask;
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 4: masked straight-through backward.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, kCtasPerSm) k_ste_bwd(const uint4* __restrict__ g, Shape sh,
                                                      const uint8_t* __restrict__ mask,
                                                      uint4* __restrict__ gin) {
  uint32_t t0, t1;
  cta_tile_range(sh, t0, t1);
  for (uint32_t t = t0; t < t1; ++t) {
    uint4 v[kVecPerThread];
    uint32_t m[kVecPerThread];
    const uint32_t base = t * kTileVecs + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const uint32_t vi = base + u * kThreads;
      const bool valid = vi < sh.nvec;
      v[u] = valid ? __ldcs(g + vi) : make_uint4(0u, 0u, 0u, 0u);
      m[u] = valid ? (uint32_t)__ldcs(mask + vi) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const uint32_t vi = base + u * kThreads;
      if (vi >= sh.nvec) continue;
      const uint32_t b = m[u];
      // bit pair (2k, 2k+1) -> half-word keep masks of word k
      auto keep = [&](int k) {
        return (((b >> (2 * k)) & 1u) ? 0x0000FFFFu : 0u) | (((b >> (2 * k + 1)) & 1u) ? 0xFFFF0000u : 0u);
      };
      uint4 r;
      r.x = v[u].x & keep(0);
      r.y = v[u].y & keep(1);
      r.z = v[u].z & keep(2);
      r.w = v[u].w & keep(3);
      gin[vi] = r;
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 6: plain copy with the same access pattern (bandwidth yardstick).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, kCtasPerSm) k_copy(const uint4* __restrict__ s, Shape sh,
                                                   uint4* __restrict__ d) {
  uint32_t t0, t1;
  cta_tile_range(sh, t0, t1);
  for (uint32_t t = t0; t < t1; ++t) {
    uint4 v[kVecPerThread];
    const uint32_t base = t * kTileVecs + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const uint32_t vi = base + u * kThreads;
      v[u] = vi < sh.nvec ? __ldcs(s + vi) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const uint32_t vi = base + u * kThreads;
      if (vi < sh.nvec) d[vi] = v[u];
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];  // 0 = not queried yet (benign race: same value)

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return -1;
  if (dev < kMaxDevices && g_sm_count[dev] > 0) return g_sm_count[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
  if (dev < kMaxDevices) g_sm_count[dev] = n;
  return n;
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

int check_shape(int64_t rows, int64_t cols, int32_t G, const int64_t* offs) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0 || G < 1) return TRACE_ERR_SHAPE;
  if (G > 1 && offs == nullptr) return TRACE_ERR_NULL;
  const long double n = (long double)rows * (long double)cols;
  if (n / 8 >= 4294967296.0L - (long double)kTileVecs) return TRACE_ERR_SHAPE;
  return TRACE_OK;
}

Shape make_shape(int64_t rows, int64_t cols, int32_t G) {
  Shape sh;
  const uint64_t n = (uint64_t)rows * (uint64_t)cols;
  sh.nvec = (uint32_t)(n / 8);
  sh.ntiles = (uint32_t)((sh.nvec + kTileVecs - 1) / kTileVecs);
  sh.vpr = make_fastdiv((uint32_t)(cols / 8));
  sh.G = G;
  return sh;
}

int grid_for(const Shape& sh, int* grid) {
  const int sms = sm_count();
  if (sms <= 0) return TRACE_ERR_CUDA;
  uint32_t g = (uint32_t)sms * kCtasPerSm;
  if (sh.ntiles < g) g = sh.ntiles;
  *grid = (int)(g > 0 ? g : 1);
  return TRACE_OK;
}

int launched() { return cudaGetLastError() == cudaSuccess ? TRACE_OK : TRACE_ERR_CUDA; }

}  // namespace

extern "C" {

const char* trace_strerror(int status) {
  switch (status) {
    case TRACE_OK: return "ok";
    case TRACE_ERR_NULL: return "a required pointer is NULL";
    case TRACE_ERR_SHAPE: return "invalid shape (rows < 0, cols <= 0, cols % 32 != 0, groups < 1, or N/8 >= 2^32)";
    case TRACE_ERR_ALIGN: return "a pointer is not aligned as the call requires";
    case TRACE_ERR_WORKSPACE: return "workspace smaller than trace_capture_workspace_bytes()";
    case TRACE_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    default: return "unknown status";
  }
}

int trace_abi_version(void) { return TRACE_ABI_VERSION; }

size_t trace_capture_workspace_bytes(int64_t rows, int64_t cols, int32_t num_groups) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0 || num_groups < 1) return 0;
  return ((size_t)num_groups * 4u + 255u) / 256u * 256u;
}

int trace_capture(const uint16_t* x, int64_t rows, int64_t cols, int32_t num_groups,
                  const int64_t* group_row_offsets, uint8_t* codes, uint32_t* mbits,
                  uint8_t* scales, float* gscale, void* workspace, size_t workspace_bytes,
                  void* stream) {
  int st = check_shape(rows, cols, num_groups, group_row_offsets);
  if (st) return st;
  // with no rows only the global scales are written; the data pointers of
  // empty tensors may be NULL
  const bool empty = rows == 0;
  if ((!empty && (!x || !codes || !mbits || !scales)) || !gscale || !workspace) return TRACE_ERR_NULL;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(mbits, 16) || !aligned(scales, 16) ||
      !aligned(gscale, 4) || !aligned(workspace, 256))
    return TRACE_ERR_ALIGN;
  if (workspace_bytes < trace_capture_workspace_bytes(rows, cols, num_groups)) return TRACE_ERR_WORKSPACE;
  const Shape sh = make_shape(rows, cols, num_groups);
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t* amax = (uint32_t*)workspace;
  const int64_t* offs = num_groups > 1 ? group_row_offsets : nullptr;
  const int zg = (num_groups + kThreads - 1) / kThreads;
  k_zero_u32<<<zg < 1024 ? zg : 1024, kThreads, 0, s>>>(amax, num_groups);
  if (sh.nvec > 0) k_amax<<<grid, kThreads, 0, s>>>((const uint4*)x, sh, offs, amax);
  k_capture<<<grid, kThreads, 0, s>>>((const uint4*)x, sh, offs, amax, (uint32_t*)codes,
                                      (uint8_t*)mbits, scales, gscale);
  return launched();
}

static int fake_quant_launch(bool guided, const uint16_t* x, int64_t rows, int64_t cols, int32_t G,
                             const int64_t* offs, const uint32_t* mbits, const uint8_t* scales,
                             const float* gscale, uint16_t* out, uint32_t* mask, void* stream) {
  int st = check_shape(rows, cols, G, offs);
  if (st) return st;
  if (rows == 0) return TRACE_OK;  // nothing to do; empty tensors may have NULL data
  if (!x || (guided && !mbits) || !scales || !gscale || !out || !mask) return TRACE_ERR_NULL;
  if (!aligned(x, 16) || (guided && !aligned(mbits, 16)) || !aligned(scales, 16) ||
      !aligned(gscale, 4) || !aligned(out, 16) || !aligned(mask, 16))
    return TRACE_ERR_ALIGN;
  const Shape sh = make_shape(rows, cols, G);
  if (sh.nvec == 0) return TRACE_OK;
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t* o = G > 1 ? offs : nullptr;
  if (guided)
    k_fake_quant<true><<<grid, kThreads, 0, s>>>((const uint4*)x, sh, o, (const uint8_t*)mbits,
                                                 scales, gscale, (uint4*)out, (uint8_t*)mask);
  else
    k_fake_quant<false><<<grid, kThreads, 0, s>>>((const uint4*)x, sh, o, nullptr, scales, gscale,
                                                  (uint4*)out, (uint8_t*)mask);
  return launched();
}

int trace_guided_fq_fwd(const uint16_t* x_train, int64_t rows, int64_t cols, int32_t num_groups,
                        const int64_t* group_row_offsets, const uint32_t* mbits,
                        const uint8_t* scales, const float* gscale, uint16_t* out,
                        uint32_t* ste_mask, void* stream) {
  return fake_quant_launch(true, x_train, rows, cols, num_groups, group_row_offsets, mbits, scales,
                           gscale, out, ste_mask, stream);
}

int trace_rtn_fq_fwd(const uint16_t* x, int64_t rows, int64_t cols, int32_t num_groups,
                     const int64_t* group_row_offsets, const uint8_t* scales, const float* gscale,
                     uint16_t* out, uint32_t* ste_mask, void* stream) {
  return fake_quant_launch(false, x, rows, cols, num_groups, group_row_offsets, nullptr, scales,
                           gscale, out, ste_mask, stream);
}

int trace_fq_bwd(const uint16_t* grad_out, const uint32_t* ste_mask, int64_t numel,
                 uint16_t* grad_in, void* stream) {
  if (numel < 0 || numel % 32 != 0) return TRACE_ERR_SHAPE;
  if ((long double)numel / 8 >= 4294967296.0L - (long double)kTileVecs) return TRACE_ERR_SHAPE;
  if (numel == 0) return TRACE_OK;
  if (!grad_out || !ste_mask || !grad_in) return TRACE_ERR_NULL;
  if (!aligned(grad_out, 16) || !aligned(ste_mask, 16) || !aligned(grad_in, 16)) return TRACE_ERR_ALIGN;
  const Shape sh = make_shape(numel / 32, 32, 1);
  if (sh.nvec == 0) return TRACE_OK;
  int grid, st;
  if ((st = grid_for(sh, &grid))) return st;
  k_ste_bwd<<<grid, kThreads, 0, (cudaStream_t)stream>>>((const uint4*)grad_out, sh,
                                                         (const uint8_t*)ste_mask, (uint4*)grad_in);
  return launched();
}

int trace_copy_bf16(const uint16_t* src, uint16_t* dst, int64_t numel, void* stream) {
  if (numel < 0 || numel % 8 != 0) return TRACE_ERR_SHAPE;
  if ((long double)numel / 8 >= 4294967296.0L - (long double)kTileVecs) return TRACE_ERR_SHAPE;
  if (numel == 0) return TRACE_OK;
  if (!src || !dst) return TRACE_ERR_NULL;
  if (!aligned(src, 16) || !aligned(dst, 16)) return TRACE_ERR_ALIGN;
  Shape sh;
  sh.nvec = (uint32_t)(numel / 8);
  sh.ntiles = (sh.nvec + kTileVecs - 1) / kTileVecs;
  sh.vpr = make_fastdiv(1);
  sh.G = 1;
  if (sh.nvec == 0) return TRACE_OK;
  int grid, st;
  if ((st = grid_for(sh, &grid))) return st;
  k_copy<<<grid, kThreads, 0, (cudaStream_t)stream>>>((const uint4*)src, sh, (uint4*)dst);
  return launched();
}

}  // extern "C"
