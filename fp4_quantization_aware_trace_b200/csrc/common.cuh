// common.cuh -- device helpers shared by every kernel of libtrace_fp4.so:
// launch constants, programmatic dependent launch, the fast division,
// 32-byte loads and stores, packed fp32x2 arithmetic, the hardware number
// format conversions, the exact-quotient and grid-rounding helpers, the group
// cursor, the shape record and the tiled scale offset.  Included by
// trace_fp4.cu inside its anonymous namespace (one translation unit).
#pragma once

typedef unsigned long long u64;

constexpr int kThreads = 256;
constexpr int kBlkPerThread = 2;
constexpr int kTileBlks = kThreads * kBlkPerThread;  // 512 blocks = 8192 elements
constexpr int kCtasPerSm = 4;    // resident CTAs per SM the register budget allows
constexpr int kGridPerSm = 32;   // CTAs launched per SM: about one tile each
constexpr int kAmaxTable = 256;  // groups per CTA kept in shared memory
// Polls of the one-launch capture's grid barrier before it gives up (with a
// 256 ns sleep between polls: 2.15 s on B200).  The launch is cooperative,
// so every CTA is resident and the barrier completes long before.
constexpr uint32_t kBarrierPolls = 1u << 22;

constexpr uint32_t kDMin = 0x12800000u;     // 2^-90: fast paths need d >= 2^-90
constexpr uint32_t kDMax = 0x71800000u;     // 2^100: capture / round-to-nearest
constexpr uint32_t kDMaxExactZ = 0x47800000u;  // 2^16: guided (see below)
// The guided path divides |x| * 2^64: every nonzero bf16 then has a normal
// quotient and an exactly representable remainder for d in the fast range.
constexpr float kXs = 0x1p64f;
constexpr float kSixS = 0x1p64f * 6.0f;

// ---------------------------------------------------------------------------
// Programmatic dependent launch (sm_90+): every kernel waits for the
// previous kernel in the stream to complete before it reads any global
// memory, then lets the next kernel start launching.  Launched with the
// programmatic-serialization attribute, a kernel's launch and prologue
// overlap the tail of the one before it; launched without it, both
// instructions are no-ops.
// ---------------------------------------------------------------------------
// Acquire load / release store at GPU scope (the grid barrier of the
// one-launch capture).
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void pdl_begin() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Fast unsigned 32-bit division by a runtime constant (Granlund & Montgomery,
// "Division by invariant integers using multiplication", PLDI 1994, the
// round-up method with the add-back step): block index -> row.
// ---------------------------------------------------------------------------
struct FastDiv {
  uint32_t d, m, s;  // s = ceil(log2 d); d <= 1 handled separately
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
// Memory access (public PTX ISA: 32-byte vector loads/stores on sm_100)
// ---------------------------------------------------------------------------
struct V8 {
  uint32_t w[8];
};

// One 16-element bf16 block; read once, not kept in L1.
__device__ __forceinline__ V8 ld_block_stream(const void* p) {
  V8 v;
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]),
                 "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7])
               : "l"(p));
  return v;
}

// The same load kept in L1: for the guided forwards with separate outputs,
// which read words of the block back for the pairs they recompute.
__device__ __forceinline__ V8 ld_block_l1(const void* p) {
  V8 v;
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]),
                 "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7])
               : "l"(p));
  return v;
}

// Block load and store for the rarely taken out-of-line (exact-path)
// functions, as plain 16-byte accesses: with the 32-byte asm forms inside a
// non-inlined function, ptxas 12.9 crashed (load) or, depending on the other
// code in the module, stored wrong data (store; caught by the seeded fuzz
// parity tests).
__device__ __forceinline__ V8 ld_block_ro(const V8* p) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  V8 v;
  v.w[0] = a.x; v.w[1] = a.y; v.w[2] = a.z; v.w[3] = a.w;
  v.w[4] = b.x; v.w[5] = b.y; v.w[6] = b.z; v.w[7] = b.w;
  return v;
}

__device__ __forceinline__ void st_block_plain(V8* p, const V8& v) {
  uint4* q = reinterpret_cast<uint4*>(p);
  q[0] = make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]);
  q[1] = make_uint4(v.w[4], v.w[5], v.w[6], v.w[7]);
}

__device__ __forceinline__ void st_block(void* p, const V8& v) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v.w[0]),
               "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]),
               "r"(v.w[7])
               : "memory");
}

__device__ __forceinline__ V8 zero_block() {
  V8 v;
#pragma unroll
  for (int k = 0; k < 8; ++k) v.w[k] = 0u;
  return v;
}

// ---------------------------------------------------------------------------
// Packed fp32x2 arithmetic (public PTX ISA, sm_100: mul/fma/add/sub .f32x2)
// ---------------------------------------------------------------------------
__device__ __forceinline__ u64 pk(float lo, float hi) {
  u64 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk(u64 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ u64 mul2(u64 a, u64 b) {
  u64 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
  u64 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ u64 add_rm2(u64 a, u64 b) {
  u64 r;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ u64 add_rp2(u64 a, u64 b) {
  u64 r;
  asm("add.rp.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ u64 sub2(u64 a, u64 b) {
  u64 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// ---------------------------------------------------------------------------
// Number-format helpers (hardware conversions from the public PTX ISA)
// ---------------------------------------------------------------------------

// Eight fp32 (four pairs lo, hi) -> one word of eight E2M1 codes (round to
// nearest even, satfinite; the sign of each input is kept), element j in
// bits 4j..4j+3.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float a0, float a1, float a2, float a3, float a4,
                                               float a5, float a6, float a7) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
  return r;
}

// Eight fp32 from an array (element j in bits 4j..4j+3), as above.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float* a) {
  return cvt_e2m1x8(a[0], a[1], a[2], a[3], a[4], a[5], a[6], a[7]);
}

// Two fp32 -> their round-to-nearest E2M1 codeword values (ties to the even
// code, satfinite) as f16x2, lo in the low half: the encode and the exact
// decode with the code byte kept in an 8-bit register between them.
__device__ __forceinline__ uint32_t rtn_e2m1x2_f16x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// As rtn_e2m1x2_f16x2, also returning the code byte (lo code in bits 0-3,
// hi code in bits 4-7) in `code`.
__device__ __forceinline__ uint32_t rtn_e2m1x2_f16x2_code(float lo, float hi, uint32_t& code) {
  uint32_t r, c;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %2, %3;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b;\n\t"
      "cvt.u32.u8 %1, b;\n\t}"
      : "=r"(r), "=r"(c)
      : "f"(hi), "f"(lo));
  code = c;
  return r;
}

// Byte of two E2M1 codes -> f16x2 (exact): lo code in the low half.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.u8.u32 b, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
      : "=r"(r)
      : "r"(byte));
  return r;
}

// fp32 >= 0 -> E4M3 byte (round to nearest even, saturating at 448).
__device__ __forceinline__ uint32_t cvt_e4m3(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
  return (uint32_t)(r & 0xFFu);
}

// Two E4M3 bytes (b0 | b1 << 8) -> fp32 (exact, through f16x2).
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t b2, float& lo, float& hi) {
  uint32_t h2;
  uint16_t in = (uint16_t)b2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

// Two fp32 -> bf16x2 (round to nearest even): lo in the low half.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Per half, max(|a|, |b|) of two bf16 pairs (the sign bit of each half is
// the xor of the inputs' signs; callers clear it).
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// max|x| over a block as bf16 bits (integer order = magnitude order): a tree
// of magnitude maxima over the 8 words, then the larger half.
__device__ __forceinline__ uint32_t absmax_block(const V8& v) {
  const uint32_t m = absmax2(absmax2(absmax2(v.w[0], v.w[1]), absmax2(v.w[2], v.w[3])),
                             absmax2(absmax2(v.w[4], v.w[5]), absmax2(v.w[6], v.w[7]))) &
                     0x7FFF7FFFu;
  return max(m & 0xFFFFu, m >> 16);
}

// Mantissa bits of 32 codes: bit 8k + j of the result = bit 4j of word k
// (the lowest bit of each nibble).  Per word, the two lowest bits of each
// byte's nibbles are gathered to bits 8b, 8b + 1 and one multiply moves the
// field of byte b to bits 24 + 2b; the other partial products fall below
// bit 24 at distinct even positions (no carries) or above bit 31.
__device__ __forceinline__ uint32_t nibble_lsbs4(uint4 c) {
  const uint32_t kGather = (1u << 24) | (1u << 18) | (1u << 12) | (1u << 6);
  const uint32_t tx = ((c.x & 0x01010101u) | ((c.x >> 3) & 0x02020202u)) * kGather;
  const uint32_t ty = ((c.y & 0x01010101u) | ((c.y >> 3) & 0x02020202u)) * kGather;
  const uint32_t tz = ((c.z & 0x01010101u) | ((c.z >> 3) & 0x02020202u)) * kGather;
  const uint32_t tw = ((c.w & 0x01010101u) | ((c.w >> 3) & 0x02020202u)) * kGather;
  return __byte_perm(__byte_perm(tx, ty, 0x0073u), __byte_perm(tz, tw, 0x0073u), 0x5410u);
}

// Per-block constants of the fast path.
struct BlkK {
  u64 rr;    // (r, r), r = RN(1/d)
  u64 ndd;   // (-d, -d)
  u64 sbv2;  // (s_b, s_b), times 2^-64 on the guided path
  u64 sg2;   // (s_g, s_g)
};

__device__ __forceinline__ BlkK make_blk(float d, float sbv, float s_g) {
  BlkK k;
  const float r = __frcp_rn(d);
  k.rr = pk(r, r);
  k.ndd = pk(-d, -d);
  k.sbv2 = pk(sbv, sbv);
  k.sg2 = pk(s_g, s_g);
  return k;
}

// STE mask bit of a quotient z >= 0 as a float, on the FMA pipe: 1.0 where
// z <= 6, else 0.0 (NaN and infinity included).  z * -2^100 + (6 * 2^100 +
// 2^79) is rounded once: it is 2^79 at z = 6, at most 0 from the next float
// past 6 (6 + 2^-21) on, and the saturation maps it (NaN included) to 0 or 1.
__device__ __forceinline__ float le6_step(float z) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(z), "f"(-0x1p100f), "f"(0x1.800002p102f));
  return r;
}

// The same for the W4A8 mask, z <= 448: 448 * 2^100 + 2^85 (448 = 1.75 * 2^8,
// and 2^85 is the spacing of floats at 448 * 2^100).
__device__ __forceinline__ float le448_step(float z) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(z), "f"(-0x1p100f), "f"(0x1.c00002p108f));
  return r;
}

__device__ __forceinline__ bool fast_scale(float d, uint32_t dmax_bits = kDMax) {
  const uint32_t db = __float_as_uint(d);
  return db >= kDMin && db <= dmax_bits;
}

// Correctly rounded quotients of a pair: (lo, hi) / d.
__device__ __forceinline__ u64 quot2(u64 xx, const BlkK& k) {
  const u64 q0 = mul2(xx, k.rr);
  const u64 e = fma2(q0, k.ndd, xx);
  return fma2(e, k.rr, q0);
}

// Magic addend of the grid rounding for a = min(|z|, 6) * 2^64:
// M = 2^86 * max(1, 2^E), E the binade of a / 2^64.
__device__ __forceinline__ float grid_magic_s(float a_s) {
  return __uint_as_float(max((__float_as_uint(a_s) & 0x7F800000u) + 0x0B000000u, 0x6A800000u));
}

// The same addend for a pair, with the binade scaling as one packed multiply
// (exact: the masked exponent is a power of two or zero).
__device__ __forceinline__ u64 grid_magic_s2(float al, float ah) {
  const u64 e = pk(__uint_as_float(__float_as_uint(al) & 0x7F800000u),
                   __uint_as_float(__float_as_uint(ah) & 0x7F800000u));
  float ml, mh;
  upk(mul2(e, pk(0x1p22f, 0x1p22f)), ml, mh);
  return pk(fmaxf(ml, 0x1p86f), fmaxf(mh, 0x1p86f));
}

// Power-of-two scales and the unscaled grid addend (MX formats).
// 2^k as fp32 for k in [-127, 127] (2^-127 is a subnormal).
__device__ __forceinline__ float pow2f(int k) {
  return __uint_as_float(k >= -126 ? (uint32_t)(k + 127) << 23 : 0x00800000u >> (-126 - k));
}

// Magic addend of the grid rounding for a = min(|z|, 6) (unscaled):
// M = 2^22 * max(1, 2^E).
__device__ __forceinline__ float grid_magic(float a) {
  return __uint_as_float(max((__float_as_uint(a) & 0x7F800000u) + 0x0B000000u, 0x4A800000u));
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
    if (G == 1) {
      if (lo == 0u) return false;
      g = 0;
      lo = 0u;
      hi = 0xFFFFFFFFu;
      return true;
    }
    if (row >= lo && row < hi) return false;
    int a = 0, b = G;  // last g with offs[g] <= row
    while (b - a > 1) {
      const int m = (a + b) >> 1;
      if ((uint64_t)offs[m] <= row) a = m; else b = m;
    }
    g = a;
    lo = (uint32_t)offs[a];
    hi = (uint32_t)offs[a + 1];
    return true;
  }
};

struct Shape {
  uint32_t nblk;    // N / 16
  uint32_t ntiles;  // ceil(nblk / kTileBlks)
  FastDiv bpr;      // blocks per row
  int G;
  uint32_t sw_ct;   // tiled scale layout: 128 x 4 tiles per row of tiles
};

// Byte offset of the scale at (row, col) in the tiled layout a block-scaled
// FP4 GEMM reads: the scale matrix cut into 128-row x 4-column tiles of 512
// bytes, stored in row-major tile order (ct tiles per row of tiles); inside
// a tile, row r and column c sit at 16 (r mod 32) + 4 (r div 32) + c.
__device__ __forceinline__ size_t tiled_scale_offset(uint32_t row, uint32_t col, uint32_t ct) {
  return ((size_t)(row >> 7) * ct + (col >> 2)) * 512u + ((row & 31u) << 4) +
         (((row >> 5) & 3u) << 2) + (col & 3u);
}
