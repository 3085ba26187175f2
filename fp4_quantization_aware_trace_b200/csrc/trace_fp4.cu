// trace_fp4.cu -- B200 (sm_100a) kernels and C ABI for TRACE rollout-guided
// NVFP4 rounding: rollout capture of the compact cache, the guided QAT
// fake-quant forward, the masked straight-through backward and the
// round-to-nearest comparator; with them the full-information guided
// forward, the MXFP4 (W4A4) and W4A8 variants, the 128 x 4 tiled scale
// layout, capture's two passes for sharded or streamed tensors, and the
// mismatch-distance histogram.
//
// Method: rcap.io post "TRACE: Rollout-Guided Quantization-Aware Training for
// FP4" (2026-10-06), sections "rollout-guided rounding" and "compact cache"
// and its pseudocode listing (capture; QAT forward).  The number format and
// the layouts are documented in include/trace_fp4.h.
//
// Design (everything here is HBM-bound elementwise work; no tensor cores):
//   * One thread owns one 16-element scale block: a single 32-byte load
//     (ld.global.v8) brings it in, so a warp reads 1 KiB contiguous per
//     instruction and the per-block work (scale decode, reciprocal) is done
//     once.  A CTA of 256 threads works on tiles of 512 blocks, two blocks per
//     thread with all loads issued before any use.  The grid is 32 CTAs per
//     SM (about one tile per CTA at the 64 MiB sizes), striding over tiles
//     beyond that: oversubscribing lets the block scheduler balance the tail,
//     which measured faster on B200 than persistent per-CTA ranges.
//   * Capture is a two-pass grid amax: kernel 1 reduces max|x| per group
//     (shared-memory table per CTA, one global atomicMax per group per CTA
//     into a zeroed workspace); kernel 2 walks the tiles in REVERSE order, so
//     it starts on the data kernel 1 touched last and finds much of x still
//     in the 126 MB L2.
//   * Exact quotient without a division per element: with r = RN(1/d),
//     q0 = RN(x*r), e = RN(x - q0*d) (one FMA) and z = RN(q0 + e*r) (one FMA)
//     is the correctly rounded x/d for every bf16 x and fp32 d whose
//     quotient is a normal number and whose remainder is representable --
//     the correction step of Markstein (IBM J. Res. Dev. 34(1), 1990),
//     established here by exhaustive check of all 2^31 pairs of bf16 and fp32
//     significands in both result binades (tests/test_kernel_math.py).
//     Capture and round-to-nearest only need the exact quotient from 0.25 up
//     (x >= 2^-92 when d >= 2^-90, where the remainder is exact; below
//     0.25 every decision is "code 0", and the sign comes from x).  The
//     guided path also needs "exactly zero" to be exact, so it divides
//     |x| * 2^64: for d in [2^-90, 2^16] every nonzero bf16 then has a
//     normal quotient and a normal remainder, and fl(x/d) itself is nonzero
//     (x/d >= 2^-133 / 2^16 = 2^-149), so the scaled quotient is zero exactly
//     when fl(x/d) is; the codeword found is scaled back by folding 2^-64
//     into s_b.  Two elements go through each
//     packed fp32x2 instruction (mul/fma/add .f32x2, sm_100).
//   * Rounding on the E2M1 grid without a table: with M = 2^22 * max(1, 2^E)
//     (E the binade of a = min(|z|,6); everything times 2^64 on the guided
//     path), a + M rounded down / up lands on
//     M + floor / M + ceiling of a on the grid (spacing 0.5 below 2, 1 in
//     [2,4), 2 in [4,8)), and the lowest bit of the sum is the mantissa bit
//     of that codeword.  The guided choice is "the neighbour whose bit equals
//     the cached bit"; when a is a codeword both roundings agree, which is
//     the collapsed bracket.  Round-to-nearest uses the hardware
//     cvt.rn.satfinite.e2m1x2.f32 (ties to the even code).
//   * Zero blocks (d = 0) take a short path (every z is +-0); blocks with d
//     outside [2^-90, 2^100] ([2^-90, 2^16] for the guided forward) go
//     through an exact per-element path that divides with IEEE
//     round-to-nearest.
// File layout: this file holds the host side and the C ABI; the kernels are
// in csrc/*.cuh, included below inside this file's anonymous namespace (one
// translation unit): common.cuh (shared device helpers), nvfp4.cuh, mx.cuh,
// mismatch.cuh, util.cuh.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "trace_fp4.h"

namespace {

#include "common.cuh"
#include "nvfp4.cuh"
#include "mx.cuh"
#include "mismatch.cuh"
#include "util.cuh"

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
  if (n / 16 >= 4294967296.0L - (long double)kTileBlks) return TRACE_ERR_SHAPE;
  return TRACE_OK;
}

Shape make_shape(int64_t rows, int64_t cols, int32_t G) {
  Shape sh;
  const uint64_t n = (uint64_t)rows * (uint64_t)cols;
  sh.nblk = (uint32_t)(n / 16);
  sh.ntiles = (uint32_t)(((uint64_t)sh.nblk + kTileBlks - 1) / kTileBlks);
  sh.bpr = make_fastdiv((uint32_t)(cols / 16));
  sh.G = G;
  sh.sw_ct = (uint32_t)((cols / 16 + 3) / 4);  // NVFP4: cols/16 scale columns
  return sh;
}

int grid_for(const Shape& sh, int* grid) {
  const int sms = sm_count();
  if (sms <= 0) return TRACE_ERR_CUDA;
  uint32_t g = (uint32_t)sms * kGridPerSm;
  if (sh.ntiles < g) g = sh.ntiles;
  *grid = (int)(g > 0 ? g : 1);
  return TRACE_OK;
}

// Launch with programmatic stream serialization (see pdl_begin): the kernel
// may begin launching while the previous kernel in the stream finishes; it
// waits for it before touching memory.
template <typename... KArgs, typename... Args>
int launch(void (*kernel)(KArgs...), int grid, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess ? TRACE_OK
                                                                                      : TRACE_ERR_CUDA;
}

// The guided rules: SEP when out does not overlap x (see k_fake_quant).
template <int MODE, bool SW>
int guided_dispatch(bool sep, int grid, cudaStream_t s, const uint16_t* x, const Shape& sh,
                    const int64_t* o, const uint32_t* mbits, const uint8_t* rcodes,
                    const uint8_t* scales, const float* gscale, uint16_t* out, uint32_t* mask) {
  if (sep)
    return launch(k_fake_quant<MODE, SW, kCtasPerSm, true>, grid, s, (const V8*)x, sh, o, mbits,
                  (const uint4*)rcodes, scales, gscale, (V8*)out, mask);
  return launch(k_fake_quant<MODE, SW, kCtasPerSm, false>, grid, s, (const V8*)x, sh, o, mbits,
                (const uint4*)rcodes, scales, gscale, (V8*)out, mask);
}

template <bool SW>
int fake_quant_dispatch(int mode, int grid, cudaStream_t s, const uint16_t* x,
                               const Shape& sh, const int64_t* o, const uint32_t* mbits,
                               const uint8_t* rcodes, const uint8_t* scales, const float* gscale,
                               uint16_t* out, uint32_t* mask) {
  const size_t bytes = (size_t)sh.nblk * 32u;
  const bool sep = (uintptr_t)out + bytes <= (uintptr_t)x || (uintptr_t)x + bytes <= (uintptr_t)out;
  if (mode == kGuided)
    return guided_dispatch<kGuided, SW>(sep, grid, s, x, sh, o, mbits, nullptr, scales, gscale,
                                        out, mask);
  if (mode == kFull)
    return guided_dispatch<kFull, SW>(sep, grid, s, x, sh, o, nullptr, rcodes, scales, gscale, out,
                                      mask);
  return launch(k_fake_quant<kRtn, SW>, grid, s, (const V8*)x, sh, o, (const uint32_t*)nullptr,
                (const uint4*)nullptr, scales, gscale, (V8*)out, mask);
}

template <bool SW>
int mx_fake_quant_dispatch(int mode, int grid, cudaStream_t s, const uint16_t* x,
                                  const Shape& sh, const uint32_t* mbits, const uint8_t* rcodes,
                                  const uint8_t* scales, uint16_t* out, uint32_t* mask) {
  if (mode == kGuided)
    return launch(k_mx_fake_quant<kGuided, SW>, grid, s, (const V8*)x, sh, mbits,
                  (const uint4*)nullptr, scales, (V8*)out, mask);
  if (mode == kFull)
    return launch(k_mx_fake_quant<kFull, SW>, grid, s, (const V8*)x, sh, (const uint32_t*)nullptr,
                  (const uint4*)rcodes, scales, (V8*)out, mask);
  return launch(k_mx_fake_quant<kRtn, SW>, grid, s, (const V8*)x, sh, (const uint32_t*)nullptr,
                (const uint4*)nullptr, scales, (V8*)out, mask);
}

template <int MODE>
int mx8_launch(const uint16_t* x, int64_t rows, int64_t cols, const uint32_t* mbits,
               const uint8_t* rcodes, const uint8_t* scales, uint16_t* out, uint32_t* mask,
               void* stream, bool tiled = false) {
  int st = check_shape(rows, cols, 1, nullptr);
  if (st) return st;
  if (rows == 0) return TRACE_OK;
  if (!x || (MODE == kGuided && !mbits) || (MODE == kFull && !rcodes) || !scales || !out || !mask)
    return TRACE_ERR_NULL;
  if (!aligned(x, 32) || (MODE == kGuided && !aligned(mbits, 4)) ||
      (MODE == kFull && !aligned(rcodes, 32)) || !aligned(out, 32) || !aligned(mask, 4))
    return TRACE_ERR_ALIGN;
  Shape sh = make_shape(rows, cols, 1);
  sh.sw_ct = (uint32_t)((cols / 32 + 3) / 4);
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  const size_t bytes = (size_t)sh.nblk * 32u;
  const bool sep = MODE != kRtn && ((uintptr_t)out + bytes <= (uintptr_t)x ||
                                    (uintptr_t)x + bytes <= (uintptr_t)out);
  cudaStream_t s = (cudaStream_t)stream;
  if (tiled)
    return sep ? launch(k_mx8_fake_quant<MODE, true, true>, grid, s, (const V8*)x, sh, mbits,
                        (const V8*)rcodes, scales, (V8*)out, mask)
               : launch(k_mx8_fake_quant<MODE, true, false>, grid, s, (const V8*)x, sh, mbits,
                        (const V8*)rcodes, scales, (V8*)out, mask);
  return sep ? launch(k_mx8_fake_quant<MODE, false, true>, grid, s, (const V8*)x, sh, mbits,
                      (const V8*)rcodes, scales, (V8*)out, mask)
             : launch(k_mx8_fake_quant<MODE, false, false>, grid, s, (const V8*)x, sh, mbits,
                      (const V8*)rcodes, scales, (V8*)out, mask);
}

// A cooperative launch (every CTA resident at once; the one-launch capture's
// grid barrier relies on it), with programmatic stream serialization as the
// other launches: the grid may be launched while the previous kernel
// drains (it waits for it before touching memory).  Every kernel of the
// library triggers its dependents at its start, so when this grid is
// launched every CTA of the previous kernel has already started.
template <typename... KArgs, typename... Args>
int launch_coop(void (*kernel)(KArgs...), int grid, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess ? TRACE_OK
                                                                                      : TRACE_ERR_CUDA;
}

// Grid of the one-launch capture: as many CTAs as can be resident at once
// (the occupancy of that kernel on this device, queried once), at most one
// per tile, at least one.
int g_coop_per_sm[kMaxDevices][2];  // 0 = not queried yet (benign race: same value)

template <bool SW>
int coop_grid_for(const Shape& sh, int* grid) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TRACE_ERR_CUDA;
  int per_sm = g_coop_per_sm[dev][SW ? 1 : 0];
  if (per_sm <= 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_capture_coop<SW>, kThreads, 0) !=
            cudaSuccess ||
        per_sm <= 0)
      return TRACE_ERR_CUDA;
    g_coop_per_sm[dev][SW ? 1 : 0] = per_sm;
  }
  const int sms = sm_count();
  if (sms <= 0) return TRACE_ERR_CUDA;
  uint32_t g = (uint32_t)sms * (uint32_t)per_sm;
  if (sh.ntiles < g) g = sh.ntiles;
  *grid = (int)(g > 0 ? g : 1);
  return TRACE_OK;
}

}  // namespace

extern "C" {

const char* trace_strerror(int status) {
  switch (status) {
    case TRACE_OK: return "ok";
    case TRACE_ERR_NULL: return "a required pointer is NULL";
    case TRACE_ERR_SHAPE: return "invalid shape (rows < 0, cols <= 0, cols % 32 != 0, groups < 1, or N/16 >= 2^32)";
    case TRACE_ERR_ALIGN: return "a pointer is not aligned as the call requires";
    case TRACE_ERR_WORKSPACE: return "workspace smaller than trace_capture_workspace_bytes()";
    case TRACE_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case TRACE_ERR_TIMEOUT: return "a capture gave up waiting at its grid barrier";
    default: return "unknown status";
  }
}

int trace_abi_version(void) { return TRACE_ABI_VERSION; }

size_t trace_capture_workspace_bytes(int64_t rows, int64_t cols, int32_t num_groups) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0 || num_groups < 1) return 0;
  // an arrival count, a generation, an error flag, one unused word, then
  // the G accumulators
  return ((size_t)num_groups * 4u + 16u + 255u) / 256u * 256u;
}

size_t trace_cache_record_bytes(int64_t rows, int64_t cols, int32_t num_groups,
                                size_t* mbits_offset, size_t* scales_offset,
                                size_t* gscale_offset) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0 || num_groups < 1) return 0;
  const long double nl = (long double)rows * (long double)cols;
  if (nl / 16 >= 4294967296.0L - (long double)kTileBlks) return 0;
  const size_t n = (size_t)rows * (size_t)cols;
  auto up16 = [](size_t v) { return (v + 15u) / 16u * 16u; };
  const size_t om = 0, os = up16(n / 8), og = up16(os + n / 16);
  if (mbits_offset) *mbits_offset = om;
  if (scales_offset) *scales_offset = os;
  if (gscale_offset) *gscale_offset = og;
  return up16(og + 4u * (size_t)num_groups);
}

// One cooperative launch (k_capture_coop).  zero_first: zero the workspace
// with a launch of its own first (the static-scratch entry point, whose
// array other calls share); otherwise it is as the previous call left it
// (zeros before the first): the arrival count and the accumulators zero.
static int capture_impl(const uint16_t* x, int64_t rows, int64_t cols, int32_t num_groups,
                        const int64_t* group_row_offsets, uint8_t* codes, uint32_t* mbits,
                        uint8_t* scales, float* gscale, void* workspace, size_t workspace_bytes,
                        bool tiled, void* stream, bool zero_first = false) {
  int st = check_shape(rows, cols, num_groups, group_row_offsets);
  if (st) return st;
  // with no rows only the global scales are written; the data pointers of
  // empty tensors may be NULL
  const bool empty = rows == 0;
  if ((!empty && (!x || !codes || !mbits || !scales)) || !gscale || !workspace) return TRACE_ERR_NULL;
  if (!aligned(x, 32) || !aligned(codes, 16) || !aligned(mbits, 16) || !aligned(scales, 16) ||
      !aligned(gscale, 4) || !aligned(workspace, 256))
    return TRACE_ERR_ALIGN;
  if (workspace_bytes < trace_capture_workspace_bytes(rows, cols, num_groups)) return TRACE_ERR_WORKSPACE;
  const Shape sh = make_shape(rows, cols, num_groups);
  int grid;
  if ((st = tiled ? coop_grid_for<true>(sh, &grid) : coop_grid_for<false>(sh, &grid))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t* ws = (uint32_t*)workspace;
  const int64_t* offs = num_groups > 1 ? group_row_offsets : nullptr;
  const int zn = (int)num_groups + 4;
  const int zg = (zn + kThreads - 1) / kThreads;
  if (zero_first && (st = launch(k_zero_u32, zg < 1024 ? zg : 1024, s, ws, zn))) return st;
  return tiled ? launch_coop(k_capture_coop<true>, grid, s, (const V8*)x, sh, offs, ws,
                             (uint4*)codes, (uint32_t*)mbits, scales, gscale)
               : launch_coop(k_capture_coop<false>, grid, s, (const V8*)x, sh, offs, ws,
                             (uint4*)codes, (uint32_t*)mbits, scales, gscale);
}

int trace_capture_status(void* workspace, void* stream) {
  if (!workspace) return TRACE_ERR_NULL;
  if (!aligned(workspace, 4)) return TRACE_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t* flag = (uint32_t*)workspace + 2;
  uint32_t h = 0u;
  if (cudaMemcpyAsync(&h, flag, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return TRACE_ERR_CUDA;
  if (h == 0u) return TRACE_OK;
  if (cudaMemsetAsync(flag, 0, sizeof(h), s) != cudaSuccess) return TRACE_ERR_CUDA;
  return TRACE_ERR_TIMEOUT;
}

int trace_capture(const uint16_t* x, int64_t rows, int64_t cols, int32_t num_groups,
                  const int64_t* group_row_offsets, uint8_t* codes, uint32_t* mbits,
                  uint8_t* scales, float* gscale, void* workspace, size_t workspace_bytes,
                  void* stream) {
  return capture_impl(x, rows, cols, num_groups, group_row_offsets, codes, mbits, scales, gscale,
                      workspace, workspace_bytes, false, stream);
}


static int fake_quant_launch(int mode, const uint16_t* x, int64_t rows, int64_t cols, int32_t G,
                             const int64_t* offs, const uint32_t* mbits, const uint8_t* rcodes,
                             const uint8_t* scales, const float* gscale, uint16_t* out,
                             uint32_t* mask, void* stream, bool tiled = false) {
  int st = check_shape(rows, cols, G, offs);
  if (st) return st;
  if (rows == 0) return TRACE_OK;  // nothing to do; empty tensors may have NULL data
  if (!x || (mode == kGuided && !mbits) || (mode == kFull && !rcodes) || !scales || !gscale ||
      !out || !mask)
    return TRACE_ERR_NULL;
  if (!aligned(x, 32) || (mode == kGuided && !aligned(mbits, 16)) ||
      (mode == kFull && !aligned(rcodes, 16)) || !aligned(scales, 16) || !aligned(gscale, 4) ||
      !aligned(out, 32) || !aligned(mask, 16))
    return TRACE_ERR_ALIGN;
  const Shape sh = make_shape(rows, cols, G);
  if (sh.nblk == 0) return TRACE_OK;
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t* o = G > 1 ? offs : nullptr;
  return tiled ? fake_quant_dispatch<true>(mode, grid, s, x, sh, o, mbits, rcodes, scales, gscale,
                                           out, mask)
               : fake_quant_dispatch<false>(mode, grid, s, x, sh, o, mbits, rcodes, scales,
                                            gscale, out, mask);
}

int trace_guided_fq_fwd(const uint16_t* x_train, int64_t rows, int64_t cols, int32_t num_groups,
                        const int64_t* group_row_offsets, const uint32_t* mbits,
                        const uint8_t* scales, const float* gscale, uint16_t* out,
                        uint32_t* ste_mask, void* stream) {
  return fake_quant_launch(kGuided, x_train, rows, cols, num_groups, group_row_offsets, mbits,
                           nullptr, scales, gscale, out, ste_mask, stream);
}

int trace_rtn_fq_fwd(const uint16_t* x, int64_t rows, int64_t cols, int32_t num_groups,
                     const int64_t* group_row_offsets, const uint8_t* scales, const float* gscale,
                     uint16_t* out, uint32_t* ste_mask, void* stream) {
  return fake_quant_launch(kRtn, x, rows, cols, num_groups, group_row_offsets, nullptr, nullptr,
                           scales, gscale, out, ste_mask, stream);
}

int trace_full_guided_fq_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                             int32_t num_groups, const int64_t* group_row_offsets,
                             const uint8_t* codes, const uint8_t* scales, const float* gscale,
                             uint16_t* out, uint32_t* ste_mask, void* stream) {
  return fake_quant_launch(kFull, x_train, rows, cols, num_groups, group_row_offsets, nullptr,
                           codes, scales, gscale, out, ste_mask, stream);
}

int trace_mismatch_histogram(const uint16_t* x_train, int64_t rows, int64_t cols,
                             int32_t num_groups, const int64_t* group_row_offsets,
                             const uint8_t* codes, const uint8_t* scales, const float* gscale,
                             uint64_t* hist, void* stream) {
  int st = check_shape(rows, cols, num_groups, group_row_offsets);
  if (st) return st;
  if (!hist) return TRACE_ERR_NULL;
  if (!aligned(hist, 8)) return TRACE_ERR_ALIGN;
  if (rows == 0) return TRACE_OK;  // nothing to count
  if (!x_train || !codes || !scales || !gscale) return TRACE_ERR_NULL;
  if (!aligned(x_train, 32) || !aligned(codes, 16) || !aligned(scales, 16) || !aligned(gscale, 4))
    return TRACE_ERR_ALIGN;
  const Shape sh = make_shape(rows, cols, num_groups);
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  return launch(k_mismatch_hist<false>, grid, (cudaStream_t)stream, (const V8*)x_train, sh,
                num_groups > 1 ? group_row_offsets : nullptr, (const uint4*)codes, scales, gscale,
                (unsigned long long*)hist);
}

int trace_mx_mismatch_histogram(const uint16_t* x_train, int64_t rows, int64_t cols,
                                const uint8_t* codes, const uint8_t* scales, uint64_t* hist,
                                void* stream) {
  int st = check_shape(rows, cols, 1, nullptr);
  if (st) return st;
  if (!hist) return TRACE_ERR_NULL;
  if (!aligned(hist, 8)) return TRACE_ERR_ALIGN;
  if (rows == 0) return TRACE_OK;
  if (!x_train || !codes || !scales) return TRACE_ERR_NULL;
  if (!aligned(x_train, 32) || !aligned(codes, 16)) return TRACE_ERR_ALIGN;
  const Shape sh = make_shape(rows, cols, 1);
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  return launch(k_mismatch_hist<true>, grid, (cudaStream_t)stream, (const V8*)x_train, sh,
                (const int64_t*)nullptr, (const uint4*)codes, scales, (const float*)nullptr,
                (unsigned long long*)hist);
}

static int mx_capture_impl(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* codes,
                           uint32_t* mbits, uint8_t* scales, bool tiled, void* stream) {
  int st = check_shape(rows, cols, 1, nullptr);
  if (st) return st;
  if (rows == 0) return TRACE_OK;
  if (!x || !codes || !mbits || !scales) return TRACE_ERR_NULL;
  if (!aligned(x, 32) || !aligned(codes, 16) || !aligned(mbits, 4)) return TRACE_ERR_ALIGN;
  Shape sh = make_shape(rows, cols, 1);
  sh.sw_ct = (uint32_t)((cols / 32 + 3) / 4);  // cols/32 E8M0 scale columns
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  if (tiled)
    return launch(k_mx_capture<true>, grid, (cudaStream_t)stream, (const V8*)x, sh, (uint4*)codes,
                  mbits, scales);
  return launch(k_mx_capture<false>, grid, (cudaStream_t)stream, (const V8*)x, sh, (uint4*)codes,
                mbits, scales);
}

int trace_mx_capture(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* codes,
                     uint32_t* mbits, uint8_t* scales, void* stream) {
  return mx_capture_impl(x, rows, cols, codes, mbits, scales, false, stream);
}


static int mx_fake_quant_launch(int mode, const uint16_t* x, int64_t rows, int64_t cols,
                                const uint32_t* mbits, const uint8_t* rcodes,
                                const uint8_t* scales, uint16_t* out, uint32_t* mask,
                                void* stream, bool tiled = false) {
  int st = check_shape(rows, cols, 1, nullptr);
  if (st) return st;
  if (rows == 0) return TRACE_OK;
  if (!x || (mode == kGuided && !mbits) || (mode == kFull && !rcodes) || !scales || !out || !mask)
    return TRACE_ERR_NULL;
  if (!aligned(x, 32) || (mode == kGuided && !aligned(mbits, 4)) ||
      (mode == kFull && !aligned(rcodes, 16)) || !aligned(out, 32) || !aligned(mask, 4))
    return TRACE_ERR_ALIGN;
  Shape sh = make_shape(rows, cols, 1);
  sh.sw_ct = (uint32_t)((cols / 32 + 3) / 4);
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  return tiled ? mx_fake_quant_dispatch<true>(mode, grid, s, x, sh, mbits, rcodes, scales, out, mask)
               : mx_fake_quant_dispatch<false>(mode, grid, s, x, sh, mbits, rcodes, scales, out,
                                               mask);
}

int trace_mx_guided_fq_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                           const uint32_t* mbits, const uint8_t* scales, uint16_t* out,
                           uint32_t* ste_mask, void* stream) {
  return mx_fake_quant_launch(kGuided, x_train, rows, cols, mbits, nullptr, scales, out, ste_mask,
                              stream);
}

int trace_mx_full_guided_fq_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                                const uint8_t* codes, const uint8_t* scales, uint16_t* out,
                                uint32_t* ste_mask, void* stream) {
  return mx_fake_quant_launch(kFull, x_train, rows, cols, nullptr, codes, scales, out, ste_mask,
                              stream);
}

int trace_mx_rtn_fq_fwd(const uint16_t* x, int64_t rows, int64_t cols, const uint8_t* scales,
                        uint16_t* out, uint32_t* ste_mask, void* stream) {
  return mx_fake_quant_launch(kRtn, x, rows, cols, nullptr, nullptr, scales, out, ste_mask,
                              stream);
}

size_t trace_scale_bytes(int64_t rows, int64_t cols, int32_t block_size, int32_t scale_layout) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0 || (block_size != 16 && block_size != 32)) return 0;
  const int64_t scols = cols / block_size;
  if (scale_layout == TRACE_SCALES_ROW_MAJOR) return (size_t)(rows * scols);
  if (scale_layout != TRACE_SCALES_TILED_128x4) return 0;
  return (size_t)((rows + 127) / 128) * (size_t)((scols + 3) / 4) * 512u;
}

static bool valid_layout(int32_t layout) {
  return layout == TRACE_SCALES_ROW_MAJOR || layout == TRACE_SCALES_TILED_128x4;
}

int trace_capture_amax(const uint16_t* x, int64_t rows, int64_t cols, int32_t num_groups,
                       const int64_t* group_row_offsets, uint32_t* amax, void* stream) {
  int st = check_shape(rows, cols, num_groups, group_row_offsets);
  if (st) return st;
  if ((rows > 0 && !x) || !amax) return TRACE_ERR_NULL;
  if (!aligned(x, 32) || !aligned(amax, 4)) return TRACE_ERR_ALIGN;
  const Shape sh = make_shape(rows, cols, num_groups);
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int zg = (num_groups + kThreads - 1) / kThreads;
  if ((st = launch(k_zero_u32, zg < 1024 ? zg : 1024, s, amax, (int)num_groups))) return st;
  if (sh.nblk == 0) return TRACE_OK;
  return launch(k_amax, grid, s, (const V8*)x, sh, num_groups > 1 ? group_row_offsets : nullptr,
                amax);
}

int trace_capture_amax_accumulate(const uint16_t* x, int64_t rows, int64_t cols,
                                  int32_t num_groups, const int64_t* group_row_offsets,
                                  uint32_t* amax, void* stream) {
  int st = check_shape(rows, cols, num_groups, group_row_offsets);
  if (st) return st;
  if ((rows > 0 && !x) || !amax) return TRACE_ERR_NULL;
  if (!aligned(x, 32) || !aligned(amax, 4)) return TRACE_ERR_ALIGN;
  const Shape sh = make_shape(rows, cols, num_groups);
  if (sh.nblk == 0) return TRACE_OK;
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  return launch(k_amax, grid, (cudaStream_t)stream, (const V8*)x, sh,
                num_groups > 1 ? group_row_offsets : nullptr, amax);
}

int trace_capture_with_amax(const uint16_t* x, int64_t rows, int64_t cols, int32_t num_groups,
                            const int64_t* group_row_offsets, const uint32_t* amax,
                            uint8_t* codes, uint32_t* mbits, uint8_t* scales, float* gscale,
                            int32_t scale_layout, void* stream) {
  int st = check_shape(rows, cols, num_groups, group_row_offsets);
  if (st) return st;
  if (!valid_layout(scale_layout)) return TRACE_ERR_SHAPE;
  if ((rows > 0 && (!x || !codes || !mbits || !scales)) || !gscale || !amax) return TRACE_ERR_NULL;
  if (!aligned(x, 32) || !aligned(codes, 16) || !aligned(mbits, 16) || !aligned(scales, 16) ||
      !aligned(gscale, 4) || !aligned(amax, 4))
    return TRACE_ERR_ALIGN;
  const Shape sh = make_shape(rows, cols, num_groups);
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t* offs = num_groups > 1 ? group_row_offsets : nullptr;
  if (scale_layout == TRACE_SCALES_TILED_128x4)
    return launch(k_capture<true>, grid, s, (const V8*)x, sh, offs, amax, (uint4*)codes, mbits,
                  scales, gscale);
  return launch(k_capture<false>, grid, s, (const V8*)x, sh, offs, amax, (uint4*)codes, mbits,
                scales, gscale);
}

int trace_capture_ex(const uint16_t* x, int64_t rows, int64_t cols, int32_t num_groups,
                     const int64_t* group_row_offsets, uint8_t* codes, uint32_t* mbits,
                     uint8_t* scales, float* gscale, void* workspace, size_t workspace_bytes,
                     int32_t scale_layout, void* stream) {
  if (!valid_layout(scale_layout)) return TRACE_ERR_SHAPE;
  return capture_impl(x, rows, cols, num_groups, group_row_offsets, codes, mbits, scales, gscale,
                      workspace, workspace_bytes, scale_layout == TRACE_SCALES_TILED_128x4, stream);
}

int trace_fq_fwd_ex(int32_t rule, const uint16_t* x_train, int64_t rows, int64_t cols,
                    int32_t num_groups, const int64_t* group_row_offsets, const uint32_t* mbits,
                    const uint8_t* codes, const uint8_t* scales, const float* gscale, uint16_t* out,
                    uint32_t* ste_mask, int32_t scale_layout, void* stream) {
  if (!valid_layout(scale_layout) || rule < TRACE_RULE_RTN || rule > TRACE_RULE_FULL)
    return TRACE_ERR_SHAPE;
  return fake_quant_launch(rule, x_train, rows, cols, num_groups, group_row_offsets, mbits, codes,
                           scales, gscale, out, ste_mask, stream,
                           scale_layout == TRACE_SCALES_TILED_128x4);
}

int trace_mx_capture_ex(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* codes,
                        uint32_t* mbits, uint8_t* scales, int32_t scale_layout, void* stream) {
  if (!valid_layout(scale_layout)) return TRACE_ERR_SHAPE;
  return mx_capture_impl(x, rows, cols, codes, mbits, scales,
                         scale_layout == TRACE_SCALES_TILED_128x4, stream);
}

int trace_mx_fq_fwd_ex(int32_t rule, const uint16_t* x_train, int64_t rows, int64_t cols,
                       const uint32_t* mbits, const uint8_t* codes, const uint8_t* scales,
                       uint16_t* out, uint32_t* ste_mask, int32_t scale_layout, void* stream) {
  if (!valid_layout(scale_layout) || rule < TRACE_RULE_RTN || rule > TRACE_RULE_FULL)
    return TRACE_ERR_SHAPE;
  return mx_fake_quant_launch(rule, x_train, rows, cols, mbits, codes, scales, out, ste_mask,
                              stream, scale_layout == TRACE_SCALES_TILED_128x4);
}

static int mx8_capture_impl(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* codes,
                            uint32_t* mbits, uint8_t* scales, bool tiled, void* stream) {
  int st = check_shape(rows, cols, 1, nullptr);
  if (st) return st;
  if (rows == 0) return TRACE_OK;
  if (!x || !codes || !mbits || !scales) return TRACE_ERR_NULL;
  if (!aligned(x, 32) || !aligned(codes, 32) || !aligned(mbits, 4)) return TRACE_ERR_ALIGN;
  Shape sh = make_shape(rows, cols, 1);
  sh.sw_ct = (uint32_t)((cols / 32 + 3) / 4);
  int grid;
  if ((st = grid_for(sh, &grid))) return st;
  if (tiled)
    return launch(k_mx8_capture<true>, grid, (cudaStream_t)stream, (const V8*)x, sh, (V8*)codes,
                  mbits, scales);
  return launch(k_mx8_capture<false>, grid, (cudaStream_t)stream, (const V8*)x, sh, (V8*)codes,
                mbits, scales);
}

int trace_mx8_capture(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* codes,
                      uint32_t* mbits, uint8_t* scales, void* stream) {
  return mx8_capture_impl(x, rows, cols, codes, mbits, scales, false, stream);
}

int trace_mx8_capture_ex(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* codes,
                         uint32_t* mbits, uint8_t* scales, int32_t scale_layout, void* stream) {
  if (scale_layout != TRACE_SCALES_ROW_MAJOR && scale_layout != TRACE_SCALES_TILED_128x4)
    return TRACE_ERR_SHAPE;
  return mx8_capture_impl(x, rows, cols, codes, mbits, scales,
                          scale_layout == TRACE_SCALES_TILED_128x4, stream);
}

int trace_mx8_fq_fwd_ex(int32_t rule, const uint16_t* x_train, int64_t rows, int64_t cols,
                        const uint32_t* mbits, const uint8_t* codes, const uint8_t* scales,
                        uint16_t* out, uint32_t* ste_mask, int32_t scale_layout, void* stream) {
  if ((scale_layout != TRACE_SCALES_ROW_MAJOR && scale_layout != TRACE_SCALES_TILED_128x4) ||
      rule < TRACE_RULE_RTN || rule > TRACE_RULE_FULL)
    return TRACE_ERR_SHAPE;
  const bool tiled = scale_layout == TRACE_SCALES_TILED_128x4;
  if (rule == TRACE_RULE_GUIDED)
    return mx8_launch<kGuided>(x_train, rows, cols, mbits, nullptr, scales, out, ste_mask, stream,
                               tiled);
  if (rule == TRACE_RULE_FULL)
    return mx8_launch<kFull>(x_train, rows, cols, nullptr, codes, scales, out, ste_mask, stream,
                             tiled);
  return mx8_launch<kRtn>(x_train, rows, cols, nullptr, nullptr, scales, out, ste_mask, stream,
                          tiled);
}

int trace_mx8_guided_fq_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                            const uint32_t* mbits, const uint8_t* scales, uint16_t* out,
                            uint32_t* ste_mask, void* stream) {
  return mx8_launch<kGuided>(x_train, rows, cols, mbits, nullptr, scales, out, ste_mask, stream);
}

int trace_mx8_full_guided_fq_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                                 const uint8_t* codes, const uint8_t* scales, uint16_t* out,
                                 uint32_t* ste_mask, void* stream) {
  return mx8_launch<kFull>(x_train, rows, cols, nullptr, codes, scales, out, ste_mask, stream);
}

int trace_mx8_rtn_fq_fwd(const uint16_t* x, int64_t rows, int64_t cols, const uint8_t* scales,
                         uint16_t* out, uint32_t* ste_mask, void* stream) {
  return mx8_launch<kRtn>(x, rows, cols, nullptr, nullptr, scales, out, ste_mask, stream);
}

int trace_selftest_e4m3_sweep(uint32_t first_bits, uint32_t count, uint8_t* out,
                              void* stream) {
  if (count == 0) return TRACE_OK;
  if (!out) return TRACE_ERR_NULL;
  // positive finite inputs only: the last bit pattern must stay below +inf
  if (first_bits >= 0x7F800000u || count > 0x7F800000u - first_bits) return TRACE_ERR_SHAPE;
  const int sms = sm_count();
  if (sms <= 0) return TRACE_ERR_CUDA;
  k_selftest_e4m3<<<sms * 8, 256, 0, (cudaStream_t)stream>>>(first_bits, count, out);
  return cudaGetLastError() == cudaSuccess ? TRACE_OK : TRACE_ERR_CUDA;
}

int trace_validate_offsets(const int64_t* group_row_offsets, int32_t num_groups, int64_t rows,
                           uint32_t* flag, void* stream) {
  if (num_groups < 1 || rows < 0) return TRACE_ERR_SHAPE;
  if (!group_row_offsets || !flag) return TRACE_ERR_NULL;
  if (!aligned(group_row_offsets, 8) || !aligned(flag, 4)) return TRACE_ERR_ALIGN;
  // one CTA: a debugging aid, not a hot path
  k_validate_offsets<<<1, 1024, 0, (cudaStream_t)stream>>>(group_row_offsets, num_groups, rows,
                                                          flag);
  return cudaGetLastError() == cudaSuccess ? TRACE_OK : TRACE_ERR_CUDA;
}

int trace_fq_bwd(const uint16_t* grad_out, const uint32_t* ste_mask, int64_t numel,
                 uint16_t* grad_in, void* stream) {
  if (numel < 0 || numel % 32 != 0) return TRACE_ERR_SHAPE;
  if ((long double)numel / 16 >= 4294967296.0L - (long double)kTileBlks) return TRACE_ERR_SHAPE;
  if (numel == 0) return TRACE_OK;
  if (!grad_out || !ste_mask || !grad_in) return TRACE_ERR_NULL;
  if (!aligned(grad_out, 32) || !aligned(ste_mask, 16) || !aligned(grad_in, 32)) return TRACE_ERR_ALIGN;
  const Shape sh = make_shape(numel / 32, 32, 1);
  int grid, st;
  if ((st = grid_for(sh, &grid))) return st;
  return launch(k_ste_bwd, grid, (cudaStream_t)stream, (const V8*)grad_out, sh,
                (const uint32_t*)ste_mask, (V8*)grad_in);
}

int trace_copy_bf16(const uint16_t* src, uint16_t* dst, int64_t numel, void* stream) {
  if (numel < 0 || numel % 16 != 0) return TRACE_ERR_SHAPE;
  if ((long double)numel / 16 >= 4294967296.0L - (long double)kTileBlks) return TRACE_ERR_SHAPE;
  if (numel == 0) return TRACE_OK;
  if (!src || !dst) return TRACE_ERR_NULL;
  if (!aligned(src, 32) || !aligned(dst, 32)) return TRACE_ERR_ALIGN;
  Shape sh;
  sh.nblk = (uint32_t)(numel / 16);
  sh.ntiles = (uint32_t)(((uint64_t)sh.nblk + kTileBlks - 1) / kTileBlks);
  sh.bpr = make_fastdiv(1);
  sh.G = 1;
  sh.sw_ct = 1;
  int grid, st;
  if ((st = grid_for(sh, &grid))) return st;
  return launch(k_copy, grid, (cudaStream_t)stream, (const V8*)src, sh, (V8*)dst);
}


int trace_copy_bf16_staged(const uint16_t* src, uint16_t* dst, int64_t numel, uint32_t* err,
                           void* stream) {
  if (numel < 0 || numel % 16 != 0) return TRACE_ERR_SHAPE;
  if ((long double)numel / 16 >= 4294967296.0L - (long double)kTileBlks) return TRACE_ERR_SHAPE;
  if (numel == 0) return TRACE_OK;
  if (!src || !dst || !err) return TRACE_ERR_NULL;
  if (!aligned(src, 32) || !aligned(dst, 32) || !aligned(err, 4)) return TRACE_ERR_ALIGN;
  Shape sh;
  sh.nblk = (uint32_t)(numel / 16);
  sh.ntiles = (uint32_t)(((uint64_t)sh.nblk + kTileBlks - 1) / kTileBlks);
  sh.bpr = make_fastdiv(1);
  sh.G = 1;
  sh.sw_ct = 1;
  const int sms = sm_count();
  if (sms <= 0) return TRACE_ERR_CUDA;
  const size_t smem = (size_t)kStages * kTileBytes;  // 64 KiB: two CTAs per SM
  static bool attr_set[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TRACE_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(k_copy_staged, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return TRACE_ERR_CUDA;
    attr_set[dev] = true;
  }
  uint32_t grid = (uint32_t)sms * 2u;
  if (sh.ntiles < grid) grid = sh.ntiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_copy_staged, (const V8*)src, sh, (V8*)dst, err) == cudaSuccess
             ? TRACE_OK
             : TRACE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Capture without a caller-provided workspace.
//
// Some callers cannot hand the library a scratch buffer: a host program whose
// device memory is carved up once at start-up and may not grow afterwards, or
// a thin binding that only forwards the tensors it was given and has no
// allocator to call.  This entry point therefore keeps the amax accumulators
// that trace_capture takes as `workspace` in a fixed array that lives in the
// library itself, one copy per GPU, for the life of the process.
// ---------------------------------------------------------------------------
// TRACE_STATIC_MAX_GROUPS accumulators, the four words before them and
// padding to a multiple of 256 bytes
static __device__ __align__(256) uint32_t g_capture_scratch[TRACE_STATIC_MAX_GROUPS + 64];

static void* g_capture_scratch_addr[kMaxDevices];  // per device; benign race (same value)

int trace_capture_static_ws(const uint16_t* x, int64_t rows, int64_t cols, int32_t num_groups,
                            const int64_t* group_row_offsets, uint8_t* codes, uint32_t* mbits,
                            uint8_t* scales, float* gscale, void* stream) {
  if (num_groups > TRACE_STATIC_MAX_GROUPS) return TRACE_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TRACE_ERR_CUDA;
  // The host-side name of the array is only a stand-in, so the kernels get
  // the address the runtime reports for the current device.  It is looked up
  // on the first call on a device and again on every call made outside
  // stream capture: cudaDeviceReset unloads the module, and the array may
  // come back at another address.  While the stream is capturing, the
  // address found by an earlier call is used.
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  bool capturing = true;
  if (cudaStreamIsCapturing((cudaStream_t)stream, &cs) == cudaSuccess)
    capturing = cs != cudaStreamCaptureStatusNone;
  else
    (void)cudaGetLastError();  // the query failed: treat the stream as capturing
  void* ws = g_capture_scratch_addr[dev];
  if (!capturing || ws == nullptr) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_capture_scratch) != cudaSuccess || a == nullptr)
      return TRACE_ERR_CUDA;
    g_capture_scratch_addr[dev] = ws = a;
  }
  // the array is zeroed by the capture's first kernel on every call
  return capture_impl(x, rows, cols, num_groups, group_row_offsets, codes, mbits, scales, gscale,
                      ws, sizeof(g_capture_scratch), false, stream, true);
}

}  // extern "C"
