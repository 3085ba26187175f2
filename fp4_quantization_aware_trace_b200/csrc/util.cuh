// util.cuh -- the E4M3 rounding self-test kernel and the plain copy used as
// the bandwidth yardstick.  Included by trace_fp4.cu inside its anonymous
// namespace.
#pragma once

// ---------------------------------------------------------------------------
// Self-test kernel: the block-scale rounding (cvt_e4m3, as capture uses it)
// on fp32 inputs generated from their index, for exhaustive checks.
// ---------------------------------------------------------------------------
__global__ void k_selftest_e4m3(uint32_t first_bits, uint32_t count, uint8_t* __restrict__ out) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += gridDim.x * blockDim.x)
    out[i] = (uint8_t)cvt_e4m3(__uint_as_float(first_bits + i));
}

// ---------------------------------------------------------------------------
// Kernel 6: plain copy with the same access pattern (bandwidth yardstick).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_copy(const V8* __restrict__ s, Shape sh, V8* __restrict__ d) {
  pdl_begin();
  for (uint32_t t = blockIdx.x; t < sh.ntiles; t += gridDim.x) {
    V8 v[kBlkPerThread];
    const uint32_t base = t * kTileBlks + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kBlkPerThread; ++u) {
      const uint32_t b = base + u * kThreads;
      v[u] = b < sh.nblk ? ld_block_stream(s + b) : zero_block();
    }
#pragma unroll
    for (int u = 0; u < kBlkPerThread; ++u) {
      const uint32_t b = base + u * kThreads;
      if (b < sh.nblk) st_block(d + b, v[u]);
    }
  }
}

// Group-offset check, one CTA: flag = 0 when offsets[0] == 0,
// offsets[G] == rows and offsets never decrease; else 1 + the index of the
// first offending entry.
__global__ void __launch_bounds__(1024) k_validate_offsets(const int64_t* __restrict__ offs,
                                                           int32_t G, int64_t rows,
                                                           uint32_t* __restrict__ flag) {
  __shared__ uint32_t first_bad;
  if (threadIdx.x == 0) first_bad = 0xFFFFFFFFu;
  __syncthreads();
  uint32_t bad = 0xFFFFFFFFu;
  for (int64_t i = threadIdx.x; i <= G; i += blockDim.x) {
    const int64_t v = offs[i];
    const bool ok = (i == 0 ? v == 0 : v >= offs[i - 1]) && (i < G || v == rows) && v <= rows;
    if (!ok && (uint32_t)i < bad) bad = (uint32_t)i;
  }
  if (bad != 0xFFFFFFFFu) atomicMin(&first_bad, bad);
  __syncthreads();
  if (threadIdx.x == 0) *flag = first_bad == 0xFFFFFFFFu ? 0u : first_bad + 1u;
}
