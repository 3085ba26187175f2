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
