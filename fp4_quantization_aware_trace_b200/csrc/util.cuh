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

// ---------------------------------------------------------------------------
// Kernel 6b: the same copy with its reads staged through shared memory by
// the bulk-copy engine (cp.async.bulk global -> shared, completion counted on
// an mbarrier per stage), kStages tiles in flight per CTA: the yardstick of
// a TMA-staged pipeline, to compare with the plain copy above.  Each CTA
// walks tiles c, c + gridDim.x, ...; thread 0 issues the loads; every
// thread waits for its stage, moves its two blocks to registers and stores
// them.  Waits are bounded: thread 0 alone polls the stage's mbarrier; after
// kStageSpin polls it records 1 in *err and the whole CTA leaves the loop
// together (a healthy copy never comes close).
// ---------------------------------------------------------------------------
constexpr int kStages = 4;
constexpr uint32_t kStageSpin = 1u << 22;
constexpr uint32_t kTileBytes = kTileBlks * 32u;  // 16 KiB

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok)
               : "r"(bar), "r"(parity)
               : "memory");
  return ok != 0u;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    k_copy_staged(const V8* __restrict__ s, Shape sh, V8* __restrict__ d, uint32_t* err) {
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) unsigned long long full[kStages];
  pdl_begin();
  const uint32_t G = gridDim.x;
  auto tile_bytes = [&](uint32_t t) {
    const uint32_t left = sh.nblk - t * kTileBlks;
    return (left < (uint32_t)kTileBlks ? left : (uint32_t)kTileBlks) * 32u;
  };
  if (threadIdx.x == 0) {
    for (int k = 0; k < kStages; ++k)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&full[k])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int k = 0; k < kStages; ++k) {
      const uint32_t t = blockIdx.x + (uint32_t)k * G;
      if (t < sh.ntiles)
        bulk_load(smem_u32(stage_mem + k * kTileBytes), s + (size_t)t * kTileBlks, tile_bytes(t),
                  smem_u32(&full[k]));
    }
  }
  __shared__ uint32_t abort_s;
  if (threadIdx.x == 0) abort_s = 0u;
  __syncthreads();
  uint32_t i = 0;
  for (uint32_t t = blockIdx.x; t < sh.ntiles; t += G, ++i) {
    const int k = (int)(i % kStages);
    if (threadIdx.x == 0) {
      const uint32_t parity = (i / kStages) & 1u;
      uint32_t spins = 0;
      while (!mbar_try_wait(smem_u32(&full[k]), parity)) {
        if (++spins == kStageSpin) {
          atomicExch(err, 1u);
          abort_s = 1u;
          break;
        }
      }
    }
    __syncthreads();  // the stage is full (thread 0 saw its phase complete)
    if (abort_s) break;
    const V8* st = reinterpret_cast<const V8*>(stage_mem + k * kTileBytes);
    const uint32_t base = t * kTileBlks;
    V8 v[kBlkPerThread];
#pragma unroll
    for (int u = 0; u < kBlkPerThread; ++u) {
      const uint32_t j = threadIdx.x + u * kThreads;
      if (base + j < sh.nblk) v[u] = st[j];
    }
    __syncthreads();  // every thread has read the stage
    if (threadIdx.x == 0) {
      const uint32_t tn = t + (uint32_t)kStages * G;
      if (tn < sh.ntiles) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        bulk_load(smem_u32(stage_mem + k * kTileBytes), s + (size_t)tn * kTileBlks,
                  tile_bytes(tn), smem_u32(&full[k]));
      }
    }
#pragma unroll
    for (int u = 0; u < kBlkPerThread; ++u) {
      const uint32_t j = threadIdx.x + u * kThreads;
      if (base + j < sh.nblk) st_block(d + base + j, v[u]);
    }
  }
}
