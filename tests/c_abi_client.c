/*
 * c_abi_client.c -- a plain C user of libtrace_fp4.so: no Python, no torch.
 *
 * Builds a small deterministic rollout / training pair of bf16 activations
 * (two groups of rows), runs the rollout capture, the guided fake-quant
 * forward, the straight-through backward and the round-to-nearest comparator
 * through the C ABI in include/trace_fp4.h, checks a few argument errors, and
 * writes inputs and outputs to a binary file for the test that compares them
 * with the oracle:  c_abi_client OUT_FILE
 *
 * Output file: int64 rows, int64 cols, int32 groups, int64 offsets[G+1],
 * then x_roll, x_train, grad (uint16[N] each), codes (uint8[N/2]),
 * mbits (uint32[N/32]), scales (uint8[N/16]), gscale (float[G]),
 * out (uint16[N]), mask (uint32[N/32]), grad_in (uint16[N]),
 * out_rtn (uint16[N]), mask_rtn (uint32[N/32]).
 */
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "trace_fp4.h"

#define ROWS 96
#define COLS 256
#define GROUPS 2

static uint32_t lcg_state = 12345u;
static uint32_t lcg(void) {
  lcg_state = lcg_state * 1664525u + 1013904223u;
  return lcg_state >> 8;
}

/* a finite bf16 pattern: random sign and 7-bit mantissa, exponent in a band */
static uint16_t rand_bf16(int exp_lo, int exp_span) {
  const uint32_t s = lcg() & 1u, e = (uint32_t)exp_lo + lcg() % (uint32_t)exp_span;
  return (uint16_t)((s << 15) | (e << 7) | (lcg() & 0x7Fu));
}

#define CK(call)                                                         \
  do {                                                                   \
    cudaError_t e_ = (call);                                             \
    if (e_ != cudaSuccess) {                                             \
      fprintf(stderr, "%s failed: %s\n", #call, cudaGetErrorString(e_)); \
      return 2;                                                          \
    }                                                                    \
  } while (0)

#define TK(call, want)                                                        \
  do {                                                                        \
    int s_ = (call);                                                          \
    if (s_ != (want)) {                                                       \
      fprintf(stderr, "%s returned %d (%s), expected %d\n", #call, s_,        \
              trace_strerror(s_), (want));                                    \
      return 3;                                                               \
    }                                                                         \
  } while (0)

int main(int argc, char** argv) {
  if (argc != 2) {
    fprintf(stderr, "usage: %s OUT_FILE\n", argv[0]);
    return 1;
  }
  if (trace_abi_version() != TRACE_ABI_VERSION) return 4;
  const int64_t n = (int64_t)ROWS * COLS;
  const int64_t offs[GROUPS + 1] = {0, 40, ROWS};
  uint16_t* xr = malloc(n * 2);
  uint16_t* xt = malloc(n * 2);
  uint16_t* g = malloc(n * 2);
  for (int64_t i = 0; i < n; ++i) {
    const int row = (int)(i / COLS);
    xr[i] = rand_bf16(row < 40 ? 118 : 125, 10); /* group 1 about 2^7 larger */
    /* training side: the same value, or its bf16 neighbour either way */
    const uint32_t r = lcg() % 4u;
    xt[i] = (uint16_t)(r == 0 ? xr[i] + 1 : (r == 1 && (xr[i] & 0x7F) ? xr[i] - 1 : xr[i]));
    g[i] = rand_bf16(120, 14);
  }
  /* a zero block and a negative zero */
  memset(xr + 3 * COLS, 0, 16 * 2);
  xr[5] = 0x8000;

  uint16_t *d_xr, *d_xt, *d_g, *d_out, *d_gin, *d_outr;
  uint8_t *d_codes, *d_scales;
  uint32_t *d_mbits, *d_mask, *d_maskr;
  float* d_gs;
  int64_t* d_offs;
  void* d_ws;
  const size_t ws_bytes = trace_capture_workspace_bytes(ROWS, COLS, GROUPS);
  CK(cudaMalloc((void**)&d_xr, n * 2));
  CK(cudaMalloc((void**)&d_xt, n * 2));
  CK(cudaMalloc((void**)&d_g, n * 2));
  CK(cudaMalloc((void**)&d_out, n * 2));
  CK(cudaMalloc((void**)&d_gin, n * 2));
  CK(cudaMalloc((void**)&d_outr, n * 2));
  CK(cudaMalloc((void**)&d_codes, n / 2));
  CK(cudaMalloc((void**)&d_scales, n / 16));
  CK(cudaMalloc((void**)&d_mbits, n / 8));
  CK(cudaMalloc((void**)&d_mask, n / 8));
  CK(cudaMalloc((void**)&d_maskr, n / 8));
  CK(cudaMalloc((void**)&d_gs, GROUPS * 4));
  CK(cudaMalloc((void**)&d_offs, sizeof offs));
  CK(cudaMalloc(&d_ws, ws_bytes));
  CK(cudaMemset(d_ws, 0, ws_bytes)); /* zeros before first use */
  CK(cudaMemcpy(d_xr, xr, n * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(d_xt, xt, n * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(d_g, g, n * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(d_offs, offs, sizeof offs, cudaMemcpyHostToDevice));
  cudaStream_t st;
  CK(cudaStreamCreate(&st));

  /* argument errors return before anything is enqueued */
  TK(trace_capture(d_xr, ROWS, 48, GROUPS, d_offs, d_codes, d_mbits, d_scales, d_gs, d_ws,
                   ws_bytes, st), TRACE_ERR_SHAPE);
  TK(trace_capture(d_xr, ROWS, COLS, GROUPS, d_offs, d_codes, d_mbits, d_scales, d_gs, d_ws, 0,
                   st), TRACE_ERR_WORKSPACE);
  TK(trace_guided_fq_fwd((const uint16_t*)((const char*)d_xt + 2), ROWS, COLS, GROUPS, d_offs,
                         d_mbits, d_scales, d_gs, d_out, d_mask, st), TRACE_ERR_ALIGN);
  TK(trace_fq_bwd(NULL, d_mask, n, d_gin, st), TRACE_ERR_NULL);

  /* the path: rollout capture, guided forward, backward, comparator */
  TK(trace_capture(d_xr, ROWS, COLS, GROUPS, d_offs, d_codes, d_mbits, d_scales, d_gs, d_ws,
                   ws_bytes, st), TRACE_OK);
  TK(trace_guided_fq_fwd(d_xt, ROWS, COLS, GROUPS, d_offs, d_mbits, d_scales, d_gs, d_out, d_mask,
                         st), TRACE_OK);
  TK(trace_fq_bwd(d_g, d_mask, n, d_gin, st), TRACE_OK);
  TK(trace_rtn_fq_fwd(d_xt, ROWS, COLS, GROUPS, d_offs, d_scales, d_gs, d_outr, d_maskr, st),
     TRACE_OK);
  CK(cudaStreamSynchronize(st));

  uint8_t* codes = malloc(n / 2);
  uint8_t* scales = malloc(n / 16);
  uint32_t* mbits = malloc(n / 8);
  uint32_t* mask = malloc(n / 8);
  uint32_t* maskr = malloc(n / 8);
  uint16_t* out = malloc(n * 2);
  uint16_t* gin = malloc(n * 2);
  uint16_t* outr = malloc(n * 2);
  float gs[GROUPS];
  CK(cudaMemcpy(codes, d_codes, n / 2, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(scales, d_scales, n / 16, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(mbits, d_mbits, n / 8, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(mask, d_mask, n / 8, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(maskr, d_maskr, n / 8, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(out, d_out, n * 2, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(gin, d_gin, n * 2, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(outr, d_outr, n * 2, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(gs, d_gs, sizeof gs, cudaMemcpyDeviceToHost));

  FILE* f = fopen(argv[1], "wb");
  if (!f) return 5;
  const int64_t rows = ROWS, cols = COLS;
  const int32_t groups = GROUPS;
  fwrite(&rows, 8, 1, f);
  fwrite(&cols, 8, 1, f);
  fwrite(&groups, 4, 1, f);
  fwrite(offs, 8, GROUPS + 1, f);
  fwrite(xr, 2, n, f);
  fwrite(xt, 2, n, f);
  fwrite(g, 2, n, f);
  fwrite(codes, 1, n / 2, f);
  fwrite(mbits, 4, n / 32, f);
  fwrite(scales, 1, n / 16, f);
  fwrite(gs, 4, GROUPS, f);
  fwrite(out, 2, n, f);
  fwrite(mask, 4, n / 32, f);
  fwrite(gin, 2, n, f);
  fwrite(outr, 2, n, f);
  fwrite(maskr, 4, n / 32, f);
  fclose(f);
  printf("c_abi_client: ok\n");
  return 0;
}
