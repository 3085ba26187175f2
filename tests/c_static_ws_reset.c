/*
 * c_static_ws_reset.c -- trace_capture_static_ws across cudaDeviceReset, from
 * plain C (no Python, no torch).
 *
 * cudaDeviceReset tears down the device's primary context; the next runtime
 * call builds a new one and loads the library's module again, so the static
 * scratch array can sit at a different device address afterwards.  This
 * program runs the capture without a workspace before and after a reset and
 * compares every output byte with trace_capture given a workspace that this
 * program allocates itself.  Exit code 0 when all outputs match.
 */
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "trace_fp4.h"

#define ROWS 160
#define COLS 256
#define GROUPS 3

static uint32_t lcg_state = 777u;
static uint32_t lcg(void) {
  lcg_state = lcg_state * 1664525u + 1013904223u;
  return lcg_state >> 8;
}

#define CK(call)                                                         \
  do {                                                                   \
    cudaError_t e_ = (call);                                             \
    if (e_ != cudaSuccess) {                                             \
      fprintf(stderr, "%s failed: %s\n", #call, cudaGetErrorString(e_)); \
      return 2;                                                          \
    }                                                                    \
  } while (0)

#define TK(call)                                                               \
  do {                                                                         \
    int s_ = (call);                                                           \
    if (s_ != TRACE_OK) {                                                      \
      fprintf(stderr, "%s returned %d (%s)\n", #call, s_, trace_strerror(s_)); \
      return 3;                                                                \
    }                                                                          \
  } while (0)

/* One round: fresh device buffers, both captures, byte comparison.  The
 * exponent band `e0` differs between rounds so that a stale accumulator
 * would change the global scales. */
static int one_round(int e0, int round) {
  const size_t n = (size_t)ROWS * COLS;
  uint16_t* hx = (uint16_t*)malloc(n * 2);
  for (size_t i = 0; i < n; ++i) {
    const uint32_t s = lcg() & 1u, e = (uint32_t)e0 + lcg() % 6u;
    hx[i] = (uint16_t)((s << 15) | (e << 7) | (lcg() & 0x7Fu));
  }
  const int64_t hoffs[GROUPS + 1] = {0, 64, 64, ROWS};
  uint16_t* x;
  int64_t* offs;
  void* ws;
  uint8_t *codes[2], *scales[2];
  uint32_t* mbits[2];
  float* gscale[2];
  const size_t wsb = trace_capture_workspace_bytes(ROWS, COLS, GROUPS);
  CK(cudaMalloc((void**)&x, n * 2));
  CK(cudaMalloc((void**)&offs, sizeof(hoffs)));
  CK(cudaMalloc(&ws, wsb));
  CK(cudaMemset(ws, 0, wsb)); /* zeros before first use */
  for (int k = 0; k < 2; ++k) {
    CK(cudaMalloc((void**)&codes[k], n / 2));
    CK(cudaMalloc((void**)&mbits[k], n / 8));
    CK(cudaMalloc((void**)&scales[k], n / 16));
    CK(cudaMalloc((void**)&gscale[k], GROUPS * sizeof(float)));
    CK(cudaMemset(codes[k], 0x5A + k, n / 2));
    CK(cudaMemset(mbits[k], 0xA5 + k, n / 8));
    CK(cudaMemset(scales[k], 0x33 + k, n / 16));
    CK(cudaMemset(gscale[k], 0x7F - k, GROUPS * sizeof(float)));
  }
  CK(cudaMemcpy(x, hx, n * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(offs, hoffs, sizeof(hoffs), cudaMemcpyHostToDevice));
  TK(trace_capture(x, ROWS, COLS, GROUPS, offs, codes[0], mbits[0], scales[0], gscale[0], ws,
                   wsb, NULL));
  TK(trace_capture_static_ws(x, ROWS, COLS, GROUPS, offs, codes[1], mbits[1], scales[1],
                             gscale[1], NULL));
  CK(cudaDeviceSynchronize());
  const size_t sizes[4] = {n / 2, n / 8, n / 16, GROUPS * sizeof(float)};
  void* bufs[2][4] = {{codes[0], mbits[0], scales[0], gscale[0]},
                      {codes[1], mbits[1], scales[1], gscale[1]}};
  int bad = 0;
  for (int j = 0; j < 4; ++j) {
    unsigned char* a = (unsigned char*)malloc(sizes[j]);
    unsigned char* b = (unsigned char*)malloc(sizes[j]);
    CK(cudaMemcpy(a, bufs[0][j], sizes[j], cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(b, bufs[1][j], sizes[j], cudaMemcpyDeviceToHost));
    if (memcmp(a, b, sizes[j]) != 0) {
      fprintf(stderr, "round %d: output %d differs\n", round, j);
      bad = 1;
    }
    free(a);
    free(b);
  }
  free(hx);
  return bad ? 4 : 0;
}

int main(void) {
  int rc = one_round(120, 0);
  if (rc) return rc;
  CK(cudaDeviceReset());
  rc = one_round(100, 1); /* new context: the first call after the reset */
  if (rc) return rc;
  rc = one_round(130, 2);
  if (rc) return rc;
  printf("static-workspace capture matches trace_capture before and after cudaDeviceReset\n");
  return 0;
}
