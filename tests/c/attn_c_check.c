/* A plain C caller of the attention entry point on a B200: the caller owns
 * every device buffer (cudaMalloc), the library enqueues on the default
 * stream, and the result is checked against dense softmax attention computed
 * here in double precision (every block kept, a ragged last block of 44 rows).
 * Prints "ok" and returns 0, or names the first failed check. */
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "calibatt.h"

#define CHECK(cond)                                      \
  do {                                                   \
    if (!(cond)) {                                       \
      printf("failed: %s (line %d)\n", #cond, __LINE__); \
      return 1;                                          \
    }                                                    \
  } while (0)

enum { HEADS = 2, N = 300, D = 128, NB = (N + 127) / 128 };

static uint16_t to_bf16(float x) { /* round to nearest even */
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static double from_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

int main(void) {
  const size_t elems = (size_t)HEADS * N * D;
  uint16_t* q = malloc(elems * 2);
  uint16_t* k = malloc(elems * 2);
  uint16_t* v = malloc(elems * 2);
  uint16_t* o = malloc(elems * 2);
  CHECK(q && k && v && o);
  unsigned s = 12345u;
  for (size_t i = 0; i < elems; ++i) {
    s = s * 1664525u + 1013904223u;
    q[i] = to_bf16(((s >> 8) & 0xFFFF) / 32768.0f - 1.0f);
    s = s * 1664525u + 1013904223u;
    k[i] = to_bf16(((s >> 8) & 0xFFFF) / 32768.0f - 1.0f);
    s = s * 1664525u + 1013904223u;
    v[i] = to_bf16(((s >> 8) & 0xFFFF) / 32768.0f - 1.0f);
  }
  /* every block kept */
  int32_t row_ptr[HEADS * NB + 1], col_idx[HEADS * NB * NB], work[HEADS * NB], n_work = 0;
  row_ptr[0] = 0;
  for (int u = 0; u < HEADS * NB; ++u) {
    for (int c = 0; c < NB; ++c) col_idx[u * NB + c] = c;
    row_ptr[u + 1] = row_ptr[u] + NB;
  }
  CHECK(calibatt_build_plan(row_ptr, HEADS, NB, NULL, work, &n_work) == CALIBATT_OK);

  void *dq, *dk, *dv, *do_, *drp, *dci, *dw;
  CHECK(cudaMalloc(&dq, elems * 2) == cudaSuccess && cudaMalloc(&dk, elems * 2) == cudaSuccess);
  CHECK(cudaMalloc(&dv, elems * 2) == cudaSuccess && cudaMalloc(&do_, elems * 2) == cudaSuccess);
  CHECK(cudaMalloc(&drp, sizeof row_ptr) == cudaSuccess && cudaMalloc(&dci, sizeof col_idx) == cudaSuccess);
  CHECK(cudaMalloc(&dw, sizeof work) == cudaSuccess);
  CHECK(cudaMemcpy(dq, q, elems * 2, cudaMemcpyHostToDevice) == cudaSuccess);
  CHECK(cudaMemcpy(dk, k, elems * 2, cudaMemcpyHostToDevice) == cudaSuccess);
  CHECK(cudaMemcpy(dv, v, elems * 2, cudaMemcpyHostToDevice) == cudaSuccess);
  CHECK(cudaMemcpy(drp, row_ptr, sizeof row_ptr, cudaMemcpyHostToDevice) == cudaSuccess);
  CHECK(cudaMemcpy(dci, col_idx, sizeof col_idx, cudaMemcpyHostToDevice) == cudaSuccess);
  CHECK(cudaMemcpy(dw, work, sizeof work, cudaMemcpyHostToDevice) == cudaSuccess);

  const float scale = 1.0f / sqrtf((float)D);
  CHECK(calibatt_sparse_attn_fwd(dq, dk, dv, HEADS, N, D, scale, drp, dci, row_ptr[HEADS * NB], dw, n_work, do_,
                                 NULL, NULL) == CALIBATT_OK);
  CHECK(calibatt_get_status(NULL) == CALIBATT_OK);
  CHECK(cudaMemcpy(o, do_, elems * 2, cudaMemcpyDeviceToHost) == cudaSuccess);

  /* dense softmax attention in double, every row */
  double* p = malloc(N * sizeof(double));
  double max_ref = 0.0, max_err = 0.0;
  for (int h = 0; h < HEADS; ++h)
    for (int i = 0; i < N; ++i) {
      const uint16_t* qi = q + ((size_t)h * N + i) * D;
      double m = -INFINITY, l = 0.0;
      for (int j = 0; j < N; ++j) {
        const uint16_t* kj = k + ((size_t)h * N + j) * D;
        double dot = 0.0;
        for (int c = 0; c < D; ++c) dot += from_bf16(qi[c]) * from_bf16(kj[c]);
        p[j] = dot * (double)scale;
        if (p[j] > m) m = p[j];
      }
      for (int j = 0; j < N; ++j) {
        p[j] = exp(p[j] - m);
        l += p[j];
      }
      for (int c = 0; c < D; ++c) {
        double acc = 0.0;
        for (int j = 0; j < N; ++j) acc += p[j] * from_bf16(v[((size_t)h * N + j) * D + c]);
        acc /= l;
        const double got = from_bf16(o[((size_t)h * N + i) * D + c]);
        if (fabs(acc) > max_ref) max_ref = fabs(acc);
        if (fabs(got - acc) > max_err) max_err = fabs(got - acc);
      }
    }
  printf("max |o - ref| %.3g, max |ref| %.3g\n", max_err, max_ref);
  CHECK(max_err <= 1e-2 * max_ref + 1e-3);
  cudaFree(dq);
  cudaFree(dk);
  cudaFree(dv);
  cudaFree(do_);
  cudaFree(drp);
  cudaFree(dci);
  cudaFree(dw);
  free(p);
  free(q);
  free(k);
  free(v);
  free(o);
  printf("ok\n");
  return 0;
}
