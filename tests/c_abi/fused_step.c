/*
 * A decode step driven through the C ABI alone, with no Python: a small
 * paged cache is built on the host, copied into a pool the library
 * allocates, and one fused append + decode call (the benchmark's hot path)
 * runs on the GPU.  The FP64 CPU oracle (test infrastructure, linked only
 * here) checks the result: the pool bit for bit after the append, the
 * attention output within 2e-3.  Exit status 0 on success.
 *
 * Sequence lengths 5, 40 and 17 (after the append) over 16 pages in a
 * permuted order; scale 1/8; N(0,1)-like values from a fixed LCG rounded
 * to BF16.
 */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pkv.h"
#include "pkv_oracle.h"

enum { B = 3, MAXB = 3, PAGES = 16, PAGE_ELEMS = 2 * 8 * 16 * 64 };

static uint32_t lcg = 12345u;
static float next_uniform(void) {
  lcg = lcg * 1664525u + 1013904223u;
  return ((lcg >> 8) + 0.5f) / 16777216.0f;
}
/* roughly N(0, 1): sum of 12 uniforms minus 6 */
static float next_normal(void) {
  float s = 0.f;
  for (int i = 0; i < 12; ++i) s += next_uniform();
  return s - 6.f;
}
/* float -> BF16 bits, round to nearest even */
static uint16_t bf16(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

#define CHECK(call)                                                          \
  do {                                                                       \
    int s_ = (int)(call);                                                    \
    if (s_ != 0) {                                                           \
      fprintf(stderr, "%s failed: %d (%s)\n", #call, s_, pkv_last_error_message()); \
      return 1;                                                              \
    }                                                                        \
  } while (0)

int main(void) {
  const int32_t lens[B] = {5, 40, 17};
  int32_t bt[B * MAXB];
  const int32_t perm[PAGES] = {7, 2, 11, 0, 14, 5, 9, 3, 12, 1, 15, 6, 10, 4, 13, 8};
  int next = 0;
  for (int b = 0; b < B; ++b)
    for (int j = 0; j < MAXB; ++j) bt[b * MAXB + j] = j * 16 < lens[b] ? perm[next++] : -1;

  uint16_t* pool = (uint16_t*)malloc(sizeof(uint16_t) * PAGES * PAGE_ELEMS);
  for (int i = 0; i < PAGES * PAGE_ELEMS; ++i) pool[i] = bf16(next_normal());
  uint16_t q[B * 32 * 64], kn[B * 8 * 64], vn[B * 8 * 64];
  for (int i = 0; i < B * 32 * 64; ++i) q[i] = bf16(next_normal());
  for (int i = 0; i < B * 8 * 64; ++i) kn[i] = bf16(next_normal());
  for (int i = 0; i < B * 8 * 64; ++i) vn[i] = bf16(next_normal());

  pkv_pool* p = NULL;
  CHECK(pkv_pool_create(PAGES, 16, 8, 64, NULL, 0, &p));
  CHECK(cudaMemcpy(pkv_pool_data(p), pool, sizeof(uint16_t) * PAGES * PAGE_ELEMS,
                   cudaMemcpyHostToDevice));
  int32_t *d_bt, *d_len;
  uint16_t *d_q, *d_k, *d_v;
  float* d_out;
  void* d_ws;
  size_t ws = 0;
  CHECK(pkv_decode_workspace_bytes(p, B, &ws));
  CHECK(cudaMalloc((void**)&d_bt, sizeof bt));
  CHECK(cudaMalloc((void**)&d_len, sizeof lens));
  CHECK(cudaMalloc((void**)&d_q, sizeof q));
  CHECK(cudaMalloc((void**)&d_k, sizeof kn));
  CHECK(cudaMalloc((void**)&d_v, sizeof vn));
  CHECK(cudaMalloc((void**)&d_out, sizeof(float) * B * 32 * 64));
  CHECK(cudaMalloc(&d_ws, ws));
  CHECK(cudaMemcpy(d_bt, bt, sizeof bt, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(d_len, lens, sizeof lens, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(d_q, q, sizeof q, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(d_k, kn, sizeof kn, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(d_v, vn, sizeof vn, cudaMemcpyHostToDevice));

  CHECK(paged_attention_decode_append(d_q, d_k, d_v, p, d_bt, d_len, 0, 0.125f, d_out, 1, B,
                                      MAXB, d_ws, ws, NULL));
  int32_t dev_err = 0;
  CHECK(pkv_get_device_error(p, NULL, &dev_err));
  if (dev_err != 0) {
    fprintf(stderr, "device error %d\n", dev_err);
    return 1;
  }
  float out[B * 32 * 64];
  uint16_t* got_pool = (uint16_t*)malloc(sizeof(uint16_t) * PAGES * PAGE_ELEMS);
  CHECK(cudaMemcpy(out, d_out, sizeof out, cudaMemcpyDeviceToHost));
  CHECK(cudaMemcpy(got_pool, pkv_pool_data(p), sizeof(uint16_t) * PAGES * PAGE_ELEMS,
                   cudaMemcpyDeviceToHost));

  /* the oracle: append, then decode, in FP64 */
  CHECK(pkvo_append(pool, PAGES, bt, 1, B, MAXB, lens, kn, vn, 0));
  double want[B * 32 * 64];
  CHECK(pkvo_decode(q, pool, PAGES, bt, 1, B, MAXB, lens, 0, 0.125, want, NULL, 0, 1));
  if (memcmp(pool, got_pool, sizeof(uint16_t) * PAGES * PAGE_ELEMS) != 0) {
    fprintf(stderr, "pool after the append differs from the oracle\n");
    return 1;
  }
  double err = 0.0;
  for (int i = 0; i < B * 32 * 64; ++i) {
    const double e = fabs((double)out[i] - want[i]);
    if (!(e <= err)) err = e;   /* also catches NaN */
  }
  printf("c abi fused step: max abs error %.3g\n", err);
  CHECK(pkv_pool_destroy(p));
  return err <= 2e-3 ? 0 : 1;
}
