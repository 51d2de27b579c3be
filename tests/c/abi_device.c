/* The device path of the C ABI from plain C99 with the CUDA runtime (no Python, no
 * torch): append the step's K/V rows through a slot mapping, decode one-token
 * contexts, copy a block on write.  Closed forms decide the results: a context of
 * one token returns that token's V row exactly (its softmax weight is 1), and a
 * block copy reproduces the source block bit for bit.  Exit status 0 when every
 * check holds. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "pagedkv.h"

enum { S = 3, H = 2, D = 64, B = 16, NB = 8, MB = 2 };

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

static uint32_t state = 12345u;
static float next_value(void) {
  state = state * 1664525u + 1013904223u;
  return (float)((state >> 8) & 0xffffu) / 65536.0f - 0.5f;
}

static void* to_device(const void* host, size_t bytes) {
  void* p = NULL;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return NULL;
  if (host && cudaMemcpy(p, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
  return p;
}

int main(void) {
  if (cudaSetDevice(0) != cudaSuccess) {
    fprintf(stderr, "no CUDA device\n");
    return 2;
  }
  const size_t pool_elems = (size_t)NB * H * B * D;
  const size_t row_elems = (size_t)S * H * D;
  float* hk = malloc(pool_elems * sizeof(float));
  float* hv = malloc(pool_elems * sizeof(float));
  float* knew = malloc(row_elems * sizeof(float));
  float* vnew = malloc(row_elems * sizeof(float));
  float* q = malloc(row_elems * sizeof(float));
  float* out = malloc(row_elems * sizeof(float));
  if (!hk || !hv || !knew || !vnew || !q || !out) return 2;
  for (size_t i = 0; i < pool_elems; ++i) hk[i] = next_value(), hv[i] = next_value();
  for (size_t i = 0; i < row_elems; ++i) knew[i] = next_value(), vnew[i] = next_value(), q[i] = next_value();

  /* sequence s owns blocks 2s+1 and 2s+2; its only token is appended at slot (2s+1)*B */
  int32_t tables[S * MB], ctx[S];
  int64_t slots[S];
  for (int s = 0; s < S; ++s) {
    tables[s * MB] = 2 * s + 1;
    tables[s * MB + 1] = 2 * s + 2;
    ctx[s] = 1;
    slots[s] = (int64_t)(2 * s + 1) * B;
  }
  const int64_t pairs[2] = {1, 7}; /* copy block 1 (sequence 0's) into the free block 7 */

  void* dk = to_device(hk, pool_elems * sizeof(float));
  void* dv = to_device(hv, pool_elems * sizeof(float));
  void* dknew = to_device(knew, row_elems * sizeof(float));
  void* dvnew = to_device(vnew, row_elems * sizeof(float));
  void* dq = to_device(q, row_elems * sizeof(float));
  void* dtables = to_device(tables, sizeof(tables));
  void* dctx = to_device(ctx, sizeof(ctx));
  void* dslots = to_device(slots, sizeof(slots));
  void* dpairs = to_device(pairs, sizeof(pairs));
  void* dout = to_device(NULL, row_elems * sizeof(float));
  if (!dk || !dv || !dknew || !dvnew || !dq || !dtables || !dctx || !dslots || !dpairs || !dout) return 2;

  CHECK(kv_cache_append(dknew, dvnew, dk, dv, (const int64_t*)dslots, S, H, D, B, NB, PKV_F32, NULL) == PKV_OK);
  CHECK(paged_attn_decode(dq, dk, dv, (const int32_t*)dtables, (const int32_t*)dctx, S, H, D, B, MB, NB, PKV_F32,
                          0.125f, (float*)dout, 0, NULL, 0, NULL) == PKV_OK);
  CHECK(kv_block_copy(dk, dv, (const int64_t*)dpairs, 1, H, D, B, NB, PKV_F32, NULL) == PKV_OK);
  CHECK(cudaMemcpy(out, dout, row_elems * sizeof(float), cudaMemcpyDeviceToHost) == cudaSuccess);
  CHECK(cudaMemcpy(hk, dk, pool_elems * sizeof(float), cudaMemcpyDeviceToHost) == cudaSuccess);
  CHECK(cudaMemcpy(hv, dv, pool_elems * sizeof(float), cudaMemcpyDeviceToHost) == cudaSuccess);

  /* one-token contexts: out[s][h] is the appended V row, bit for bit */
  CHECK(memcmp(out, vnew, row_elems * sizeof(float)) == 0);
  /* the appended rows sit at offset 0 of block 2s+1 for every head */
  for (int s = 0; s < S; ++s)
    for (int h = 0; h < H; ++h) {
      const size_t at = (((size_t)(2 * s + 1) * H + h) * B) * D;
      CHECK(memcmp(hk + at, knew + ((size_t)s * H + h) * D, D * sizeof(float)) == 0);
      CHECK(memcmp(hv + at, vnew + ((size_t)s * H + h) * D, D * sizeof(float)) == 0);
    }
  /* copy-on-write: block 7 equals block 1 in both pools */
  const size_t block = (size_t)H * B * D;
  CHECK(memcmp(hk + 7 * block, hk + 1 * block, block * sizeof(float)) == 0);
  CHECK(memcmp(hv + 7 * block, hv + 1 * block, block * sizeof(float)) == 0);

  int reason = -1;
  CHECK(pkv_get_device_error(NULL, &reason) == PKV_OK && reason == PKV_DEV_OK);

  cudaFree(dk), cudaFree(dv), cudaFree(dknew), cudaFree(dvnew), cudaFree(dq);
  cudaFree(dtables), cudaFree(dctx), cudaFree(dslots), cudaFree(dpairs), cudaFree(dout);
  free(hk), free(hv), free(knew), free(vnew), free(q), free(out);
  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("C device path checks passed\n");
  return 0;
}
