/* The serving loop from plain C: a pool in CUDA-runtime device memory, the
 * allocator and scheduler, and kv_serve_* over three buffer sets with host
 * staging (kv_serve_upload / kv_serve_readback).  Reads argv[1]:
 *   int32 num_blocks, block_size, kv_heads, head_dim, num_q_heads, steps,
 *         num_requests; float32 scale; int32 free order [num_blocks];
 *   per request int64 id, int32 prompt_len;
 *   per step int32 num_tokens, batch, then bf16 q [batch][num_q_heads][head_dim]
 *         and bf16 K, V rows [num_tokens][kv_heads][head_dim].
 * Writes argv[2]: per step fp32 out [batch][num_q_heads][head_dim], then the
 * bf16 K and V pools.  Exits non-zero on the first failure. */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pagedkv.h"

#define CK(call)                                                             \
  do {                                                                       \
    int rc_ = (call);                                                        \
    if (rc_ != 0) {                                                          \
      fprintf(stderr, "%s failed (%d): %s\n", #call, rc_, kv_last_error()); \
      return 1;                                                              \
    }                                                                        \
  } while (0)
#define CU(call)                                                             \
  do {                                                                       \
    cudaError_t e_ = (call);                                                 \
    if (e_ != cudaSuccess) {                                                 \
      fprintf(stderr, "%s failed: %s\n", #call, cudaGetErrorString(e_));     \
      return 1;                                                              \
    }                                                                        \
  } while (0)
#define RD(p, n)                                   \
  do {                                             \
    if (fread((p), 1, (n), f) != (size_t)(n)) {    \
      fprintf(stderr, "short input\n");            \
      return 2;                                    \
    }                                              \
  } while (0)

enum { SETS = 3, MAX_BATCH = 4, MAX_TOKENS = 256, MAX_WIDTH = 16, MAX_CONTEXT = 512 };

int main(int argc, char** argv) {
  if (argc != 3) return 2;
  FILE* f = fopen(argv[1], "rb");
  FILE* g = fopen(argv[2], "wb");
  if (!f || !g) return 2;
  int32_t h[7];
  float scale;
  RD(h, sizeof h);
  RD(&scale, sizeof scale);
  const int nb = h[0], bs = h[1], hkv = h[2], d = h[3], hq = h[4], steps = h[5], nreq = h[6];
  int32_t* order = (int32_t*)malloc(sizeof(int32_t) * nb);
  RD(order, sizeof(int32_t) * nb);

  const size_t pool_n = (size_t)nb * hkv * bs * d * 2;
  void *k = NULL, *v = NULL;
  CU(cudaMalloc(&k, pool_n));
  CU(cudaMalloc(&v, pool_n));
  CU(cudaMemset(k, 0, pool_n));
  CU(cudaMemset(v, 0, pool_n));
  kv_pool* pool = NULL;
  kv_alloc* a = NULL;
  kv_sched* s = NULL;
  CK(kv_pool_create(bs, nb, hkv, d, KV_BF16, 1, &pool));
  CK(kv_pool_bind(pool, 0, k, v, NULL, NULL));
  CK(kv_alloc_create(nb, bs, order, &a));
  CK(kv_sched_create(a, MAX_BATCH, -1, &s));
  for (int i = 0; i < nreq; ++i) {
    int64_t id;
    int32_t plen;
    RD(&id, sizeof id);
    RD(&plen, sizeof plen);
    CK(kv_sched_add_request(s, id, plen));
  }

  const size_t meta_n = kv_step_packed_bytes(MAX_BATCH, MAX_TOKENS, MAX_WIDTH, 0);
  void *hm[SETS], *dm[SETS], *din[SETS], *dout[SETS];
  const size_t in_n = ((size_t)MAX_BATCH * hq + 2 * (size_t)MAX_TOKENS * hkv) * d * 2;
  const size_t out_n = (size_t)MAX_BATCH * hq * d * 4;
  for (int i = 0; i < SETS; ++i) {
    CU(cudaMallocHost(&hm[i], meta_n));
    CU(cudaMalloc(&dm[i], meta_n));
    CU(cudaMalloc(&din[i], in_n));
    CU(cudaMalloc(&dout[i], out_n));
  }
  const size_t ws_n = kv_serve_workspace_bytes(pool, hq, MAX_BATCH, MAX_CONTEXT);
  void* ws = NULL;
  CU(cudaMalloc(&ws, ws_n ? ws_n : 16));
  void *hin = NULL, *hout = NULL;
  CU(cudaMallocHost(&hin, in_n));
  CU(cudaMallocHost(&hout, out_n));
  cudaStream_t up, main_s, rb;
  CU(cudaStreamCreate(&up));
  CU(cudaStreamCreate(&main_s));
  CU(cudaStreamCreate(&rb));
  kv_serve* sv = NULL;
  CK(kv_serve_create(pool, s, hq, KV_BF16, scale, KV_ORDER_BATCH, MAX_BATCH, MAX_TOKENS, MAX_WIDTH, NULL, 0, SETS,
                     hm, dm, meta_n, ws, ws_n ? ws_n : 16, &sv));

  for (int step = 0; step < steps; ++step) {
    int32_t tb[2];
    RD(tb, sizeof tb);
    const int t = tb[0], b = tb[1];
    int64_t running[MAX_BATCH];
    kv_step_layout lay;
    CK(kv_serve_schedule(sv, NULL, 0, up, running, &lay));
    if (lay.info.num_tokens != t || lay.info.batch != b || lay.buffer != step % SETS) {
      fprintf(stderr, "step %d: %d tokens, batch %d, set %d\n", step, lay.info.num_tokens, lay.info.batch,
              lay.buffer);
      return 3;
    }
    const size_t qn = (size_t)b * hq * d * 2, kn = (size_t)t * hkv * d * 2;
    RD(hin, qn + 2 * kn);
    const int set = lay.buffer;
    char* base = (char*)din[set];
    CK(kv_serve_upload(sv, base, hin, qn + 2 * kn));
    CK(kv_serve_launch(sv, 0, base, base + qn, base + qn + kn, NULL, NULL, dout[set], KV_F32, NULL, NULL, main_s));
    CK(kv_serve_readback(sv, hout, dout[set], (size_t)b * hq * d * 4, rb));
    CU(cudaStreamSynchronize(rb));
    CU(cudaStreamSynchronize(up));  /* the staging buffer is rewritten next step */
    if (fwrite(hout, 1, (size_t)b * hq * d * 4, g) != (size_t)b * hq * d * 4) return 5;
  }
  CU(cudaDeviceSynchronize());
  int err = 0;
  CK(kv_get_device_error(main_s, &err));
  if (err != KV_OK) {
    fprintf(stderr, "device error %d\n", err);
    return 4;
  }
  char* pools = (char*)malloc(2 * pool_n);
  CU(cudaMemcpy(pools, k, pool_n, cudaMemcpyDeviceToHost));
  CU(cudaMemcpy(pools + pool_n, v, pool_n, cudaMemcpyDeviceToHost));
  if (fwrite(pools, 1, 2 * pool_n, g) != 2 * pool_n) return 5;
  fclose(g);
  fclose(f);
  CK(kv_serve_destroy(sv));
  CK(kv_sched_destroy(s));
  CK(kv_alloc_destroy(a));
  CK(kv_pool_destroy(pool));
  for (int i = 0; i < SETS; ++i) {
    cudaFreeHost(hm[i]);
    cudaFree(dm[i]);
    cudaFree(din[i]);
    cudaFree(dout[i]);
  }
  cudaFreeHost(hin);
  cudaFreeHost(hout);
  cudaFree(ws);
  cudaFree(k);
  cudaFree(v);
  cudaStreamDestroy(up);
  cudaStreamDestroy(main_s);
  cudaStreamDestroy(rb);
  free(order);
  free(pools);
  printf("ok\n");
  return 0;
}
