/* The GPU path from plain C: device memory from the CUDA runtime, a pool
 * bound to it, the slot-mapped cache write and the decode through the C ABI.
 * Reads its inputs from argv[1] and writes the pool and the outputs to
 * argv[2] (raw little-endian arrays, layout in read_inputs).  Exits non-zero
 * on any failed call. */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "pagedkv.h"

#define CK(call)                                                                      \
  do {                                                                                \
    int rc_ = (call);                                                                 \
    if (rc_ != 0) {                                                                   \
      fprintf(stderr, "%s failed (%d): %s\n", #call, rc_, kv_last_error());          \
      return 1;                                                                       \
    }                                                                                 \
  } while (0)
#define CU(call)                                                                      \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess) {                                                          \
      fprintf(stderr, "%s failed: %s\n", #call, cudaGetErrorString(e_));              \
      return 1;                                                                       \
    }                                                                                 \
  } while (0)

static int read_all(FILE* f, void* p, size_t n) { return fread(p, 1, n, f) == n ? 0 : 1; }

static void* to_device(const void* h, size_t n) {
  void* d = NULL;
  if (cudaMalloc(&d, n ? n : 16) != cudaSuccess) return NULL;
  if (n && cudaMemcpy(d, h, n, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
  return d;
}

int main(int argc, char** argv) {
  if (argc != 3) return 2;
  FILE* f = fopen(argv[1], "rb");
  if (!f) return 2;
  /* header: num_blocks, block_size, kv_heads, head_dim, num_q_heads, batch, width, tokens (int32),
   * scale (float32); then bf16 K pool, V pool, q, k_new, v_new, int32 tables, int32 lens, int64 slots */
  int32_t h[8];
  float scale;
  if (read_all(f, h, sizeof h) || read_all(f, &scale, sizeof scale)) return 2;
  const int nb = h[0], bs = h[1], hkv = h[2], d = h[3], hq = h[4], b = h[5], w = h[6], t = h[7];
  const size_t pool_n = (size_t)nb * hkv * bs * d * 2, q_n = (size_t)b * hq * d * 2, new_n = (size_t)t * hkv * d * 2;
  const size_t tab_n = (size_t)b * w * 4, lens_n = (size_t)b * 4, slots_n = (size_t)t * 8;
  char* buf = (char*)malloc(2 * pool_n + q_n + 2 * new_n + tab_n + lens_n + slots_n);
  if (!buf || read_all(f, buf, 2 * pool_n + q_n + 2 * new_n + tab_n + lens_n + slots_n)) return 2;
  fclose(f);
  char* p = buf;
  void* k = to_device(p, pool_n); p += pool_n;
  void* v = to_device(p, pool_n); p += pool_n;
  void* q = to_device(p, q_n); p += q_n;
  void* kn = to_device(p, new_n); p += new_n;
  void* vn = to_device(p, new_n); p += new_n;
  const int32_t* tables_h = (const int32_t*)p;
  void* tables = to_device(p, tab_n); p += tab_n;
  const int32_t* lens_h = (const int32_t*)p;
  void* lens = to_device(p, lens_n); p += lens_n;
  void* slots = to_device(p, slots_n);
  if (!k || !v || !q || !kn || !vn || !tables || !lens || !slots) return 3;
  (void)tables_h;
  int max_ctx = 0;
  for (int i = 0; i < b; ++i) max_ctx = lens_h[i] > max_ctx ? lens_h[i] : max_ctx;

  kv_pool* pool = NULL;
  CK(kv_pool_create(bs, nb, hkv, d, KV_BF16, 1, &pool));
  CK(kv_pool_bind(pool, 0, k, v, NULL, NULL));
  cudaStream_t st;
  CU(cudaStreamCreate(&st));
  CK(paged_kv_write(pool, 0, kn, vn, KV_BF16, (const int64_t*)slots, t, NULL, NULL, st));
  const size_t ws_n = paged_attention_workspace_bytes(pool, b, hq, max_ctx);
  void* ws = NULL;
  CU(cudaMalloc(&ws, ws_n ? ws_n : 16));
  void* out = NULL;
  const size_t out_n = (size_t)b * hq * d * 4;
  CU(cudaMalloc(&out, out_n));
  CK(paged_attention_decode(pool, 0, q, KV_BF16, hq, (const int32_t*)tables, w, (const int32_t*)lens, b, max_ctx,
                            scale, out, KV_F32, ws, ws_n, NULL, st));
  CU(cudaStreamSynchronize(st));
  int err = 0;
  CK(kv_get_device_error(st, &err));
  if (err != KV_OK) {
    fprintf(stderr, "device error %d\n", err);
    return 4;
  }
  char* res = (char*)malloc(pool_n + out_n);
  CU(cudaMemcpy(res, k, pool_n, cudaMemcpyDeviceToHost));
  CU(cudaMemcpy(res + pool_n, out, out_n, cudaMemcpyDeviceToHost));
  FILE* g = fopen(argv[2], "wb");
  if (!g || fwrite(res, 1, pool_n + out_n, g) != pool_n + out_n) return 5;
  fclose(g);
  CK(kv_pool_destroy(pool));
  cudaFree(k); cudaFree(v); cudaFree(q); cudaFree(kn); cudaFree(vn); cudaFree(tables); cudaFree(lens);
  cudaFree(slots); cudaFree(ws); cudaFree(out);
  cudaStreamDestroy(st);
  free(buf);
  free(res);
  printf("ok\n");
  return 0;
}
