/* Plain C use of the libkvq C ABI on the GPU, with no Python and no torch:
 * cudaMalloc'd buffers, then kvq_alloc_bits -> kvq_quantize_append ->
 * kvq_decode_attn for one sequence.
 *
 * Usage: kvq_device_abi <in> <out>. <in>: int32 n_kv, bits_k, bits_v, T,
 * n_q, v_seed, then bf16 keys [T][n_kv][128], bf16 values [T][n_kv][128],
 * bf16 queries [n_q][128]. <out>: int32 return codes of the three calls, the
 * status word and the final length, then fp32 outputs [n_q][128] and the
 * plan records [n_kv][kvq_plan_bytes()] as built on the device.
 * Compiled and run by tests/test_c_device_abi.py. */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "kvq.h"

#define CK(x)                                                            \
  do {                                                                   \
    cudaError_t e_ = (x);                                                \
    if (e_ != cudaSuccess) {                                             \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));           \
      return 2;                                                          \
    }                                                                    \
  } while (0)

static void* read_all(const char* path, size_t* n) {
  FILE* f = fopen(path, "rb");
  if (!f) return NULL;
  fseek(f, 0, SEEK_END);
  *n = (size_t)ftell(f);
  fseek(f, 0, SEEK_SET);
  void* p = malloc(*n);
  if (p && fread(p, 1, *n, f) != *n) {
    free(p);
    p = NULL;
  }
  fclose(f);
  return p;
}

int main(int argc, char** argv) {
  if (argc != 3) return 1;
  size_t n_in = 0;
  int32_t* hdr = (int32_t*)read_all(argv[1], &n_in);
  if (!hdr || n_in < 6 * sizeof(int32_t)) return 1;
  const int n_kv = hdr[0], bits_k = hdr[1], bits_v = hdr[2], T = hdr[3], n_q = hdr[4];
  kvq_cfg cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.head_dim = 128;
  cfg.n_kv_heads = n_kv;
  cfg.bits_k = bits_k;
  cfg.bits_v = bits_v;
  cfg.b_max = 8;
  cfg.alloc_mode = KVQ_ALLOC_GREEDY;
  cfg.v_seed = (uint64_t)hdr[5];
  const size_t kv_bytes = (size_t)T * n_kv * 128 * 2, q_bytes = (size_t)n_q * 128 * 2;
  if (n_in != 6 * sizeof(int32_t) + 2 * kv_bytes + q_bytes) return 1;
  const uint8_t* kh = (const uint8_t*)(hdr + 6);
  const uint8_t* vh = kh + kv_bytes;
  const uint8_t* qh = vh + kv_bytes;

  void *k, *v, *q, *plans, *cache, *ws_a, *ws_d, *plan_ptrs, *cache_ptrs;
  int32_t* len;
  uint32_t* status;
  float* out;
  const size_t plan_bytes = kvq_plan_bytes(), cache_bytes = kvq_cache_bytes(&cfg, T);
  const size_t wa = kvq_alloc_workspace_bytes(&cfg);
  const size_t wd = kvq_decode_workspace_bytes(&cfg, 1, n_q, T);
  CK(cudaMalloc(&k, kv_bytes));
  CK(cudaMalloc(&v, kv_bytes));
  CK(cudaMalloc(&q, q_bytes));
  CK(cudaMalloc(&plans, n_kv * plan_bytes));
  CK(cudaMalloc(&cache, cache_bytes));
  CK(cudaMalloc(&ws_a, wa));
  CK(cudaMalloc(&ws_d, wd));
  CK(cudaMalloc(&plan_ptrs, sizeof(void*)));
  CK(cudaMalloc(&cache_ptrs, sizeof(void*)));
  CK(cudaMalloc((void**)&len, sizeof(int32_t)));
  CK(cudaMalloc((void**)&status, sizeof(uint32_t)));
  CK(cudaMalloc((void**)&out, (size_t)n_q * 128 * sizeof(float)));
  CK(cudaMemcpy(k, kh, kv_bytes, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(v, vh, kv_bytes, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(q, qh, q_bytes, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(plan_ptrs, &plans, sizeof(void*), cudaMemcpyHostToDevice));
  CK(cudaMemcpy(cache_ptrs, &cache, sizeof(void*), cudaMemcpyHostToDevice));
  CK(cudaMemset(cache, 0, cache_bytes));
  CK(cudaMemset(ws_d, 0, wd));
  CK(cudaMemset(len, 0, sizeof(int32_t)));
  CK(cudaMemset(status, 0, sizeof(uint32_t)));

  int32_t res[5];
  res[0] = kvq_alloc_bits(&cfg, 0, k, KVQ_BF16, T, ws_a, wa, plans, NULL, NULL, status, 0);
  res[1] = kvq_quantize_append(&cfg, (const void* const*)plan_ptrs, k, v, KVQ_BF16, 1, T,
                               (void* const*)cache_ptrs, len, T, status, 0);
  res[2] = kvq_decode_attn(&cfg, (const void* const*)plan_ptrs, (const void* const*)cache_ptrs,
                           len, 1, T, q, KVQ_BF16, n_q, out, ws_d, wd, status, 0);
  CK(cudaDeviceSynchronize());
  float* oh = (float*)malloc((size_t)n_q * 128 * sizeof(float));
  uint8_t* ph = (uint8_t*)malloc(n_kv * plan_bytes);
  uint32_t st = 0;
  int32_t ln = 0;
  CK(cudaMemcpy(oh, out, (size_t)n_q * 128 * sizeof(float), cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(ph, plans, n_kv * plan_bytes, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(&st, status, sizeof st, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(&ln, len, sizeof ln, cudaMemcpyDeviceToHost));
  res[3] = (int32_t)st;
  res[4] = ln;
  FILE* f = fopen(argv[2], "wb");
  if (!f) return 1;
  fwrite(res, sizeof res, 1, f);
  fwrite(oh, sizeof(float), (size_t)n_q * 128, f);
  fwrite(ph, 1, n_kv * plan_bytes, f);
  fclose(f);
  printf("%s\n", res[0] || res[1] || res[2] ? kvq_last_error() : "ok");
  return 0;
}
