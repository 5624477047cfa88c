/*
 * c_abi_layer.c -- one POEM prefill layer through the C ABI of libpoem (include/poem.h)
 * from plain C: CUDA runtime allocations and a stream, no PyTorch.  Used by the tests
 * to check the ABI without the Python binding.
 *
 * usage: c_abi_layer DIR N HQ HKV D B TAU
 *   reads  DIR/q.bin [N, HQ, D], DIR/k.bin and DIR/v.bin [N, HKV, D] (raw bf16)
 *   writes DIR/o.bin [N, HQ, D] (raw bf16), DIR/row_ptr.bin and DIR/col_idx.bin (int32)
 * Exit status 0 on success; otherwise prints the failing call and its status.
 */
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime.h>

#include "poem.h"

#define CHECK_CUDA(x)                                                                  \
  do {                                                                                 \
    cudaError_t e_ = (x);                                                              \
    if (e_ != cudaSuccess) {                                                           \
      fprintf(stderr, "%s failed: %s\n", #x, cudaGetErrorString(e_));                  \
      return 2;                                                                        \
    }                                                                                  \
  } while (0)

#define CHECK_POEM(x)                                                                  \
  do {                                                                                 \
    poem_status s_ = (x);                                                              \
    if (s_ != POEM_OK) {                                                               \
      fprintf(stderr, "%s failed: %s (%s)\n", #x, poem_status_string(s_), poem_last_error()); \
      return 3;                                                                        \
    }                                                                                  \
  } while (0)

static void* read_file(const char* dir, const char* name, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "rb");
  if (!f) return NULL;
  void* buf = malloc(bytes);
  size_t got = buf ? fread(buf, 1, bytes, f) : 0;
  fclose(f);
  if (got != bytes) {
    free(buf);
    return NULL;
  }
  return buf;
}

static int write_file(const char* dir, const char* name, const void* buf, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "wb");
  if (!f) return 0;
  size_t put = fwrite(buf, 1, bytes, f);
  fclose(f);
  return put == bytes;
}

int main(int argc, char** argv) {
  if (argc != 8) {
    fprintf(stderr, "usage: %s DIR N HQ HKV D B TAU\n", argv[0]);
    return 1;
  }
  const char* dir = argv[1];
  const int n = atoi(argv[2]), hq = atoi(argv[3]), hkv = atoi(argv[4]), d = atoi(argv[5]), b = atoi(argv[6]);
  const float tau = (float)atof(argv[7]);
  const int T = n / b;

  poem_shape shape = {0};
  shape.n_tokens = n;
  shape.n_q_heads = hq;
  shape.n_kv_heads = hkv;
  shape.head_dim = d;
  shape.block = b;
  shape.n_sample = 16;
  shape.softmax_scale = 0.f;
  shape.q_offset = 0;
  shape.q_stride_tok = (int64_t)hq * d;
  shape.q_stride_head = d;
  shape.kv_stride_tok = (int64_t)hkv * d;
  shape.kv_stride_head = d;
  shape.o_stride_tok = (int64_t)hq * d;
  shape.o_stride_head = d;

  size_t ws_score = 0, ws_select = 0, ws_fwd = 0;
  CHECK_POEM(poem_workspace_size(&shape, &ws_score, &ws_select, &ws_fwd));

  const size_t q_bytes = (size_t)n * hq * d * 2, kv_bytes = (size_t)n * hkv * d * 2;
  const size_t entries = (size_t)hq * T * (T + 1) / 2;
  void* hq_buf = read_file(dir, "q.bin", q_bytes);
  void* hk_buf = read_file(dir, "k.bin", kv_bytes);
  void* hv_buf = read_file(dir, "v.bin", kv_bytes);
  if (!hq_buf || !hk_buf || !hv_buf) {
    fprintf(stderr, "cannot read the inputs in %s\n", dir);
    return 1;
  }

  cudaStream_t stream;
  CHECK_CUDA(cudaStreamCreate(&stream));
  void *q, *k, *v, *o, *I_hat, *m_hat, *row_ptr, *col_idx, *order, *w_score, *w_select, *w_fwd;
  CHECK_CUDA(cudaMalloc(&q, q_bytes));
  CHECK_CUDA(cudaMalloc(&k, kv_bytes));
  CHECK_CUDA(cudaMalloc(&v, kv_bytes));
  CHECK_CUDA(cudaMalloc(&o, q_bytes));
  CHECK_CUDA(cudaMalloc(&I_hat, entries * 4));
  CHECK_CUDA(cudaMalloc(&m_hat, entries * 4));
  CHECK_CUDA(cudaMalloc(&row_ptr, ((size_t)hq * T + 1) * 4));
  CHECK_CUDA(cudaMalloc(&col_idx, entries * 4));
  CHECK_CUDA(cudaMalloc(&order, (size_t)hq * T * 4));
  CHECK_CUDA(cudaMalloc(&w_score, ws_score));
  CHECK_CUDA(cudaMalloc(&w_select, ws_select));
  CHECK_CUDA(cudaMalloc(&w_fwd, ws_fwd));
  /* workspaces start zeroed (the error word) */
  CHECK_CUDA(cudaMemsetAsync(w_score, 0, ws_score, stream));
  CHECK_CUDA(cudaMemsetAsync(w_select, 0, ws_select, stream));
  CHECK_CUDA(cudaMemsetAsync(w_fwd, 0, ws_fwd, stream));
  CHECK_CUDA(cudaMemcpyAsync(q, hq_buf, q_bytes, cudaMemcpyHostToDevice, stream));
  CHECK_CUDA(cudaMemcpyAsync(k, hk_buf, kv_bytes, cudaMemcpyHostToDevice, stream));
  CHECK_CUDA(cudaMemcpyAsync(v, hv_buf, kv_bytes, cudaMemcpyHostToDevice, stream));

  CHECK_POEM(poem_score(&shape, q, k, v, (float*)I_hat, (float*)m_hat, w_score, ws_score, stream));
  CHECK_POEM(poem_select(&shape, (const float*)I_hat, (const float*)m_hat, tau, (int32_t*)row_ptr,
                         (int32_t*)col_idx, (int64_t)entries, (int32_t*)order, w_select, ws_select, stream));
  CHECK_POEM(bsa_fwd(&shape, q, k, v, (const int32_t*)row_ptr, (const int32_t*)col_idx, (const int32_t*)order,
                     (poem_bf16*)o, NULL, w_fwd, ws_fwd, stream));
  CHECK_POEM(poem_check(stream, w_score));
  CHECK_POEM(poem_check(stream, w_select));
  CHECK_POEM(poem_check(stream, w_fwd));

  void* ho = malloc(q_bytes);
  int32_t* hrp = (int32_t*)malloc(((size_t)hq * T + 1) * 4);
  if (!ho || !hrp) return 1;
  CHECK_CUDA(cudaMemcpy(ho, o, q_bytes, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hrp, row_ptr, ((size_t)hq * T + 1) * 4, cudaMemcpyDeviceToHost));
  const size_t nnz = (size_t)hrp[(size_t)hq * T];
  int32_t* hci = (int32_t*)malloc(nnz * 4 + 4);
  if (!hci) return 1;
  CHECK_CUDA(cudaMemcpy(hci, col_idx, nnz * 4, cudaMemcpyDeviceToHost));
  if (!write_file(dir, "o.bin", ho, q_bytes) || !write_file(dir, "row_ptr.bin", hrp, ((size_t)hq * T + 1) * 4) ||
      !write_file(dir, "col_idx.bin", hci, nnz * 4)) {
    fprintf(stderr, "cannot write the outputs in %s\n", dir);
    return 1;
  }
  printf("ok: %zu of %zu blocks kept\n", nnz, entries);
  cudaFree(q); cudaFree(k); cudaFree(v); cudaFree(o); cudaFree(I_hat); cudaFree(m_hat);
  cudaFree(row_ptr); cudaFree(col_idx); cudaFree(order); cudaFree(w_score); cudaFree(w_select); cudaFree(w_fwd);
  cudaStreamDestroy(stream);
  free(hq_buf); free(hk_buf); free(hv_buf); free(ho); free(hrp); free(hci);
  return 0;
}
