/*
 * A plain C99 client of libawqsearch.so: no Python, no torch. It reads one layer from a
 * binary file, searches it through three entry points of include/awq_search.h — the
 * device call (awq_search_ex), the asynchronous device call (awq_search_async +
 * awq_search_status) and the host-buffer call (awq_search_host) — and writes each
 * result to an output file, so a test can compare them with the Python binding and
 * with the CPU oracle.
 *
 *   awq_client IN OUT
 *
 * IN:  int64 M, K, N; int32 group, n_grid, dtype (0 bf16, 1 fp32); X (M x K), W (K x N).
 * OUT: three records, each: int32 status; scales [K] fp32; codes [K][N/8] int32;
 *      steps, zeros [K/group][N] fp16; losses [n_grid] fp32; best (the chosen index) int32.
 * Exit status 0 when every call returned AWQ_OK, 1 on a call error, 2 on I/O or CUDA
 * setup errors.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "awq_search.h"

static int read_all(FILE* f, void* p, size_t n) { return fread(p, 1, n, f) == n; }
static int write_all(FILE* f, const void* p, size_t n) { return fwrite(p, 1, n, f) == n; }

int main(int argc, char** argv) {
  if (argc != 3) {
    fprintf(stderr, "usage: %s IN OUT\n", argv[0]);
    return 2;
  }
  FILE* in = fopen(argv[1], "rb");
  if (!in) return 2;
  int64_t M, K, N;
  int32_t group, n_grid, dtype;
  if (!read_all(in, &M, 8) || !read_all(in, &K, 8) || !read_all(in, &N, 8) || !read_all(in, &group, 4) ||
      !read_all(in, &n_grid, 4) || !read_all(in, &dtype, 4))
    return 2;
  const size_t elem = dtype == AWQ_DTYPE_F32 ? 4 : 2;
  const size_t bx = (size_t)M * K * elem, bw = (size_t)K * N * elem;
  void* hX = malloc(bx);
  void* hW = malloc(bw);
  if (!hX || !hW || !read_all(in, hX, bx) || !read_all(in, hW, bw)) return 2;
  fclose(in);

  /* scales, codes, steps, zeros, losses, chosen index */
  const size_t nb[6] = {(size_t)K * 4, (size_t)K * (N / 8) * 4, (size_t)(K / group) * N * 2,
                        (size_t)(K / group) * N * 2, (size_t)n_grid * 4, 4};
  void *dX, *dW, *dout[6], *hout[6];
  if (cudaMalloc(&dX, bx) != cudaSuccess || cudaMalloc(&dW, bw) != cudaSuccess) return 2;
  for (int i = 0; i < 6; ++i) {
    if (cudaMalloc(&dout[i], nb[i]) != cudaSuccess) return 2;
    hout[i] = malloc(nb[i]);
    if (!hout[i]) return 2;
  }
  cudaStream_t stream;
  int32_t* status_word = NULL;
  if (cudaStreamCreate(&stream) != cudaSuccess || cudaMallocHost((void**)&status_word, 4) != cudaSuccess) return 2;
  if (cudaMemcpy(dX, hX, bx, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(dW, hW, bw, cudaMemcpyHostToDevice) != cudaSuccess)
    return 2;

  FILE* out = fopen(argv[2], "wb");
  if (!out) return 2;
  int failed = 0;
  for (int call = 0; call < 3; ++call) {
    int32_t st;
    if (call == 0) {
      st = awq_search_ex(dX, dW, dtype, M, K, N, group, n_grid, (float*)dout[0], (int32_t*)dout[1], dout[2], dout[3],
                         (float*)dout[4], (int32_t*)dout[5], NULL, 0, (awq_stream_t)stream);
    } else if (call == 1) {
      *status_word = -1;
      st = awq_search_async(dX, dW, dtype, M, K, N, group, n_grid, (float*)dout[0], (int32_t*)dout[1], dout[2],
                            dout[3], (float*)dout[4], (int32_t*)dout[5], status_word, (awq_stream_t)stream);
      if (st == AWQ_OK) {
        if (cudaStreamSynchronize(stream) != cudaSuccess) return 2;
        st = awq_search_status(*status_word);
      }
    } else {
      st = awq_search_host(hX, hW, dtype, M, K, N, group, n_grid, (float*)hout[0], (int32_t*)hout[1], hout[2],
                           hout[3], (float*)hout[4], (int32_t*)hout[5], (awq_stream_t)stream);
    }
    if (st != AWQ_OK) {
      fprintf(stderr, "call %d: %s: %s\n", call, awq_status_string(st), awq_last_error_message());
      failed = 1;
    }
    if (call < 2)
      for (int i = 0; i < 6; ++i)
        if (cudaMemcpy(hout[i], dout[i], nb[i], cudaMemcpyDeviceToHost) != cudaSuccess) return 2;
    if (!write_all(out, &st, 4)) return 2;
    for (int i = 0; i < 6; ++i)
      if (!write_all(out, hout[i], nb[i])) return 2;
  }
  fclose(out);
  for (int i = 0; i < 6; ++i) {
    cudaFree(dout[i]);
    free(hout[i]);
  }
  cudaFree(dX);
  cudaFree(dW);
  cudaFreeHost(status_word);
  cudaStreamDestroy(stream);
  free(hX);
  free(hW);
  return failed;
}
