/*
 * A plain C program that uses the library the way a C or C++ caller would:
 * device buffers from the CUDA runtime, the forward and the backward through the
 * C ABI of include/fa.h, status checks on every call.
 *
 *   c_abi_example IN OUT B H N d causal
 *
 * IN holds q, k, v, dO as bf16 bit patterns, [B, H, N, d] each, one after the
 * other; OUT receives o, dq, dk, dv (bf16, same shape) and lse (float, [B, H, N]).
 * The test that runs it compares OUT with the oracle on the same seeded inputs.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "fa.h"

#define CHECK_CUDA(x)                                                        \
  do {                                                                       \
    cudaError_t e_ = (x);                                                    \
    if (e_ != cudaSuccess) {                                                 \
      fprintf(stderr, "%s failed: %s\n", #x, cudaGetErrorString(e_));        \
      return 2;                                                              \
    }                                                                        \
  } while (0)
#define CHECK_FA(x)                                                          \
  do {                                                                       \
    fa_status s_ = (x);                                                      \
    if (s_ != FA_OK) {                                                       \
      fprintf(stderr, "%s failed: %s\n", #x, fa_status_string(s_));         \
      return 3;                                                              \
    }                                                                        \
  } while (0)

int main(int argc, char** argv) {
  if (argc != 8) {
    fprintf(stderr, "usage: %s IN OUT B H N d causal\n", argv[0]);
    return 1;
  }
  const int B = atoi(argv[3]), H = atoi(argv[4]), N = atoi(argv[5]), d = atoi(argv[6]), causal = atoi(argv[7]);
  const size_t n = (size_t)B * H * N * d, nbytes = n * 2, lbytes = (size_t)B * H * N * 4;
  const float scale = 1.0f / sqrtf((float)d);

  uint16_t* host = (uint16_t*)malloc(4 * nbytes);
  FILE* f = fopen(argv[1], "rb");
  if (!host || !f || fread(host, 1, 4 * nbytes, f) != 4 * nbytes) {
    fprintf(stderr, "cannot read %s\n", argv[1]);
    return 1;
  }
  fclose(f);

  void *q, *k, *v, *dout, *o, *dq, *dk, *dv, *ws;
  float* lse;
  CHECK_CUDA(cudaMalloc(&q, nbytes));
  CHECK_CUDA(cudaMalloc(&k, nbytes));
  CHECK_CUDA(cudaMalloc(&v, nbytes));
  CHECK_CUDA(cudaMalloc(&dout, nbytes));
  CHECK_CUDA(cudaMalloc(&o, nbytes));
  CHECK_CUDA(cudaMalloc(&dq, nbytes));
  CHECK_CUDA(cudaMalloc(&dk, nbytes));
  CHECK_CUDA(cudaMalloc(&dv, nbytes));
  CHECK_CUDA(cudaMalloc((void**)&lse, lbytes));
  const size_t ws_bytes = fa_bwd_workspace_size(B, H, N, d);
  CHECK_CUDA(cudaMalloc(&ws, ws_bytes));
  CHECK_CUDA(cudaMemcpy(q, host, nbytes, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(k, host + n, nbytes, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(v, host + 2 * n, nbytes, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dout, host + 3 * n, nbytes, cudaMemcpyHostToDevice));

  cudaStream_t stream;
  CHECK_CUDA(cudaStreamCreate(&stream));
  CHECK_FA(fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, (fa_stream_t)stream));
  CHECK_FA(fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, ws, ws_bytes, (fa_stream_t)stream));
  CHECK_CUDA(cudaStreamSynchronize(stream));
  CHECK_FA(fa_get_device_status((fa_stream_t)stream));

  uint16_t* out = (uint16_t*)malloc(4 * nbytes + lbytes);
  if (!out) return 1;
  CHECK_CUDA(cudaMemcpy(out, o, nbytes, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(out + n, dq, nbytes, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(out + 2 * n, dk, nbytes, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(out + 3 * n, dv, nbytes, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(out + 4 * n, lse, lbytes, cudaMemcpyDeviceToHost));
  f = fopen(argv[2], "wb");
  if (!f || fwrite(out, 1, 4 * nbytes + lbytes, f) != 4 * nbytes + lbytes) {
    fprintf(stderr, "cannot write %s\n", argv[2]);
    return 1;
  }
  fclose(f);
  cudaStreamDestroy(stream);
  cudaFree(q); cudaFree(k); cudaFree(v); cudaFree(dout); cudaFree(o);
  cudaFree(dq); cudaFree(dk); cudaFree(dv); cudaFree(lse); cudaFree(ws);
  free(host);
  free(out);
  printf("ok\n");
  return 0;
}
