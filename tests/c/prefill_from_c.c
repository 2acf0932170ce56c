/*
 * A prefill through the C ABI from plain C, with device memory from the CUDA
 * runtime and no Python: reads Q, K, V (bf16, row-major [B, L, H, D]) from
 * files, runs jl_bifocal_prefill on the default stream, and writes O (bf16)
 * and LSE (fp32) to files.
 *
 * usage: prefill_from_c B L Hq Hkv D w0 w_pretrained base q.bin k.bin v.bin o.bin lse.bin
 * Exit status 0 on success; the failing step's number otherwise.
 */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>

#include "jl_api.h"

static int read_file(const char* path, void* dst, size_t bytes) {
  FILE* f = fopen(path, "rb");
  size_t n;
  if (!f) return 0;
  n = fread(dst, 1, bytes, f);
  fclose(f);
  return n == bytes;
}

static int write_file(const char* path, const void* src, size_t bytes) {
  FILE* f = fopen(path, "wb");
  size_t n;
  if (!f) return 0;
  n = fwrite(src, 1, bytes, f);
  fclose(f);
  return n == bytes;
}

int main(int argc, char** argv) {
  int B, L, Hq, Hkv, D, w0, W, st, dev_err = -1;
  double base;
  size_t nq, nkv, ws_bytes;
  void *hq, *hk, *hv, *ho, *hl;
  void *dq = NULL, *dk = NULL, *dv = NULL, *d_o = NULL, *dl = NULL, *dws = NULL, *derr = NULL;
  if (argc != 14) return 1;
  B = atoi(argv[1]);
  L = atoi(argv[2]);
  Hq = atoi(argv[3]);
  Hkv = atoi(argv[4]);
  D = atoi(argv[5]);
  w0 = atoi(argv[6]);
  W = atoi(argv[7]);
  base = atof(argv[8]);
  nq = (size_t)B * L * Hq * D * 2;
  nkv = (size_t)B * L * Hkv * D * 2;
  hq = malloc(nq);
  hk = malloc(nkv);
  hv = malloc(nkv);
  ho = malloc(nq);
  hl = malloc((size_t)B * Hq * L * 4);
  if (!hq || !hk || !hv || !ho || !hl) return 2;
  if (!read_file(argv[9], hq, nq) || !read_file(argv[10], hk, nkv) || !read_file(argv[11], hv, nkv)) return 3;
  ws_bytes = jl_prefill_workspace_bytes(B, L, Hq, Hkv, D);
  if (ws_bytes == 0) return 4;
  if (cudaMalloc(&dq, nq) != cudaSuccess || cudaMalloc(&dk, nkv) != cudaSuccess ||
      cudaMalloc(&dv, nkv) != cudaSuccess || cudaMalloc(&d_o, nq) != cudaSuccess ||
      cudaMalloc(&dl, (size_t)B * Hq * L * 4) != cudaSuccess || cudaMalloc(&dws, ws_bytes) != cudaSuccess ||
      cudaMalloc(&derr, sizeof(int)) != cudaSuccess)
    return 5;
  if (cudaMemcpy(dq, hq, nq, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(dk, hk, nkv, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(dv, hv, nkv, cudaMemcpyHostToDevice) != cudaSuccess || cudaMemset(derr, 0, sizeof(int)) != cudaSuccess)
    return 6;
  st = jl_bifocal_prefill(dq, dk, dv, d_o, (float*)dl, B, L, Hq, Hkv, D, w0, W, base, 0.f, JL_QSHIFT_SELF_EXTEND,
                          dws, ws_bytes, (int*)derr, NULL);
  if (st != JL_OK) {
    fprintf(stderr, "jl_bifocal_prefill: %s\n", jl_status_string(st));
    return 7;
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return 8;
  if (cudaMemcpy(&dev_err, derr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess || dev_err != 0) return 9;
  if (cudaMemcpy(ho, d_o, nq, cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(hl, dl, (size_t)B * Hq * L * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return 10;
  if (!write_file(argv[12], ho, nq) || !write_file(argv[13], hl, (size_t)B * Hq * L * 4)) return 11;
  cudaFree(dq);
  cudaFree(dk);
  cudaFree(dv);
  cudaFree(d_o);
  cudaFree(dl);
  cudaFree(dws);
  cudaFree(derr);
  free(hq);
  free(hk);
  free(hv);
  free(ho);
  free(hl);
  return 0;
}
