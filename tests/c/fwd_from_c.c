/* A forward through the C ABI from plain C: reads q, k, v (bf16, dense
 * [B, S, H, D]) from a file, runs fa_fwd on the GPU and writes O (bf16) and
 * the LSE (fp32 [B, H, S]) to another file.
 *   usage: fwd_from_c <in> <out> B Sq Sk Hq Hkv D causal */
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "fa_b200.h"

static int fail(const char *what) {
  fprintf(stderr, "%s\n", what);
  return 1;
}

int main(int argc, char **argv) {
  if (argc != 10) return fail("usage: fwd_from_c <in> <out> B Sq Sk Hq Hkv D causal");
  const int B = atoi(argv[3]), Sq = atoi(argv[4]), Sk = atoi(argv[5]), Hq = atoi(argv[6]),
            Hkv = atoi(argv[7]), D = atoi(argv[8]), causal = atoi(argv[9]);
  const size_t nq = (size_t)B * Sq * Hq * D, nk = (size_t)B * Sk * Hkv * D;
  const size_t nl = (size_t)B * Hq * Sq;
  unsigned short *h_in = malloc((nq + 2 * nk) * 2), *h_o = malloc(nq * 2);
  float *h_l = malloc(nl * 4);
  if (!h_in || !h_o || !h_l) return fail("host allocation failed");
  FILE *f = fopen(argv[1], "rb");
  if (!f || fread(h_in, 2, nq + 2 * nk, f) != nq + 2 * nk) return fail("reading the inputs failed");
  fclose(f);

  void *q, *k, *v, *o;
  float *lse;
  if (cudaMalloc(&q, nq * 2) || cudaMalloc(&k, nk * 2) || cudaMalloc(&v, nk * 2) ||
      cudaMalloc(&o, nq * 2) || cudaMalloc((void **)&lse, nl * 4))
    return fail("cudaMalloc failed");
  cudaMemcpy(q, h_in, nq * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(k, h_in + nq, nk * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(v, h_in + nq + nk, nk * 2, cudaMemcpyHostToDevice);

  fa_status s = fa_fwd(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, D, FA_BF16, causal, 0.f, NULL,
                       NULL, 0, NULL);
  if (s != FA_OK) {
    fprintf(stderr, "fa_fwd: %s (%s)\n", fa_status_string(s), fa_last_error_message());
    return 1;
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return fail("the forward failed on the device");
  int code = 0;
  if (fa_check_device_error(&code, 1) != FA_OK || code != 0) return fail("device watchdog");
  cudaMemcpy(h_o, o, nq * 2, cudaMemcpyDeviceToHost);
  cudaMemcpy(h_l, lse, nl * 4, cudaMemcpyDeviceToHost);

  f = fopen(argv[2], "wb");
  if (!f || fwrite(h_o, 2, nq, f) != nq || fwrite(h_l, 4, nl, f) != nl)
    return fail("writing the outputs failed");
  fclose(f);
  cudaFree(q); cudaFree(k); cudaFree(v); cudaFree(o); cudaFree(lse);
  free(h_in); free(h_o); free(h_l);
  printf("ok\n");
  return 0;
}
