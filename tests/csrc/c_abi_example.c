/*
 * c_abi_example.c -- the library from plain C99: fit a small mixture with the
 * C ABI of include/gmm.h, with device memory from the CUDA runtime.
 *
 * Synthetic data: two well-separated blobs in DIM = 8 dimensions; NCOMP = 2 initial
 * means at rows 0 and N-1; 10 EM iterations through gmm_fit; prints the final
 * log-likelihood and weights.  With no CUDA device it prints the status of the
 * first call that needs one and exits 0, so the example also shows that the
 * library reports a missing device instead of failing in some other way.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "gmm.h"

#define NPTS 4096
#define DIM 8
#define NCOMP 2

static int check(gmm_status s, const char* what) {
  if (s != GMM_OK) {
    printf("%s: %s\n", what, gmm_status_string(s));
    return 1;
  }
  return 0;
}

int main(void) {
  gmm_problem p;
  size_t ws_bytes = 0;
  float* X = (float*)malloc(sizeof(float) * NPTS * DIM);
  int64_t rows[NCOMP] = {0, NPTS - 1};
  float w[NCOMP];
  double ll[10];
  void *dX = NULL, *dw = NULL, *dmu = NULL, *dvar = NULL, *dll = NULL, *ws = NULL;
  int n, d, rc = 0;

  p.N = NPTS;
  p.D = DIM;
  p.K = NCOMP;
  p.xdtype = GMM_F32;
  p.var_floor = 1e-6f;
  srand(7);
  for (n = 0; n < NPTS; n++)
    for (d = 0; d < DIM; d++)
      X[n * DIM + d] = (n < NPTS / 2 ? -3.0f : 3.0f) + (float)rand() / (float)RAND_MAX - 0.5f;

  if (check(gmm_workspace_size(&p, &ws_bytes), "gmm_workspace_size")) goto done;
  if (cudaMalloc(&dX, sizeof(float) * NPTS * DIM) != cudaSuccess ||
      cudaMalloc(&dw, sizeof(float) * NCOMP) != cudaSuccess ||
      cudaMalloc(&dmu, sizeof(float) * NCOMP * DIM) != cudaSuccess ||
      cudaMalloc(&dvar, sizeof(float) * NCOMP * DIM) != cudaSuccess ||
      cudaMalloc(&dll, sizeof(double) * 10) != cudaSuccess ||
      cudaMalloc(&ws, ws_bytes) != cudaSuccess || cudaMemset(ws, 0, ws_bytes) != cudaSuccess) {
    printf("cudaMalloc failed\n");
    rc = 1;
    goto done;
  }
  cudaMemcpy(dX, X, sizeof(float) * NPTS * DIM, cudaMemcpyHostToDevice);
  if (check(gmm_init_rows(&p, dX, rows, GMM_INIT_VAR_DATA, (float*)dw, (float*)dmu, (float*)dvar, ws,
                     ws_bytes, NULL), "gmm_init_rows") ||
      check(gmm_fit(&p, dX, 10, (float*)dw, (float*)dmu, (float*)dvar, (double*)dll, ws,
                    ws_bytes, NULL), "gmm_fit") ||
      check(gmm_device_status(ws, ws_bytes, NULL, NULL, 1), "gmm_device_status")) {
    rc = 1;
    goto done;
  }
  cudaMemcpy(ll, dll, sizeof(ll), cudaMemcpyDeviceToHost);
  cudaMemcpy(w, dw, sizeof(w), cudaMemcpyDeviceToHost);
  printf("LL(theta_9) = %.6f  w = %.4f %.4f\n", ll[9], w[0], w[1]);
done:
  cudaFree(dX);
  cudaFree(dw);
  cudaFree(dmu);
  cudaFree(dvar);
  cudaFree(dll);
  cudaFree(ws);
  free(X);
  return rc;
}
