// tc_layout_check.cu -- host-only check of the tensor-core kernel's shape rule
// and shared-memory layout (no device needed: only host functions run).
// Prints one line per D (multiple of 4, 4..128): "D maxK nfb@256 nfb@1024 nfb@maxK",
// where maxK is the largest K <= 2048 that tc_shape_ok accepts (0 if none) and
// nfb@K is the number of F buffers the layout takes at that K (0 past maxK).
#include <stdio.h>

#include "tc_em.cuh"

int main() {
  using namespace scem;
  for (int D = 4; D <= 128; D += 4) {
    int maxk = 0;
    for (int K = 1; K <= 2048; K++)
      if (tc_shape_ok(D, K)) maxk = K;
    unsigned nfb[3];
    const int ks[3] = {256, 1024, maxk};
    for (int i = 0; i < 3; i++)
      nfb[i] = (ks[i] >= 1 && ks[i] <= maxk)
                   ? tc_smem_layout(D, tc_cluster(ks[i]), tc_nchunks(D)).nfb
                   : 0u;
    printf("%d %d %u %u %u\n", D, maxk, nfb[0], nfb[1], nfb[2]);
  }
  return 0;
}
