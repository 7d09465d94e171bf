// tc_layout_check.cu -- host-only check of the tensor-core kernel's shape rule
// and shared-memory layout (no device needed: only host functions run).
// Prints one line per D (multiple of 4, 4..128):
//   "D maxK1 nfb@256 nfb@1024 nfb@maxK1 C@4096 G@4096"
// where maxK1 is the largest K <= 2048 that one component group (one cluster)
// serves, nfb@K the number of F buffers the layout takes at that K (0 past
// maxK1), and C@4096 / G@4096 the cluster size and group count chosen for
// K = 4096 on 148 SMs (0 0 if no tensor-core shape serves it).
#include <stdio.h>

#include "tc_em.cuh"

int main() {
  using namespace scem;
  for (int D = 4; D <= 128; D += 4) {
    int maxk = 0;
    for (int K = 1; K <= 2048; K++) {
      int C = 0, G = 0;
      if (tc_shape(D, K, 148, &C, &G) && G == 1) maxk = K;
    }
    unsigned nfb[3];
    const int ks[3] = {256, 1024, maxk};
    for (int i = 0; i < 3; i++)
      nfb[i] = (ks[i] >= 1 && ks[i] <= maxk)
                   ? tc_smem_layout(D, tc_cluster(ks[i]), tc_nchunks(D)).nfb
                   : 0u;
    int C4 = 0, G4 = 0;
    if (!tc_shape(D, 4096, 148, &C4, &G4)) C4 = G4 = 0;
    printf("%d %d %u %u %u %d %d\n", D, maxk, nfb[0], nfb[1], nfb[2], C4, G4);
  }
  return 0;
}
