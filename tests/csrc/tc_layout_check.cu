// tc_layout_check.cu -- host-only check of the tensor-core kernel's shape rule
// and shared-memory layout (no device needed: only host functions run).
// Prints one line per D (multiple of 4, 4..128):
//   "D maxK1 nfb@256 nfb@1024 nfb@maxK1 C@4096 G@4096"
// where maxK1 is the largest K <= 2048 that one component group (one cluster)
// serves, nfb@K the number of F buffers the layout takes at that K (0 past
// maxK1), and C@4096 / G@4096 the cluster size and group count chosen for
// K = 4096 on 148 SMs (0 0 if no tensor-core shape serves it).
//
// With the argument "streamed": one line per (D, K) with streamed features
// (D > 128):
//   "D K C G nchunks nfg NFG R smem feature_chunk_bytes rbuf_bytes"
// and with "maxk": one line per D, "D maxK" (the largest K with a plan).
#include <stdio.h>
#include <string.h>

#include "tc_em.cuh"

int main(int argc, char** argv) {
  using namespace scem;
  if (argc > 1 && strcmp(argv[1], "streamed") == 0) {
    const int Ds[] = {132, 260, 516, 768, 1024};
    const int Ks[] = {130, 1024, 4096};
    for (int D : Ds)
      for (int K : Ks) {
        int C = 0, G = 0;
        if (!tc_shape(D, K, 148, &C, &G)) {
          printf("%d %d 0 0 0 0 0 0 0 0 0\n", D, K);
          continue;
        }
        const TcLayout L = tc_layout(D, K, 148);
        const TcSmem S = tc_smem_layout(D, C, L.nchunks);
        printf("%d %d %d %d %d %d %d %lld %u %zu %zu\n", D, K, C, G, L.nchunks, L.nfg, L.NFG,
               (long long)L.R, S.total, L.flo - L.fhi, L.cand - L.rbuf);
      }
    return 0;
  }
  if (argc > 1 && strcmp(argv[1], "maxk") == 0) {
    for (int D = 4; D <= 1024; D += 4) {
      int lo = 1, hi = 70000;
      while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        int C, G;
        if (tc_shape(D, mid, 148, &C, &G)) lo = mid; else hi = mid - 1;
      }
      printf("%d %d\n", D, lo);
    }
    return 0;
  }
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
