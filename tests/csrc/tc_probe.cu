// tc_probe.cu -- test-only probe of the sm_100a building blocks used by the
// tensor-core EM kernel (128-byte-swizzled shared-memory operands written by
// threads and by TMA, tcgen05 MMA with K-major and MN-major operands, commit
// to an mbarrier, tensor-memory loads).  One CTA computes one small product
// whose exact value the test gets from torch.
//
// mode 0: D[128 x N]  = A[128 x 64] * B[N x 64]^T   A, B K-major; B via TMA; N in {16,64,128,256}
// mode 1: D[128 x 64] = At[128 x 128]^T * Bt[128 x 64]  both MN-major (K = 128 rows)
// mode 2: D[128 x 16] = At^T * ones                     A MN-major, B K-major ones
#include <cuda_bf16.h>
#include <stdint.h>
#include <string.h>

#include "sm100_prims.cuh"
#include "tma_host.h"

using namespace scem::sm100;

namespace {

constexpr uint64_t kWaitLimit = 1000000000ull;  // 1 s

struct ProbeArgs {
  int mode, N;
  const __nv_bfloat16* A;
  const __nv_bfloat16* B;
  float* out;
  unsigned int* status;
};

__global__ void __launch_bounds__(128) tc_probe_kernel(ProbeArgs a,
                                                       const __grid_constant__ CUtensorMap tmB) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;               // 32 KB
  uint8_t* sB = smem + 32768;       // 32 KB
  uint8_t* sOnes = smem + 65536;    // 4 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 69632);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 69632 + 64);
  const int tid = threadIdx.x, warp = tid >> 5;

  if (tid == 0) {
    mbar_init(&bars[0], 1);  // TMA
    mbar_init(&bars[1], 1);  // MMA done
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  // operands written by threads into the swizzled layout
  if (a.mode == 0) {
    for (int i = tid; i < 128 * 64; i += 128) {
      const int r = i / 64, c = i % 64;
      *reinterpret_cast<__nv_bfloat16*>(sA + sw128_offset(r, c)) = a.A[i];
    }
  } else {
    for (int i = tid; i < 128 * 128; i += 128) {
      const int k = i / 128, m = i % 128;
      *reinterpret_cast<__nv_bfloat16*>(sA + (m / 64) * 16384 + sw128_offset(k, m % 64)) = a.A[i];
    }
    if (a.mode == 1) {
      for (int i = tid; i < 128 * 64; i += 128) {
        const int k = i / 64, n = i % 64;
        *reinterpret_cast<__nv_bfloat16*>(sB + sw128_offset(k, n)) = a.B[i];
      }
    } else {
      for (int i = tid; i < 2048; i += 128)
        reinterpret_cast<__nv_bfloat16*>(sOnes)[i] = __float2bfloat16_rn(1.0f);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    bool ok = true;
    if (a.mode == 0) {
      mbar_arrive_expect_tx(&bars[0], (uint32_t)a.N * 128u);
      tma_load_2d(sB, &tmB, 0, 0, &bars[0]);
      ok = mbar_wait_bounded(&bars[0], 0, a.status, 1u, kWaitLimit);
    }
    if (ok) {
      if (a.mode == 0) {
        const uint32_t idesc = idesc_bf16_f32(128, a.N, false, false);
        for (int ks = 0; ks < 4; ks++) {
          const uint64_t ad = sw128_desc(smem_u32(sA) + 32u * ks, 16, 1024);
          const uint64_t bd = sw128_desc(smem_u32(sB) + 32u * ks, 16, 1024);
          mma_bf16(tmem, ad, bd, idesc, ks > 0);
        }
      } else if (a.mode == 1) {
        const uint32_t idesc = idesc_bf16_f32(128, 64, true, true);
        for (int ks = 0; ks < 8; ks++) {
          const uint64_t ad = sw128_desc(smem_u32(sA) + 2048u * ks, 16384, 1024);
          const uint64_t bd = sw128_desc(smem_u32(sB) + 2048u * ks, 16384, 1024);
          mma_bf16(tmem, ad, bd, idesc, ks > 0);
        }
      } else {
        const uint32_t idesc = idesc_bf16_f32(128, 16, true, false);
        for (int ks = 0; ks < 8; ks++) {
          const uint64_t ad = sw128_desc(smem_u32(sA) + 2048u * ks, 16384, 1024);
          const uint64_t bd = sw128_desc(smem_u32(sOnes), 16, 1024);
          mma_bf16(tmem, ad, bd, idesc, ks > 0);
        }
      }
      mma_commit(&bars[1]);
    } else {
      mbar_arrive(&bars[1]);  // nothing was issued: release the waiters
    }
  }
  __syncwarp();
  const bool done = mbar_wait_bounded(&bars[1], 0, a.status, 2u, kWaitLimit);
  tc_fence_after_sync();
  const int N = a.mode == 0 ? a.N : (a.mode == 1 ? 64 : 16);
  if (done) {
    const int row = warp * 32 + (tid & 31);
    for (int c0 = 0; c0 < N; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
      for (int j = 0; j < 32 && c0 + j < N; j++) a.out[row * N + c0 + j] = v[j];
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

extern "C" int tc_probe_run(int mode, int N, const void* A, const void* B, float* out,
                            unsigned int* status, void* stream) {
  if (mode < 0 || mode > 2) return 1;
  if (mode == 0 && !(N == 16 || N == 64 || N == 128 || N == 256)) return 1;
  CUtensorMap tm;
  memset(&tm, 0, sizeof(tm));
  if (mode == 0 && !scem::make_tmap_16b_sw128(&tm, B, 64, (uint64_t)N, 128, (uint32_t)N))
    return 2;
  const size_t smem = 69632 + 128 + 1024;
  if (cudaFuncSetAttribute(tc_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return 3;
  ProbeArgs a{mode, N, (const __nv_bfloat16*)A, (const __nv_bfloat16*)B, out, status};
  tc_probe_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(a, tm);
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}
