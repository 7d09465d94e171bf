// common.cuh -- workspace layout and small device helpers shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gmm.h"

namespace scem {

constexpr int kMaxTopM = 8;
constexpr int kMaxD = 1024;
constexpr int kMaxK = 65536;

// Every region of the workspace starts on a 256-byte boundary.
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Scratch of the initialisation at the start of the workspace (the step's own
// tables overwrite it; nothing in it scales with N):
//   status : uint32 device status word (GMM_DEVFLAG_* bits), sticky until read
//   rows   : K int64, the chosen row indices
//   part   : P x D fp64 partial column sums (P = SMs), then D fp64 means
struct InitLayout {
  size_t status, rows, part, total;
  int P;
};

inline InitLayout init_layout(int D, int K, int num_sms) {
  InitLayout L;
  size_t off = 0;
  L.status = off;
  off = align_up(off + 16, 256);
  L.rows = off;
  off = align_up(off + (size_t)K * 8, 256);
  L.P = num_sms;
  L.part = off;
  off = align_up(off + ((size_t)L.P + 1) * D * 8, 256);
  L.total = off;
  return L;
}

__device__ __forceinline__ float load_x(const float* X, size_t i) { return __ldg(X + i); }
__device__ __forceinline__ float load_x(const __nv_bfloat16* X, size_t i) {
  return __bfloat162float(X[i]);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace scem
