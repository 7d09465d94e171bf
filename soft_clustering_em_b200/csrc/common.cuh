// common.cuh -- workspace layout and small device helpers shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gmm.h"

namespace scem {

// Row tile of the CUDA-core fused kernel and its component chunk.
constexpr int kSimtRows = 32;
constexpr int kSimtThreads = 256;
constexpr int kMaxTopM = 8;
constexpr int kMaxD = 1024;
constexpr int kMaxK = 65536;

// Every region of the workspace starts on a 256-byte boundary.
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Layout of the caller-owned workspace.  Nothing in it scales with N.
//   status : uint32 device status word (GMM_DEVFLAG_* bits), sticky until read
//   pmu    : D x K f32, the means transposed (dimension-major) for coalesced reads
//   piv    : D x K f32, 1 / var, transposed
//   plogc  : K f32, log pi_k - 1/2 sum_d log(2 pi var_kd)   (-inf for pi_k = 0)
//   scratch: K int64 (init row indices)
//   slots  : P per-CTA partial-statistic slots of slot_stride doubles each:
//            [ N_k (K) | A (D x K) | B (D x K) | LL (1) | pad ]
//            A_dk = sum r (x - mu_k)_d,  B_dk = sum r (x - mu_k)_d^2  (moments
//            about the means the step started from)
struct WsLayout {
  size_t status, pmu, piv, plogc, scratch, slots, total;
  int P;               // number of slots = CTAs of the fused kernel
  size_t slot_stride;  // doubles per slot
};

inline WsLayout ws_layout(int D, int K, int num_sms) {
  WsLayout L;
  const size_t KD = (size_t)K * D;
  size_t off = 0;
  L.status = off;
  off = align_up(off + 16, 256);
  L.pmu = off;
  off = align_up(off + KD * 4, 256);
  L.piv = off;
  off = align_up(off + KD * 4, 256);
  L.plogc = off;
  off = align_up(off + (size_t)K * 4, 256);
  L.scratch = off;
  off = align_up(off + (size_t)K * 8, 256);
  L.slot_stride = align_up((size_t)K * (2 * (size_t)D + 1) + 1, 32);
  // two CTAs per SM while a slot is small, one otherwise: bounds the workspace
  L.P = (L.slot_stride * 8 <= (1u << 20)) ? 2 * num_sms : num_sms;
  L.slots = off;
  off = align_up(off + (size_t)L.P * L.slot_stride * 8, 256);
  L.total = off;
  return L;
}

// The same layout with the number of slots cut down until the whole layout
// fits in cap bytes (P = 0 when not even one slot fits).
inline WsLayout ws_layout_capped(int D, int K, int num_sms, size_t cap) {
  WsLayout L = ws_layout(D, K, num_sms);
  const size_t fixed = L.slots;
  const size_t per = L.slot_stride * 8;
  size_t fit = cap > fixed ? (cap - fixed) / per : 0;
  if ((size_t)L.P > fit) L.P = (int)fit;
  L.total = align_up(fixed + (size_t)L.P * per, 256);
  return L;
}

// Pointers into one workspace, passed to kernels by value.
struct WsPtrs {
  unsigned int* status;
  float* pmu;
  float* piv;
  float* plogc;
  int64_t* scratch;
  double* slots;
  size_t slot_stride;
  int P;
};

inline WsPtrs ws_ptrs(void* ws, const WsLayout& L) {
  char* b = (char*)ws;
  WsPtrs p;
  p.status = (unsigned int*)(b + L.status);
  p.pmu = (float*)(b + L.pmu);
  p.piv = (float*)(b + L.piv);
  p.plogc = (float*)(b + L.plogc);
  p.scratch = (int64_t*)(b + L.scratch);
  p.slots = (double*)(b + L.slots);
  p.slot_stride = L.slot_stride;
  p.P = L.P;
  return p;
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
