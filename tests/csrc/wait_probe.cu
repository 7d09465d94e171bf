// wait_probe.cu -- test-only probe of the bounded mbarrier wait that every
// spin of the tensor-core EM kernel uses (mbar_wait_bounded in
// sm100_prims.cuh).  One CTA of 64 threads allocates tensor memory, then
// thread 0 waits on phase 0 of an mbarrier with a budget of budget_ns.  With
// arrive = 0 nothing ever arrives, so the wait must give up after the budget,
// set the expire bit in *status and return false; with arrive = 1 thread 32
// arrives first and the wait must succeed.  Either way the CTA frees its
// tensor memory and returns: the kernel always ends.
#include <stdint.h>

#include "sm100_prims.cuh"

using namespace scem::sm100;

namespace {

__global__ void __launch_bounds__(64) wait_probe_kernel(uint64_t budget_ns, int arrive,
                                                        unsigned int* status,
                                                        unsigned long long* out) {
  __shared__ uint64_t bar;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (tid < 32) {
    tmem_alloc(&tslot, 32);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (tid == 32 && arrive) mbar_arrive(&bar);
  if (tid == 0) {
    const uint64_t t0 = globaltimer_ns();
    const bool done = mbar_wait_bounded(&bar, 0u, status, 0u, budget_ns);
    out[0] = done ? 1ull : 0ull;
    out[1] = globaltimer_ns() - t0;
  }
  tc_fence_before_sync();
  __syncthreads();
  if (tid < 32) {
    tc_fence_after_sync();
    tmem_dealloc(tslot, 32);
  }
}

}  // namespace

// Enqueues one probe launch on `stream`; returns the launch's error code.
extern "C" int wait_probe_run(unsigned long long budget_ns, int arrive, void* status, void* out,
                              void* stream) {
  wait_probe_kernel<<<1, 64, 0, (cudaStream_t)stream>>>(
      budget_ns, arrive, (unsigned int*)status, (unsigned long long*)out);
  return (int)cudaGetLastError();
}
