// Diagnostic kernel behind spark_selftest_wait: one warp allocates tensor
// memory, waits through the bounded-wait routine every kernel uses on an
// mbarrier phase that nothing completes, and takes the same exit a kernel
// takes when a wait expires: status word set, tensor memory freed, return.
// It lets a caller (and the test suite) see a device-side timeout surface as
// SPARK_ERR_TIMEOUT with the context still usable, without any fault.
#include "plan.h"
#include "tc_ptx.cuh"

namespace spark {

__global__ void __launch_bounds__(32, 1) selftest_wait_kernel(unsigned long long limit_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tmem_sh;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_sh)),
               "r"(32));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  tc::fence_before();
  __syncwarp();
  tc::fence_after();
  const uint32_t tmem = tmem_sh;
  bool ok = true;
  if (threadIdx.x == 0) ok = tc::mbar_wait_for(b, 0, status, limit_ns);   // nothing ever arrives
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  (void)ok;
  tc::fence_before();
  __syncwarp();
  tc::fence_after();
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(32));
}

cudaError_t launch_selftest_wait(unsigned long long limit_ns, int* status, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace spark
