// m3_selftest.cu -- m3_selftest_wait: exercises the bounded-wait error path of the library.
//
// One CTA waits on an mbarrier that nothing arrives at.  The wait is bounded by %globaltimer,
// exactly like the waits of the scan and decode kernels; when the limit passes, the kernel
// records M3_ERR_TIMEOUT in the device status word and returns, so the context stays usable
// and m3_check() reports the timeout.  No GPU fault is involved.
#include "m3_common.cuh"

namespace m3 {
namespace {

__global__ void selftest_wait_kernel(int* status, unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(a));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  uint64_t t0, t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  uint32_t done = 0;
  while (true) {
    asm volatile(
        "{\n .reg .pred q;\n mbarrier.try_wait.parity.shared::cta.b64 q, [%1], 0;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(done)
        : "r"(a)
        : "memory");
    if (done) break;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > limit_ns) break;
  }
  if (!done && threadIdx.x == 0) set_status(status, M3_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_selftest_wait(int* status, unsigned long long limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace m3
