// Self-test of the device-side failure path, without a GPU fault: a kernel whose
// only thread waits on an mbarrier that nothing arrives on.  The wait is the same
// bounded helper every product kernel uses (mbar_wait_bounded), given a short limit;
// it gives up, records kSiteSelftest in the library's status word and the kernel
// returns normally, so the context stays usable and the host reads the failure
// through aqlm_check_device_status.
#include "aqlm_device.cuh"

namespace aqlm {
namespace {

__global__ void __launch_bounds__(32) selftest_wait_kernel(uint32_t* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0u, status, kSiteSelftest, timeout_ns);
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t timeout_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace aqlm
