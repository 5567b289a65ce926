// Self-test of the failure path of the bounded device-side waits: one CTA
// waits, through the same mbarrier wait the tcgen05 attention kernels use, on
// a barrier that nothing ever signals.  The wait gives up after its cycle
// budget, raises the CTA's abort word and records LH_ERR_TIMEOUT in the
// device status word; the kernel then returns normally, so the context stays
// usable and the host reads the status with lh_device_status.
#include <cuda_runtime.h>

#include "host.h"
#include "tc.cuh"

namespace lh {
namespace {

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(unsigned int* status) {
  __shared__ alignas(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = tc::smem_addr(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);  // one arrival completes phase 0; none ever comes
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) tc::mbar_wait(b, 0, &abort_flag, status);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(cudaStream_t st) {
  unsigned int* status = device_status_ptr();
  if (status == nullptr) return cudaErrorInvalidSymbol;
  wait_timeout_kernel<<<1, 32, 0, st>>>(status);
  return cudaGetLastError();
}

}  // namespace lh
