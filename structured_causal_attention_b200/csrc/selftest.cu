// selftest.cu - exercises the bounded-wait failure path without a fault.
//
// Every mbarrier wait in the tensor-core kernels gives up after a bounded
// number of cycles, records HD_ERR_TIMEOUT in the device status word and lets
// the kernel return; a later kernel that finds HD_ERR_TIMEOUT recorded skips
// its work. This kernel makes one thread wait, through the same helper, on an
// mbarrier that nothing will ever arrive on, with a caller-chosen limit, so
// the path can be tested: the wait ends, the status reads HD_ERR_TIMEOUT and
// the context stays usable.
#include "hd_common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace hd {

namespace {

__global__ void wait_timeout_kernel(long long limit, int* status) {
  __shared__ __align__(8) uint64_t bar_mem;
  __shared__ int abort_flag;
  const uint32_t bar = smem_u32(&bar_mem);
  if (threadIdx.x == 0) {
    tc::mbar_init(bar, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 never completes: no thread arrives
    tc::mbar_wait(bar, 0, reinterpret_cast<volatile int*>(&abort_flag), status, limit);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout(long long limit_cycles, int* status, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_cycles, status);
  return cudaGetLastError();
}

}  // namespace hd
