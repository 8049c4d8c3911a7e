// swa_selftest.cu -- swa_selftest_wait_timeout: a check of the failure path
// that every tensor-core kernel's waits share, without a GPU fault.
//
// Two blocks of two warps wait on mbarriers that nothing arrives at, through
// the two bounded waits the tensor-core kernels use: block 0 through
// mbar_wait_parked (a probe, then try_wait with a suspend hint), block 1
// through mbar_wait_spin (try_wait without the hint), each until the clock
// budget of about 2 s runs out.  In each block the first waiter to give up
// records kDevTimeoutOther in the device error word and raises the block's
// abort flag; the other sees the flag and leaves.  Both blocks then exit
// normally, so the context stays usable, and swa_get_device_error() reports
// SWA_ERR_DEVICE_TIMEOUT.
#include "swa_internal.cuh"
#include "tc_ptx.cuh"

namespace {

using namespace swa::tc;

__global__ void __launch_bounds__(64) selftest_wait_kernel(unsigned* err) {
  __shared__ uint64_t bars[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;
  const int w = threadIdx.x >> 5;
  // phase 0 of a barrier that expects one arrival never completes
  if (blockIdx.x == 0)
    mbar_wait_parked(&bars[w], 0, abort, err, swa::kDevTimeoutOther);
  else
    mbar_wait_spin(&bars[w], 0, abort, err, swa::kDevTimeoutOther);
  __syncthreads();
}

}  // namespace

extern "C" swa_status swa_selftest_wait_timeout(void* stream) {
  swa::api_begin_call();
  swa_status st;
  unsigned* err = swa::api_error_word(&st);
  if (!err) return st;
  selftest_wait_kernel<<<2, 64, 0, static_cast<cudaStream_t>(stream)>>>(err);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return swa::api_cuda_fail(e, "selftest_wait_kernel");
  swa::api_end_call(1);
  return SWA_OK;
}
