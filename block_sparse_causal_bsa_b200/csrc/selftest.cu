// bsa_selftest_wait: runs the library's bounded mbarrier wait (the one every
// tensor-core kernel uses) on a barrier that nothing will complete, so the
// timeout path can be exercised on a real GPU without faulting it.
//
// One CTA of 64 threads. Warp 0's lane 0 waits on barrier A; warp 1's lane 0
// waits on barrier B. In mode 0 neither barrier is ever arrived on: warp 0's
// wait gives up after the library's wait limit (one second of globaltimer),
// sets BSA_DEV_TIMEOUT in the device status word and the CTA-wide abort flag,
// and warp 1's wait then returns early through that flag -- the same path a
// stalled pipeline stage takes inside attend or decode. In mode 1 a thread
// arrives on both barriers first, so both waits complete and the status stays
// 0 (the control case). The kernel then returns normally either way: no trap,
// no assert, no unbounded spin, and the context stays usable.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace {

__global__ void __launch_bounds__(64) selftest_wait_kernel(int mode, int32_t* dev_status,
                                                         int32_t* out) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    bsa::tc::mbar_init(&bar[0], 1);
    bsa::tc::mbar_init(&bar[1], 1);
    abort_flag = 0;
    bsa::tc::fence_mbar_init();
  }
  __syncthreads();
  if (mode == 1 && threadIdx.x == 32) {
    bsa::tc::mbar_arrive(&bar[0]);
    bsa::tc::mbar_arrive(&bar[1]);
  }
  const int warp = threadIdx.x / 32;
  if ((threadIdx.x & 31) == 0) {
    const bool ok = bsa::tc::mbar_wait(&bar[warp], 0, &abort_flag, dev_status);
    out[warp] = ok ? 1 : 0;
  }
}

}  // namespace

extern "C" bsa_status bsa_selftest_wait(int mode, int32_t* dev_status, int32_t* completed,
                                        void* stream) {
  if ((mode != 0 && mode != 1) || !dev_status || !completed) {
    bsa::set_last_error("bsa_selftest_wait: mode must be 0 or 1 and both pointers non-null");
    return BSA_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), st);
  if (e == cudaSuccess) {
    selftest_wait_kernel<<<1, 64, 0, st>>>(mode, dev_status, completed);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    bsa::set_last_error("bsa_selftest_wait: %s", cudaGetErrorString(e));
    return BSA_ERR_CUDA;
  }
  return BSA_OK;
}
