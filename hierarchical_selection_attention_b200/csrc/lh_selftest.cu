// Failure detection of the bounded waits.  Every mbarrier wait in the
// attention and GEMM kernels goes through sm100::mbar_wait, which gives up
// after sm100::kWaitCycles clock cycles, records LH_ERR_DEVICE_TIMEOUT in the
// device status word and lets the kernel unwind.  This kernel exercises that
// path on purpose without any fault: one warp waits on an mbarrier that
// nothing arrives at, so its first phase never completes; the wait runs out,
// the status is recorded, and the kernel returns with the context intact.
#include "lh_sm100.cuh"

namespace {

__global__ void __launch_bounds__(32) k_wait_timeout(int* status, int where) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  sm100::mbar_wait_w(&bar, 0, status, where);   // nothing arrives: phase 0 never completes
}

}  // namespace

cudaError_t lh_launch_wait_timeout_check(int* status, int where, cudaStream_t st) {
  k_wait_timeout<<<1, 32, 0, st>>>(status, where);
  return cudaGetLastError();
}
