// A check of the bounded on-chip wait that every tensor-core kernel here uses around its
// mbarriers (TMA copies landed, MMAs committed, epilogue done): one CTA waits on an mbarrier
// phase with a caller-chosen poll limit, exactly as those kernels do.  If the phase is completed
// first (its own thread arrives) the wait succeeds and nothing is recorded; if nothing arrives,
// the wait gives up after the limit, records HILS_ERR_TIMEOUT in the status word and the kernel
// returns normally, so a wait that can never finish ends the kernel with a readable status
// instead of hanging the GPU.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
using namespace sm100;

namespace {

__global__ void __launch_bounds__(32, 1)
    wait_check_kernel(uint32_t polls, int complete, int32_t* __restrict__ status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (complete && threadIdx.x == 0) mbar_arrive(&bar);
  __syncwarp();
  // every lane polls, as in the kernels' epilogue warps (warp-uniform answer)
  if (!mbar_wait_warp(&bar, 0, polls) && threadIdx.x == 0) record_status(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_wait_check(uint32_t polls, int complete, int32_t* status, cudaStream_t st) {
  wait_check_kernel<<<1, 32, 0, st>>>(polls, complete, status);
  return cudaGetLastError();
}

}  // namespace hils
