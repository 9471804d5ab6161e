// Self-test of the bounded mbarrier wait used by the tcgen05 kernels: one
// thread waits on a barrier that nothing ever arrives on, so the wait must give
// up after its wall-clock limit, set DCU_ST_TIMEOUT in the status word and let
// the kernel finish (the context stays usable).  Failure detection is tested
// this way, without any fault, trap or hang.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcu {
namespace {

__global__ void k_wait_timeout_probe(int32_t *status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 of a fresh barrier never completes: nobody arrives
    if (wait_bounded(smem_u32(&bar), 0u, &abort_flag, status)) atomicOr(status, 1 << 30);  // must not happen
    if (!abort_flag) atomicOr(status, 1 << 29);  // the expiry must also raise the CTA's abort flag
  }
}

}  // namespace

cudaError_t launch_wait_timeout_probe(int32_t *status, cudaStream_t s) {
  k_wait_timeout_probe<<<1, 32, 0, s>>>(status);
  return cudaGetLastError();
}

}  // namespace dcu
