// Self-check of the bounded pipeline wait: one kernel waits, with the same bounded
// mbarrier wait the tensor-core kernels use, on a barrier that nothing arrives at.  The
// wait gives up after the given limit, the kernel raises the status word to
// LSA_ERR_TIMEOUT and returns, and the context stays usable.  A stuck pipeline thus ends
// as a status, not as a hang; the tests check exactly that.
#include "lsa_common.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

__global__ void wait_check_kernel(unsigned long long limit_ns, int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0, &abort_flag, limit_ns)) raise_status(status, LSA_ERR_TIMEOUT);
  __syncthreads();
}

}  // namespace

int launch_wait_check(unsigned long long limit_ns, int32_t* status, cudaStream_t s) {
  wait_check_kernel<<<1, 32, 0, s>>>(limit_ns, status);
  return check_launch("check_bounded_wait");
}

}  // namespace lsa
