// Failure-detection self-test: a wait on an mbarrier that nothing completes. The bounded wait
// gives up after budget_ns, records DSA_ERR_TIMEOUT in the workspace header and the kernel
// returns normally, leaving the context usable.
#include "common.cuh"
#include "internal.h"

namespace dsa {

__global__ void selftest_wait_kernel(WsHeader* hdr, uint64_t budget_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{hdr, &abort_flag, budget_ns};
    (void)mbar_wait(&bar, 0, ctl, DETAIL_WAIT_SELFTEST);
  }
  __syncthreads();
}

dsa_status launch_selftest_wait(void* ws, uint64_t budget_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<WsHeader*>(ws), budget_ns);
  return cuda_status(cudaGetLastError());
}

}  // namespace dsa
