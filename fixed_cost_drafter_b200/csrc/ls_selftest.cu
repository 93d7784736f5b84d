// Check of the failure detection on the device: one bounded wait on an mbarrier that
// nothing signals. The wait gives up after its poll limit, sets LS_DEVERR_WAIT_TIMEOUT in
// the state's error word and the kernel returns, which is what every wait of the path
// kernels does when a partner role never arrives. No fault, trap or endless loop.
#include "ls_common.cuh"

namespace ls {

__global__ void wait_timeout_kernel(int32_t* err, uint32_t polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait_bounded(&bar, 0, polls)) set_err(err, LS_DEVERR_WAIT_TIMEOUT);
}

cudaError_t launch_wait_timeout(const Dev& p, uint32_t polls, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(p.err, polls);
  return cudaGetLastError();
}

}  // namespace ls
