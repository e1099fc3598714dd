// Failure-detection self test: the path a stalled pipeline takes, without a fault.
//
// One thread waits, through the same bounded mbarrier wait the attention kernels
// use, on a barrier that nothing ever arrives on.  After the wait limit (1 s of
// %globaltimer) it records DIT_ERR_TIMEOUT in the device error word and
// returns; the kernel ends normally and the context stays usable.
#include "dit_device.cuh"

namespace dit {

__global__ void selftest_wait_kernel(int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival; none comes
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, kErrTimeout);
}

cudaError_t launch_selftest_wait(int* err, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(err);
  return cudaGetLastError();
}

}  // namespace dit
