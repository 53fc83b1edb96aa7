// Self-test of the bounded waits every streaming kernel uses (mbar_wait in
// stream.cuh): a one-CTA kernel waits on an mbarrier that no copy and no
// thread will ever complete.  The wait gives up after kWaitCycles (about a
// second) and the kernel reports TQ_DEV_ERR_TIMEOUT in the caller's error
// word and returns, exactly the path a kernel takes when one of its copies
// never lands.  Nothing is in flight when it returns.

#include "stream.cuh"

namespace tqd {

__global__ void wait_timeout_kernel(uint32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival expected; none will come
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0)) report(err, TQ_DEV_ERR_TIMEOUT);
}

}  // namespace tqd

extern "C" tq_status tq_selftest_wait_timeout(uint32_t* error_word, void* stream) {
  if (!error_word) return tq::fail(TQ_EINVAL, "tq_selftest_wait_timeout: error_word is NULL");
  tqd::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(error_word);
  return tq::cuda_fail(cudaGetLastError(), "tq_selftest_wait_timeout launch");
}
