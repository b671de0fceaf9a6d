// Self-test of the library's failure reporting: a bounded device wait that
// runs out must end the kernel normally and surface as CG_ERR_TIMEOUT.
//
// The kernel initializes an mbarrier that nothing ever arrives on and waits on
// it with the same bounded wait every codec kernel uses (mbar_wait), with a
// short caller-chosen limit.  The wait gives up, ORs the timeout flag into the
// device status word and returns; the kernel then exits.  Nothing faults,
// traps or hangs, and the context stays usable.
#include "cg_kernels.cuh"

namespace cg {

__global__ void selftest_wait_kernel(unsigned long long limit_ns, unsigned int* status, unsigned int* result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // phase 0 never completes: no thread arrives and no copy is pending
  const bool done = mbar_wait(&bar, 0u, status, limit_ns);
  if (threadIdx.x == 0) *result = done ? 1u : 0u;
}

}  // namespace cg

extern "C" cg_status cg_selftest_wait_timeout(int64_t limit_ns, uint32_t* result_dev, void* stream) {
  if (limit_ns <= 0 || limit_ns > 2000000000LL || !result_dev) return CG_ERR_INVALID;
  unsigned int* status = cg::device_status_word();
  if (!status) return CG_ERR_CUDA;
  cg::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)limit_ns, status, result_dev);
  return cg::from_cuda(cudaGetLastError());
}
