// Self-test of the bounded pipeline waits: a single thread waits on an mbarrier
// phase that nothing completes, through the same mbar_wait() the attention
// pipeline uses, and must give up after `timeout_ns`, record BSA_ERR_TIMEOUT in
// the status word and return -- the context stays usable.
#include "bsa_common.cuh"
#include "nvtx_range.cuh"

namespace bsa {
namespace {

__global__ void wait_selftest_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // phase 0 never completes: nobody arrives
    const bool ok = mbar_wait(smem_u32(&bar), 0, &abort_flag, status, timeout_ns);
    if (ok) set_status(status, BSA_ERR_INVALID_ARG);  // cannot happen: flag it loudly
  }
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_wait_selftest(int* device_status, unsigned long long timeout_ns, void* stream) {
  BSA_NVTX_RANGE("bsa_wait_selftest");
  using namespace bsa;
  if (!device_status || timeout_ns == 0 || timeout_ns > 10000000000ULL) return BSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(device_status, 0, sizeof(int), st);
  if (e != cudaSuccess) return record_cuda_error(e);
  wait_selftest_kernel<<<1, 32, 0, st>>>(device_status, timeout_ns);
  return check_launch();
}
