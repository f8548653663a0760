// Bounded-wait self-test: the waiting primitive of the tensor-core kernels,
// run on an mbarrier that nothing ever completes, so that the expiry path
// (status report, orderly exit) can be exercised without any fault.
#include "kernels.cuh"
#include "sm100.cuh"

namespace mla {
namespace {

__global__ void wait_selftest_kernel(uint64_t limit_ns, int *dev_status) {
  __shared__ __align__(8) uint64_t bar;
  using namespace sm100;
  if (threadIdx.x != 0) return;
  mbar_init(smem_u32(&bar), 1);
  fence_mbar_init();
  // Phase 0 needs one arrival; none comes, so the wait gives up after limit_ns.
  if (!mbar_wait(smem_u32(&bar), 0, limit_ns)) report(dev_status, MLA_ERR_TIMEOUT);
}

}  // namespace
}  // namespace mla

extern "C" MLA_API int mla_wait_selftest(long long limit_ns, int *dev_status, mla_stream_t stream) {
  if (limit_ns <= 0 || limit_ns > 10000000000ll || !dev_status) return MLA_ERR_INVALID_ARG;
  mla::wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((uint64_t)limit_ns, dev_status);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
