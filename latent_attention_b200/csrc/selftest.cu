// Failure-detection self-test: a bounded mbarrier wait that nothing satisfies.
#include "sm100.cuh"

namespace mla {
namespace {

__global__ void wait_timeout_kernel(uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);    // expects one arrival that never comes
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) sm100::mbar_wait(&bar, 0, &abort_flag, status);
  __syncthreads();
}

}  // namespace
}  // namespace mla

extern "C" mla_status mla_selftest_wait_timeout(void* workspace, void* stream) {
  if (!workspace) return MLA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return MLA_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, 4, st) != cudaSuccess) return MLA_ERR_CUDA;
  mla::wait_timeout_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t*>(workspace));
  mla::count_launches();
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
