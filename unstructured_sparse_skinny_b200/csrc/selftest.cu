// Diagnostic for the bounded in-kernel waits: one thread waits on an mbarrier
// that nothing ever completes.  When its budget runs out the wait records
// FLASHSPMM_ERR_TIMEOUT in the device status word and the kernel returns, so
// the failure path of every pipeline wait can be exercised without hanging or
// faulting the GPU.
#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flashspmm {
namespace {

__global__ void wait_timeout_kernel(uint64_t budget_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, budget_ns, status);  // no arrival ever comes
}

}  // namespace
}  // namespace flashspmm

using namespace flashspmm;

extern "C" flashspmm_status flashspmm_selftest_wait_timeout(uint32_t timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 1000000u) return FLASHSPMM_ERR_INVALID_ARG;
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || n <= 0) return FLASHSPMM_ERR_NO_DEVICE;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(timeout_us) * 1000u,
                                                                      device_status_ptr());
  note_launch();
  return cudaGetLastError() == cudaSuccess ? FLASHSPMM_OK : FLASHSPMM_ERR_CUDA;
}
