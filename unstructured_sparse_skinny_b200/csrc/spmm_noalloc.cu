// Allocation-free form of the SpMM entry point.
//
// flashspmm_spmm_lscd needs a caller-provided device workspace for its split-K
// partial sums and arrival counters.  Some callers cannot obtain one on
// demand: plugins running inside a host engine that owns every byte of device
// memory and forbids allocation while it executes, or latency-critical paths
// where cudaMalloc's implicit device synchronisation is not acceptable.  This
// file gives them flashspmm_spmm_lscd_noalloc, which takes its scratch from a
// fixed-size array that the library itself places in device memory when it is
// loaded, so the call allocates nothing.
#include <cstdint>

#include "common.cuh"

namespace flashspmm {
namespace {

// Scratch shared by every flashspmm_spmm_lscd_noalloc call on a device.  Each
// GPU that loads the library holds its own copy until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FLASHSPMM_NOALLOC_SCRATCH_BYTES];

// In host code `g_noalloc_scratch` names a host-side stand-in, not device
// memory.  The device address is looked up with cudaGetSymbolAddress on the
// first call in each context (with that device current) and cached; a device
// reset makes a new context and so a new lookup.
void* noalloc_scratch_ptr() { return symbol_address_cached(1, &g_noalloc_scratch); }

}  // namespace
}  // namespace flashspmm

using namespace flashspmm;

extern "C" flashspmm_status flashspmm_spmm_lscd_noalloc(const flashspmm_tcsl* A, const void* B, void* C, int32_t M,
                                                        int32_t K, int32_t N, int32_t split_k, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SpmmPlan plan{};
  bool done = true;
  const flashspmm_status st = prepare_spmm(A, B, C, false, M, K, N, split_k, s, &plan, &done);
  if (st != FLASHSPMM_OK || done) return st;
  if (plan.workspace_bytes > static_cast<size_t>(FLASHSPMM_NOALLOC_SCRATCH_BYTES)) return FLASHSPMM_ERR_CAPACITY;
  void* scratch = nullptr;
  if (plan.workspace_bytes > 0) {
    scratch = noalloc_scratch_ptr();
    if (!scratch) return FLASHSPMM_ERR_CUDA;
  }
  // The array keeps whatever the last call left in it: clear the arrival
  // counters (which must start at zero) on the stream before the kernel,
  // unless the launcher clears them itself.  The partial sums are always
  // written before they are read.
  if (plan.counter_bytes && !plan.counters_cleared &&
      cudaMemsetAsync(static_cast<uint8_t*>(scratch) + plan.counter_offset, 0, plan.counter_bytes, s) != cudaSuccess)
    return FLASHSPMM_ERR_CUDA;
  return launch_spmm_lscd(A, B, C, false, M, K, N, plan, scratch, s);
}
