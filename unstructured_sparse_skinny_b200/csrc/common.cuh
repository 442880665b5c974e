// Internal declarations shared by the library's translation units.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/flashspmm.h"

namespace flashspmm {

constexpr uint32_t kSentinel = 0xFFFF0000u;

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }
__host__ __device__ __forceinline__ uint32_t minu32(uint32_t a, uint32_t b) { return a < b ? a : b; }

// Counts every kernel this library launches (flashspmm_launch_count()).
void note_launch();

// Device address of the library's status word on the current device.
int* device_status_ptr();

// Device address of a __device__ symbol in the current context (looked up
// once per context: a device reset creates a new context and a new lookup).
// `slot` names the symbol's cache (0: status word, 1: allocation-free scratch).
void* symbol_address_cached(int slot, const void* symbol);

// Kernel launchers (argument validation happens in the C-ABI layer).
cudaError_t launch_tcsl_count(const void* A, int32_t M, int32_t K, int32_t tile_m, int32_t tile_k,
                              int32_t* tile_offsets, int64_t* nnz, cudaStream_t s);
cudaError_t launch_tcsl_fill(const void* A, int32_t M, int32_t K, int32_t tile_m, int32_t tile_k,
                             const int32_t* tile_offsets, uint32_t* words, int64_t capacity, cudaStream_t s);
cudaError_t launch_tcsl_reorder_banks(const int32_t* tile_offsets, uint32_t* words, int64_t num_tiles, int64_t nwords,
                                      cudaStream_t s);
cudaError_t launch_tcsl_validate(const flashspmm_tcsl* A, cudaStream_t s);

// Work plan of one SpMM call: how the step space is cut into pieces and how
// much workspace the partial sums need.
// Workspace layout: [0, kCounterRegionBytes) arrival counters that are only
// ever incremented and reset to zero by the last arriver (so they are zero
// between calls, whatever the plans), then the fp32 partial sums, then (only
// for explicit split-K plans with more units than the counter region holds)
// per-unit counters that are cleared before each launch.
constexpr size_t kCounterRegionBytes = 4096;
constexpr int64_t kCounterRegionSlots = kCounterRegionBytes / sizeof(int32_t);

struct SpmmPlan {
  int32_t TM, TK, U;       // format strips, K tiles, 128-row units
  int64_t T;               // steps = U * TK
  int32_t mode;            // 0: even pieces over all steps; 1: split-K inside each unit
  int32_t split;           // mode 1: K-chunks per unit
  int32_t num_pieces;      // one CTA per piece
  int64_t partial_slots;   // fp32 [slot][N][128] blocks
  int64_t counters;        // int32 arrival counters in use when partials exist
  bool counters_cleared;   // counters sit after the partials and are cleared before the launch
  size_t partial_offset, partial_bytes, counter_offset, counter_bytes, workspace_bytes;
};

SpmmPlan make_spmm_plan(int32_t M, int32_t K, int32_t N, int32_t split_k, int num_sms);
int device_sm_count();
flashspmm_status launch_spmm_lscd(const flashspmm_tcsl* A, const void* B, void* C, int32_t M, int32_t K,
                                  int32_t N, const SpmmPlan& plan, void* workspace, cudaStream_t s);

}  // namespace flashspmm
