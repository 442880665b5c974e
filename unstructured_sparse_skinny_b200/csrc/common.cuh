// Internal declarations shared by the library's translation units.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
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
// Largest piece table the SpMM copies into shared memory (pieces; one CTA each).
constexpr int kMaxTablePieces = 512;

struct SpmmPlan {
  int32_t TM, TK, U;       // format strips, K tiles, 128-row units
  int64_t T;               // steps = U * TK
  int32_t mode;            // 0: pieces over all steps; 1: split-K inside each unit
  bool table;              // mode 0 pieces come from the operand's word-balanced table
  int32_t split;           // mode 1: K-chunks per unit
  int32_t num_pieces;      // one CTA per piece
  int64_t partial_slots;   // fp32 [slot][N][128] blocks
  int64_t counters;        // int32 arrival counters in use when partials exist
  bool counters_cleared;   // counters sit after the partials and are cleared before the launch
  size_t partial_offset, partial_bytes, counter_offset, counter_bytes, workspace_bytes;
};

// `table`: the operand carries a word-balanced piece table for this plan
// (used in mode 0 when the plan has at most kMaxTablePieces pieces).
SpmmPlan make_spmm_plan(int32_t M, int32_t K, int32_t N, int32_t split_k, int num_sms, bool table = false);
int device_sm_count();
flashspmm_status launch_spmm_lscd(const flashspmm_tcsl* A, const void* B, void* C, bool c_f32, int32_t M,
                                  int32_t K, int32_t N, const SpmmPlan& plan, void* workspace, cudaStream_t s);
// Argument checks and plan of an SpMM call, shared by its entry points.  On
// return *done says whether the call is complete (an error, or a shape that
// needs no kernel: M or N zero, or K zero, whose zero C is written here).
flashspmm_status prepare_spmm(const flashspmm_tcsl* A, const void* B, void* C, bool c_f32, int32_t M, int32_t K,
                              int32_t N, int32_t split_k, cudaStream_t s, SpmmPlan* plan, bool* done);
// Most 128-row units the partition kernel handles (its unit prefix sums live
// in shared memory).
constexpr int64_t kMaxPartitionUnits = 16384;
cudaError_t launch_round_f16(const float* x, __half* y, int64_t n, cudaStream_t s);
cudaError_t launch_tcsl_partition(const flashspmm_tcsl* A, int32_t num_pieces, int64_t* bounds, cudaStream_t s);
// Host form of the partition rule (the same functions the device runs).
bool partition_host(const int32_t* off, int64_t ld, int32_t M, int32_t K, int32_t num_pieces, int64_t* bounds);

}  // namespace flashspmm
