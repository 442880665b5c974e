// Word-balanced work partition of the automatic SpMM plan.
//
// The SpMM cuts its step space (step q = u * TK + j: 128-row unit u, 64-wide
// K tile j) into one run of consecutive steps per CTA.  Even runs of steps
// suit matrices whose words are spread evenly; with rows of very different
// density (power-law rows, magnitude pruning) some runs hold far more words
// than others and the CTA holding the most sets the kernel's time.  The
// Flash-LLM review (section 5, "project structure") splits the work of one
// SpMM over thread blocks and merges partial sums in its Reduction kernel;
// this file chooses where those splits fall so that every CTA gets about the
// same cost: cost(step) = kStepCostWords + the words of its two strip tiles.
//
// The rule is written once, as host-and-device functions over the tile
// offsets, and run by one CTA on the device (flashspmm_tcsl_partition) or on
// the host (flashspmm_partition_host, for tests).
#include <vector>

#include "common.cuh"

namespace flashspmm {
namespace {

// A step's fixed cost in word equivalents: on B200 a 128 x 64 step costs
// about as much as expanding 1024 more words (fitted per-call times:
// 0.127 us per step at N <= 16 against 0.12 ns per word).
constexpr int64_t kStepCostWords = 1024;
constexpr int kPartThreads = 512;

struct OffsetsView {
  const int32_t* off;  // tile (i, j) starts at off[i * ld + j]
  int64_t ld;
  int64_t TM, TK, U, T;
};

// Words of strip s's tiles [0, j) (0 for the missing odd strip of a ragged last unit).
__host__ __device__ __forceinline__ int64_t strip_words(const OffsetsView& v, int64_t s, int64_t j) {
  if (s >= v.TM) return 0;
  return static_cast<int64_t>(v.off[s * v.ld + j]) - v.off[s * v.ld];
}

// Words of unit u (both strips, every K tile).
__host__ __device__ __forceinline__ int64_t unit_words(const OffsetsView& v, int64_t u) {
  return strip_words(v, 2 * u, v.TK) + strip_words(v, 2 * u + 1, v.TK);
}

// Cost of steps [0, q); unit_pre[u] = words of units [0, u), u = 0 .. U.
__host__ __device__ __forceinline__ int64_t cost_before(const OffsetsView& v, const int64_t* unit_pre, int64_t q) {
  const int64_t u = q / v.TK, j = q - (q / v.TK) * v.TK;
  int64_t w = unit_pre[u];
  if (j) w += strip_words(v, 2 * u, j) + strip_words(v, 2 * u + 1, j);
  return kStepCostWords * q + w;
}

// Smallest q in [0, T] with P * cost_before(q) >= pc * total: first over
// unit starts, then over the K tiles of the unit it falls in.
__host__ __device__ int64_t raw_bound(const OffsetsView& v, const int64_t* unit_pre, int64_t P, int64_t pc,
                                      int64_t total) {
  const int64_t target = pc * total;
  int64_t lo = 0, hi = v.U;
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (P * (kStepCostWords * mid * v.TK + unit_pre[mid]) >= target) hi = mid;
    else lo = mid + 1;
  }
  if (lo == 0) return 0;
  const int64_t base = (lo - 1) * v.TK;
  int64_t a = 1, b = v.TK;  // j = TK (the next unit's start) satisfies the test
  while (a < b) {
    const int64_t mid = (a + b) >> 1;
    if (P * cost_before(v, unit_pre, base + mid) >= target) b = mid;
    else a = mid + 1;
  }
  return base + a;
}

// Every piece keeps at least one step (P <= T): raise each bound above its
// predecessor, then lower each below its successor.
__host__ __device__ void fix_bounds(int64_t* b, int64_t P, int64_t T) {
  b[0] = 0;
  b[P] = T;
  for (int64_t pc = 1; pc < P; ++pc)
    if (b[pc] < b[pc - 1] + 1) b[pc] = b[pc - 1] + 1;
  for (int64_t pc = P - 1; pc >= 1; --pc)
    if (b[pc] > b[pc + 1] - 1) b[pc] = b[pc + 1] - 1;
}

OffsetsView make_view(const int32_t* off, int64_t ld, int32_t M, int32_t K) {
  OffsetsView v{};
  v.off = off;
  v.TM = (M + 63) / 64;
  v.TK = (K + 63) / 64;
  v.ld = ld > 0 ? ld : v.TK;
  v.U = (v.TM + 1) / 2;
  v.T = v.U * v.TK;
  return v;
}

// One CTA: unit word totals, their prefix sums (in shared memory), one
// bound per thread-strided piece, then the fix-up by one thread.
__global__ void __launch_bounds__(kPartThreads) tcsl_partition_kernel(OffsetsView v, int32_t P, int64_t* bounds) {
  extern __shared__ int64_t part_smem[];
  int64_t* unit_pre = part_smem;       // U + 1
  int64_t* b = part_smem + v.U + 1;    // P + 1
  __shared__ int64_t warp_tot[kPartThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // each thread sums a contiguous run of units
  const int64_t per = (v.U + kPartThreads - 1) / kPartThreads;
  const int64_t u0 = min64(v.U, tid * per), u1 = min64(v.U, u0 + per);
  int64_t run = 0;
  for (int64_t u = u0; u < u1; ++u) {
    const int64_t w = unit_words(v, u);
    unit_pre[u + 1] = w;
    run += w;
  }
  // exclusive scan of the runs across the block
  int64_t x = run;
  for (int d = 1; d < 32; d <<= 1) {
    const int64_t y = __shfl_up_sync(0xFFFFFFFFu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int64_t t = lane < kPartThreads / 32 ? warp_tot[lane] : 0;
    for (int d = 1; d < 32; d <<= 1) {
      const int64_t y = __shfl_up_sync(0xFFFFFFFFu, t, d);
      if (lane >= d) t += y;
    }
    if (lane < kPartThreads / 32) warp_tot[lane] = t;
  }
  __syncthreads();
  int64_t acc = x - run + (warp > 0 ? warp_tot[warp - 1] : 0);
  if (tid == 0) unit_pre[0] = 0;
  for (int64_t u = u0; u < u1; ++u) {
    acc += unit_pre[u + 1];
    unit_pre[u + 1] = acc;
  }
  __syncthreads();
  const int64_t total = kStepCostWords * v.T + unit_pre[v.U];
  for (int pc = tid; pc <= P; pc += kPartThreads)
    b[pc] = (pc == 0 || pc == P) ? 0 : raw_bound(v, unit_pre, P, pc, total);
  __syncthreads();
  if (tid == 0) fix_bounds(b, P, v.T);
  __syncthreads();
  for (int pc = tid; pc <= P; pc += kPartThreads) bounds[pc] = b[pc];
}

}  // namespace

cudaError_t launch_tcsl_partition(const flashspmm_tcsl* A, int32_t num_pieces, int64_t* bounds, cudaStream_t s) {
  const OffsetsView v = make_view(A->tile_offsets, A->offsets_ld, A->M, A->K);
  const size_t smem = static_cast<size_t>(v.U + 1 + num_pieces + 1) * sizeof(int64_t);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(tcsl_partition_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return cudaErrorInvalidValue;
  tcsl_partition_kernel<<<1, kPartThreads, smem, s>>>(v, num_pieces, bounds);
  note_launch();
  return cudaGetLastError();
}

bool partition_host(const int32_t* off, int64_t ld, int32_t M, int32_t K, int32_t num_pieces, int64_t* bounds) {
  const OffsetsView v = make_view(off, ld, M, K);
  if (v.ld < v.TK || num_pieces > v.T || v.U > kMaxPartitionUnits) return false;
  std::vector<int64_t> unit_pre(static_cast<size_t>(v.U) + 1, 0);
  for (int64_t u = 0; u < v.U; ++u) unit_pre[u + 1] = unit_pre[u] + unit_words(v, u);
  const int64_t total = kStepCostWords * v.T + unit_pre[v.U];
  for (int64_t pc = 1; pc < num_pieces; ++pc) bounds[pc] = raw_bound(v, unit_pre.data(), num_pieces, pc, total);
  fix_bounds(bounds, num_pieces, v.T);
  return true;
}

}  // namespace flashspmm
