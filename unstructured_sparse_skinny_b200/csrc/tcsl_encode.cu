// GPU Tiled-CSL encoder (Flash-LLM paper review, section 3, "sparse encoding
// format: Tiled-CSL"): the nonzeros of every tile are stored together as
// 32-bit [16-bit value | 16-bit in-tile index] words and TileOffsets[] locates
// each tile.  The pages describe the encoding as an offline step; here it runs
// as three HBM-bound kernels whose output is bit-identical to the format's
// definition (ascending loc inside a tile, lists padded to 16 bytes with the
// sentinel 0xFFFF0000, offsets in words):
//   1. count:    one warp per tile counts nonzero fp16 bit patterns;
//   2. scan:     one CTA turns counts into padded running offsets and sums nnz;
//   3. fill:     one warp per tile compacts the tile in loc order with a warp
//                prefix sum (no atomics, so positions are deterministic);
//   4. optional: the bank-balanced word order (v2), in place.
// A further kernel validates a given encoding (checked mode).
#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flashspmm {
namespace {

constexpr int kEncThreads = 256;
constexpr int kWarpsPerBlock = kEncThreads / 32;

__device__ __forceinline__ int nonzero_halves(uint32_t w) {
  return static_cast<int>((w & 0xFFFFu) != 0u) + static_cast<int>((w >> 16) != 0u);
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

struct TileGeom {
  int64_t row0, col0;  // tile origin in A
  int rows, cols;      // valid extent (ragged at the matrix edge)
  int chunks_per_row;  // cols / 8 (16-byte chunks)
};

__device__ __forceinline__ TileGeom tile_geom(int64_t t, int TK, int M, int K, int tile_m, int tile_k) {
  TileGeom g;
  const int64_t i = t / TK, j = t - (t / TK) * TK;
  g.row0 = i * tile_m;
  g.col0 = j * tile_k;
  g.rows = static_cast<int>(min64(tile_m, M - g.row0));
  g.cols = static_cast<int>(min64(tile_k, K - g.col0));
  g.chunks_per_row = g.cols >> 3;
  return g;
}

// Pass 1: true nonzero count of tile t -> tile_offsets[t + 1].
__global__ void __launch_bounds__(kEncThreads) tcsl_count_kernel(const uint4* __restrict__ A, int M, int K,
                                                                int tile_m, int tile_k, int TK,
                                                                int64_t num_tiles, int32_t* __restrict__ off) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kEncThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarpsPerBlock;
  const int64_t row_chunks = K >> 3;
  for (int64_t t = warp0; t < num_tiles; t += nwarps) {
    const TileGeom g = tile_geom(t, TK, M, K, tile_m, tile_k);
    const int nchunks = g.rows * g.chunks_per_row;
    const uint4* base = A + g.row0 * row_chunks + (g.col0 >> 3);
    int cnt = 0;
    for (int e = lane; e < nchunks; e += 32) {
      const int r = e / g.chunks_per_row, ch = e - r * g.chunks_per_row;
      const uint4 v = __ldg(base + r * row_chunks + ch);
      cnt += nonzero_halves(v.x) + nonzero_halves(v.y) + nonzero_halves(v.z) + nonzero_halves(v.w);
    }
    cnt = warp_sum(cnt);
    if (lane == 0) off[t + 1] = cnt;
  }
}

// Pass 2 (one CTA): tile_offsets[t + 1] <- sum_{t' <= t} roundup4(count_t'),
// tile_offsets[0] <- 0, *nnz <- sum count_t.
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) tcsl_scan_kernel(int32_t* __restrict__ off, int64_t num_tiles,
                                                                int64_t* __restrict__ nnz, int* status) {
  __shared__ int64_t s_pad[kScanThreads];
  __shared__ int64_t s_true[kScanThreads];
  const int tid = threadIdx.x;
  const int64_t chunk = (num_tiles + kScanThreads - 1) / kScanThreads;
  const int64_t b = min64(num_tiles, tid * chunk), e = min64(num_tiles, b + chunk);
  int64_t pad = 0, tru = 0;
  for (int64_t i = b; i < e; ++i) {
    const int32_t c = off[i + 1];
    tru += c;
    pad += (c + 3) & ~3;
  }
  s_pad[tid] = pad;
  s_true[tid] = tru;
  __syncthreads();
  for (int d = 1; d < kScanThreads; d <<= 1) {  // inclusive Hillis-Steele scan
    const int64_t x = tid >= d ? s_pad[tid - d] : 0;
    const int64_t y = tid >= d ? s_true[tid - d] : 0;
    __syncthreads();
    s_pad[tid] += x;
    s_true[tid] += y;
    __syncthreads();
  }
  const int64_t total = s_pad[kScanThreads - 1];
  if (tid == 0) {
    off[0] = 0;
    *nnz = s_true[kScanThreads - 1];
    if (total > INT32_MAX) record_status(status, FLASHSPMM_ERR_CAPACITY);
  }
  int64_t run = s_pad[tid] - pad;
  for (int64_t i = b; i < e; ++i) {
    const int32_t c = off[i + 1];
    run += (c + 3) & ~3;
    off[i + 1] = static_cast<int32_t>(min64(run, INT32_MAX));
  }
}

// Pass 3: words of tile t in ascending loc, then sentinel padding.
__global__ void __launch_bounds__(kEncThreads) tcsl_fill_kernel(const uint4* __restrict__ A, int M, int K,
                                                               int tile_m, int tile_k, int TK, int64_t num_tiles,
                                                               const int32_t* __restrict__ off,
                                                               uint32_t* __restrict__ words, int64_t capacity,
                                                               int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kEncThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarpsPerBlock;
  const int64_t row_chunks = K >> 3;
  for (int64_t t = warp0; t < num_tiles; t += nwarps) {
    const int64_t w0 = off[t], w1 = off[t + 1];
    if (w0 < 0 || w1 < w0 || w1 > capacity || (w0 & 3) || ((w1 - w0) & 3)) {
      if (lane == 0) record_status(status, FLASHSPMM_ERR_CAPACITY);
      continue;
    }
    const int room = static_cast<int>(w1 - w0);
    uint32_t* dst = words + w0;
    const TileGeom g = tile_geom(t, TK, M, K, tile_m, tile_k);
    const int nchunks = g.rows * g.chunks_per_row;
    const uint4* base = A + g.row0 * row_chunks + (g.col0 >> 3);
    int carry = 0;
    bool overflow = false;
    for (int e0 = 0; e0 < nchunks; e0 += 32) {
      const int e = e0 + lane;
      uint32_t h[4] = {0u, 0u, 0u, 0u};
      uint32_t loc0 = 0;
      if (e < nchunks) {
        const int r = e / g.chunks_per_row, ch = e - r * g.chunks_per_row;
        const uint4 v = __ldg(base + r * row_chunks + ch);
        h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w;
        loc0 = static_cast<uint32_t>(r * tile_k + ch * 8);
      }
      uint32_t mask = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t half = (h[k >> 1] >> ((k & 1) * 16)) & 0xFFFFu;
        mask |= (half != 0u ? 1u : 0u) << k;
      }
      const int cnt = __popc(mask);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = carry + incl - cnt;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (mask & (1u << k)) {
          const uint32_t half = (h[k >> 1] >> ((k & 1) * 16)) & 0xFFFFu;
          if (pos < room) dst[pos] = half | ((loc0 + k) << 16);
          else overflow = true;
          ++pos;
        }
      }
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    const int padded = (carry + 3) & ~3;
    if (padded != room) overflow = true;
    for (int q = carry + lane; q < min(padded, room); q += 32) dst[q] = kSentinel;
    if (__any_sync(0xFFFFFFFFu, overflow) && lane == 0) record_status(status, FLASHSPMM_ERR_CAPACITY);
  }
}

// Checked mode: one warp per tile verifies the offsets and the words.  A
// tile's real words must hold distinct in-range locations with nonzero value
// bits (in any order, so both the ascending and the bank-balanced word order
// pass), followed only by exact sentinels, fewer than four of them.
constexpr int kValWarps = 4;
constexpr int kValBitmapWords = 65536 / 32;  // one bit per location of the largest tile

__global__ void __launch_bounds__(kValWarps * 32) tcsl_validate_kernel(const int32_t* __restrict__ off,
                                                                      const uint32_t* __restrict__ words,
                                                                      int64_t nwords, int M, int K, int tile_m,
                                                                      int tile_k, int TK, int64_t num_tiles, int* status) {
  __shared__ uint32_t s_seen[kValWarps][kValBitmapWords];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* seen = s_seen[warp];
  const int64_t nw = static_cast<int64_t>(gridDim.x) * kValWarps;
  const int area = tile_m * tile_k;
  const int max_words = (area + 3) & ~3;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kValWarps + warp; t < num_tiles; t += nw) {
    const int64_t w0 = off[t], w1 = off[t + 1];
    bool bad = w0 < 0 || w1 < w0 || (w0 & 3) || (w1 & 3) || w1 > nwords || (w1 - w0) > max_words;
    if (t == 0 && w0 != 0) bad = true;
    if (t == num_tiles - 1 && w1 != nwords) bad = true;
    if (bad) {
      if (lane == 0) record_status(status, FLASHSPMM_ERR_CORRUPT_FORMAT);
      continue;
    }
    const TileGeom g = tile_geom(t, TK, M, K, tile_m, tile_k);
    for (int i = lane; i < (area + 31) / 32; i += 32) seen[i] = 0u;
    __syncwarp();
    bool seen_sentinel = false;  // a sentinel appeared in an earlier batch
    int nreal = 0;
    for (int64_t b0 = w0; b0 < w1; b0 += 32) {
      const int64_t idx = b0 + lane;
      const bool valid = idx < w1;
      const uint32_t w = valid ? words[idx] : kSentinel;
      const int loc = static_cast<int>(w >> 16);
      const bool sent = loc == 0xFFFF;
      bool lane_bad = false;
      if (valid && sent && w != kSentinel) lane_bad = true;
      if (valid && !sent) {
        const int r = loc / tile_k, c = loc - (loc / tile_k) * tile_k;
        if (loc >= area || r >= g.rows || c >= g.cols || (w & 0xFFFFu) == 0u) {
          lane_bad = true;
        } else {
          const uint32_t bit = 1u << (loc & 31);
          if (atomicOr(&seen[loc >> 5], bit) & bit) lane_bad = true;  // location stored twice
        }
      }
      const uint32_t real_mask = __ballot_sync(0xFFFFFFFFu, valid && !sent);
      const uint32_t sent_mask = __ballot_sync(0xFFFFFFFFu, valid && sent);
      if (seen_sentinel && real_mask) lane_bad = true;
      if (sent_mask) {
        const int first_sent = __ffs(sent_mask) - 1;
        if (real_mask >> first_sent) lane_bad = true;
      }
      seen_sentinel |= sent_mask != 0u;
      nreal += __popc(real_mask);
      if (__any_sync(0xFFFFFFFFu, lane_bad)) bad = true;
    }
    __syncwarp();
    if ((w1 - w0) - nreal >= 4) bad = true;
    if (bad && lane == 0) record_status(status, FLASHSPMM_ERR_CORRUPT_FORMAT);
  }
}

// Word order v2 (bank-balanced), 64 x 64 tiles, one warp per tile, in place
// on an ascending-loc encoding.  A tile's words are stored in the dense
// shared-memory tile at byte x = 2*loc with the 128-byte swizzle
// x ^ ((x >> 3) & 0x70), so a word's bank is bits 2-6 of that offset.  The
// real words (before the first sentinel) are placed window by window, a
// window being 32 consecutive positions from the tile start: at a window's
// start the banks are ranked by unplaced words (most first, ties to the lower
// bank), and the window takes the lowest-loc unplaced word of each bank in
// rank order, round after round, until it is full.  In round r the banks
// still holding more than r words are exactly the first k_r ranks, so bank b
// of rank q places its r-th word at position k_0 + ... + k_{r-1} + q.
constexpr int kReorderWarps = 2;
constexpr int kReorderListWords = 4096;  // longest tile (64 x 64 words)
constexpr int kBankCap = 128;            // locations per shared-memory bank in a 64 x 64 fp16 tile
constexpr int kLoadBatch = 4;            // 32-word loads in flight per lane

__device__ __forceinline__ uint32_t word_bank(uint32_t w) {
  const uint32_t x = (w >> 15) & 0x1FFEu;  // 2 * loc for loc < 4096
  return ((x ^ ((x >> 3) & 0x70u)) >> 2) & 31u;
}

__global__ void __launch_bounds__(kReorderWarps * 32)
    tcsl_reorder_banks_kernel(const int32_t* __restrict__ off, uint32_t* __restrict__ words, int64_t num_tiles,
                              int64_t nwords, int* status) {
  // A bank of the dense 64 x 64 fp16 tile holds 128 locations, so the tile's
  // words fit per-bank lists of kBankCap entries; a tile that overflows one
  // (duplicate locations) is corrupt.
  __shared__ uint32_t s_list[kReorderWarps][32 * kBankCap];
  __shared__ int s_fill[kReorderWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t* list = s_list[warp];
  int* fill = s_fill[warp];
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kReorderWarps;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kReorderWarps + warp; t < num_tiles; t += nwarps) {
    const int64_t b0 = off[t], e0 = off[t + 1];
    const int64_t len64 = e0 - b0;
    if (b0 < 0 || len64 < 0 || len64 > kReorderListWords || e0 > nwords || (b0 & 3) || (len64 & 3)) {
      if (lane == 0) record_status(status, FLASHSPMM_ERR_CORRUPT_FORMAT);
      continue;
    }
    const int len = static_cast<int>(len64);
    uint32_t* tw = words + b0;
    fill[lane] = 0;
    __syncwarp();
    // One pass, kLoadBatch x 32 words loaded at a time: the real words are
    // those before the first sentinel; each goes to the end of its bank's
    // list, in input (ascending loc) order.
    int n = len;
    bool corrupt = false, done = false;
    for (int i0 = 0; i0 < len && !done; i0 += 32 * kLoadBatch) {
      uint32_t w[kLoadBatch];
#pragma unroll
      for (int b = 0; b < kLoadBatch; ++b) {
        const int i = i0 + 32 * b + lane;
        w[b] = i < len ? tw[i] : kSentinel;
      }
#pragma unroll
      for (int b = 0; b < kLoadBatch; ++b) {
        if (done) break;
        const int j0 = i0 + 32 * b, i = j0 + lane;
        const uint32_t sent = __ballot_sync(0xFFFFFFFFu, i < len && w[b] == kSentinel);
        const int stop = sent ? j0 + __ffs(sent) - 1 : len;
        const bool real = i < len && i < stop;
        if (real && (w[b] >> 16) >= 4096u) corrupt = true;
        const uint32_t bank = real ? word_bank(w[b]) : 32u;
        const uint32_t same = __match_any_sync(0xFFFFFFFFu, bank);
        const int pos = (real ? fill[bank] : 0) + __popc(same & lt_mask);
        if (real) {
          if (pos < kBankCap) list[bank * kBankCap + pos] = w[b];
          else corrupt = true;
        }
        __syncwarp();
        // the highest lane of each bank group advances that bank's fill
        if (real && (same >> lane) == 1u) fill[bank] += __popc(same);
        __syncwarp();
        if (sent || j0 + 32 >= len) {
          n = stop;
          done = true;
        }
      }
    }
    if (__any_sync(0xFFFFFFFFu, corrupt)) {
      if (lane == 0) record_status(status, FLASHSPMM_ERR_CORRUPT_FORMAT);
      continue;
    }
    const int cnt = fill[lane];  // lane b: words of bank b
    const int start = lane * kBankCap;
    // windows
    int taken = 0;  // lane b: words of bank b placed so far
    for (int placed = 0; placed < n;) {
      const int room = min(32, n - placed);
      const int rem = cnt - taken;
      int rank = 0;  // banks with more unplaced words, or as many and a lower index
#pragma unroll
      for (int l = 0; l < 32; ++l) {
        const int rl = __shfl_sync(0xFFFFFFFFu, rem, l);
        rank += (rl > rem || (rl == rem && l < lane)) ? 1 : 0;
      }
      int s = 0, mine = 0;
      for (int r = 0; s < room; ++r) {
        const int k = __popc(__ballot_sync(0xFFFFFFFFu, rem > r));
        if (k == 0) break;  // cannot happen while the counts are consistent
        if (rem > r && s + rank < room) {
          tw[placed + s + rank] = list[start + taken + r];
          ++mine;
        }
        s += k;
      }
      taken += mine;
      placed += room;
    }
  }
}

int enc_grid(int64_t num_tiles) {
  const int64_t blocks = (num_tiles + kWarpsPerBlock - 1) / kWarpsPerBlock;
  return static_cast<int>(max64(1, min64(blocks, 148 * 64)));
}

}  // namespace

cudaError_t launch_tcsl_count(const void* A, int32_t M, int32_t K, int32_t tile_m, int32_t tile_k,
                              int32_t* tile_offsets, int64_t* nnz, cudaStream_t s) {
  const int TK = (K + tile_k - 1) / tile_k;
  const int64_t nt = static_cast<int64_t>((M + tile_m - 1) / tile_m) * TK;
  if (nt > 0) {
    tcsl_count_kernel<<<enc_grid(nt), kEncThreads, 0, s>>>(static_cast<const uint4*>(A), M, K, tile_m, tile_k,
                                                          TK, nt, tile_offsets);
    note_launch();
  }
  tcsl_scan_kernel<<<1, kScanThreads, 0, s>>>(tile_offsets, nt, nnz, device_status_ptr());
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_tcsl_fill(const void* A, int32_t M, int32_t K, int32_t tile_m, int32_t tile_k,
                             const int32_t* tile_offsets, uint32_t* words, int64_t capacity, cudaStream_t s) {
  const int TK = (K + tile_k - 1) / tile_k;
  const int64_t nt = static_cast<int64_t>((M + tile_m - 1) / tile_m) * TK;
  if (nt == 0) return cudaSuccess;
  tcsl_fill_kernel<<<enc_grid(nt), kEncThreads, 0, s>>>(static_cast<const uint4*>(A), M, K, tile_m, tile_k, TK,
                                                       nt, tile_offsets, words, capacity, device_status_ptr());
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_tcsl_reorder_banks(const int32_t* tile_offsets, uint32_t* words, int64_t num_tiles, int64_t nwords,
                                      cudaStream_t s) {
  if (num_tiles == 0) return cudaSuccess;
  const int64_t blocks = (num_tiles + kReorderWarps - 1) / kReorderWarps;
  const int grid = static_cast<int>(max64(1, min64(blocks, 148 * 32)));
  tcsl_reorder_banks_kernel<<<grid, kReorderWarps * 32, 0, s>>>(tile_offsets, words, num_tiles, nwords,
                                                                device_status_ptr());
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_tcsl_validate(const flashspmm_tcsl* A, cudaStream_t s) {
  const int TK = (A->K + A->tile_k - 1) / A->tile_k;
  const int64_t nt = static_cast<int64_t>((A->M + A->tile_m - 1) / A->tile_m) * TK;
  if (nt == 0) return cudaSuccess;
  const int grid = static_cast<int>(max64(1, min64((nt + kValWarps - 1) / kValWarps, 148 * 32)));
  tcsl_validate_kernel<<<grid, kValWarps * 32, 0, s>>>(A->tile_offsets, A->words, A->nwords, A->M, A->K, A->tile_m,
                                                       A->tile_k, TK, nt, device_status_ptr());
  note_launch();
  return cudaGetLastError();
}

}  // namespace flashspmm
