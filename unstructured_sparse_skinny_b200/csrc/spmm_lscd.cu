// LSCD SpMM for sm_100a: C = A x B with A in Tiled-CSL (64 x 64 tiles), B a
// skinny fp16 K x N matrix, fp32 accumulation in tensor memory, fp16 C.
//
// Method (Flash-LLM paper review, xllm-io.github.io): the weights are loaded
// in their sparse form to cut HBM bytes, expanded on chip into dense tiles and
// multiplied densely on the tensor cores (section 2, "solution overview";
// section 3, pipeline stages gmem2reg / rst_smem / extract / ld_dense /
// smem2tc / TC_compute, overlapped across iterations).  The A100 kernel on the
// page (register-staged extraction, ldmatrix + mma.sync, cp.async double
// buffering) is prior art; this kernel keeps the stages and replaces each
// mechanism with its sm_100a counterpart:
//
//   gmem2reg  -> warp 0 streams each step's word lists HBM -> a shared-memory
//                byte ring with cp.async.bulk (evict-first L2 policy), up to
//                the ring size in flight, gated by mbarriers;
//   ld_dense  -> warp 1 loads the 64 x N_MMA B slab of the step with a TMA
//                tensor copy in the 128-byte swizzled layout (rows >= N and
//                columns >= K are zero-filled by TMA);
//   rst_smem  -> 8 decompress warps zero a 128 x 64 dense A buffer with
//   + extract    16-byte stores, then scatter every word's value to its
//                swizzled position (UMMA K-major canonical layout);
//   smem2tc   -> gone: tcgen05.mma reads both operands from shared memory;
//   TC_compute-> warp 2 issues 4 x tcgen05.mma (M = 128, K = 16) per step into
//                a double-buffered fp32 accumulator in tensor memory;
//   epilogue  -> 4 warps read the accumulator with tcgen05.ld and write fp16 C
//                (or fp32 partial sums, see below).
//
// A "unit" is 128 rows of A (two 64-row format strips stacked on the MMA M
// side); a "step" is one 64-wide K tile of one unit.  The T = units x K-tiles
// steps are cut into contiguous pieces, one CTA each.  When a unit is shared
// by several pieces, every piece writes its fp32 partial sum to the workspace
// and the last piece to finish (atomic arrival counter) adds them in piece
// order and writes C: the split-K reduction of the page's Reduction kernel
// (section 5, "project structure"), fused and deterministic.
#include <cuda.h>
#include <cuda_fp16.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flashspmm {
namespace {

constexpr int kTile = 64;                         // format tile edge (rows and K)
constexpr int kUnitRows = 128;                    // MMA M
constexpr int kDenseBytes = kUnitRows * kTile * 2;  // 16 KB dense A buffer
constexpr int kMaxTileWords = kTile * kTile;      // 4096 words (already a multiple of 4)
constexpr int kThreads = 480;                     // 15 warps
constexpr int kWarpWords = 0, kWarpB = 1, kWarpMma = 2, kWarpEpi = 3, kWarpDec = 7;
constexpr int kEpiThreads = 128, kDecThreads = 256;
constexpr int kBarDec = 1, kBarEpi = 2;          // named barrier ids
constexpr int kMinStepsPerPiece = 4;

template <int N_MMA>
struct Cfg {
  static_assert(N_MMA == 16 || N_MMA == 32 || N_MMA == 64 || N_MMA == 128 || N_MMA == 256, "N bucket");
  static constexpr int kNumDense = N_MMA <= 64 ? 3 : 2;
  static constexpr int kNumB = N_MMA <= 64 ? 6 : (N_MMA == 128 ? 4 : 3);
  static constexpr int kBSlabBytes = N_MMA * kTile * 2;
  static constexpr int kRingBytes = N_MMA <= 32 ? 128 * 1024 : (N_MMA <= 128 ? 96 * 1024 : 64 * 1024);
  static constexpr int kRingWords = kRingBytes / 4;
  static constexpr int kNumSlots = 16;  // word-ring stages (metadata + barriers)
  static constexpr int kTmemCols = 2 * N_MMA < 32 ? 32 : 2 * N_MMA;
  static constexpr uint32_t kIdesc = umma_idesc_f16_f32(kUnitRows, N_MMA);
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int kOffDense = 0;
  static constexpr int kOffB = kOffDense + kNumDense * kDenseBytes;
  static constexpr int kOffRing = kOffB + kNumB * kBSlabBytes;
  static constexpr int kOffMeta = kOffRing + kRingBytes;
  static constexpr int kOffEnd = kOffMeta + kNumSlots * 16;
  static constexpr int kOffBars = kOffEnd + kNumSlots * 8;
  static constexpr int kNumBars = 2 * kNumSlots + 2 * kNumB + 2 * kNumDense + 4 + 1;
  static constexpr int kOffMisc = kOffBars + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kRingBytes >= 2 * kMaxTileWords * 4, "a step must fit the ring");
};

struct SpmmParams {
  const int32_t* tile_offsets;
  const uint32_t* words;
  int64_t nwords;
  __half* C;
  float* partials;    // [slot][N][128]
  int32_t* counters;  // [U]
  int32_t M, K, N;
  int32_t TM, TK, U;
  int64_t T;
  int32_t mode, split, num_pieces;
  uint64_t timeout_ns;
  int* status;
};

struct Range {
  int64_t b, e;
};

__device__ __forceinline__ Range piece_range(const SpmmParams& p, int64_t pc) {
  if (p.mode == 0) return {pc * p.T / p.num_pieces, (pc + 1) * p.T / p.num_pieces};
  const int64_t u = pc / p.split, c = pc - (pc / p.split) * p.split;
  return {u * p.TK + c * p.TK / p.split, u * p.TK + (c + 1) * p.TK / p.split};
}

// Piece that owns step q in mode 0: the largest pc with floor(pc*T/P) <= q.
__device__ __forceinline__ int64_t piece_of_step(const SpmmParams& p, int64_t q) {
  return ((q + 1) * p.num_pieces + p.T - 1) / p.T - 1;
}

// Workspace slot of piece pc's partial sum for unit u.
__device__ __forceinline__ int64_t partial_slot(const SpmmParams& p, int64_t pc, int64_t u) {
  if (p.mode == 1) return pc;
  return 2 * pc + ((piece_range(p, pc).b / p.TK) != u ? 1 : 0);
}

__device__ __forceinline__ bool named_barrier_or(uint32_t id, uint32_t nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void scatter_word(uint32_t dense_u32, uint32_t w, uint32_t top, bool& bad) {
  const uint32_t loc = w >> 16;
  if (loc < static_cast<uint32_t>(kMaxTileWords)) {
    const uint32_t r = top + (loc >> 6), c = loc & 63u;
    // 128-byte swizzle: 16-byte chunk index XOR (row mod 8) inside each 1024-byte atom
    const uint32_t addr = dense_u32 + r * 128u + ((((c >> 3) ^ (r & 7u)) << 4) | ((c & 7u) << 1));
    const uint16_t v = static_cast<uint16_t>(w & 0xFFFFu);
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
  } else if (loc != 0xFFFFu) {
    bad = true;
  }
}

template <int N_MMA>
__global__ void __launch_bounds__(kThreads, 1)
    spmm_lscd_sm100_kernel(const __grid_constant__ CUtensorMap tmap_b, const SpmmParams p) {
  using Cf = Cfg<N_MMA>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* dense = smem + Cf::kOffDense;
  uint8_t* bslab = smem + Cf::kOffB;
  uint8_t* ring = smem + Cf::kOffRing;
  int4* meta = reinterpret_cast<int4*>(smem + Cf::kOffMeta);
  int64_t* stage_end = reinterpret_cast<int64_t*>(smem + Cf::kOffEnd);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::kOffBars);
  uint64_t* words_full = bars;
  uint64_t* words_empty = words_full + Cf::kNumSlots;
  uint64_t* b_full = words_empty + Cf::kNumSlots;
  uint64_t* b_empty = b_full + Cf::kNumB;
  uint64_t* a_full = b_empty + Cf::kNumB;
  uint64_t* a_empty = a_full + Cf::kNumDense;
  uint64_t* acc_full = a_empty + Cf::kNumDense;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cf::kOffMisc + 4);
  volatile int* epi_last = reinterpret_cast<volatile int*>(smem + Cf::kOffMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Range rg = piece_range(p, blockIdx.x);
  const uint64_t budget = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < Cf::kNumSlots; ++i) { mbar_init(&words_full[i], 1); mbar_init(&words_empty[i], 1); }
    for (int i = 0; i < Cf::kNumB; ++i) { mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1); }
    for (int i = 0; i < Cf::kNumDense; ++i) { mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 1); }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    *epi_last = 0;
    fence_barrier_init();
  }
  if (warp == kWarpB && lane == 0) prefetch_tensor_map(&tmap_b);
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, Cf::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kWarpWords) {
    // ------------------------------------------------ sparse word producer
    const uint64_t policy = l2_policy_evict_first();
    int64_t head = 0, released = 0, next_confirm = 0, n = 0;
    bool stop = false;
    auto confirm_next = [&]() -> bool {
      const int s = static_cast<int>(next_confirm % Cf::kNumSlots);
      if (!mbar_wait(&words_empty[s], static_cast<uint32_t>((next_confirm / Cf::kNumSlots) & 1), abort_flag,
                     budget, p.status))
        return false;
      released = stage_end[s];
      ++next_confirm;
      return true;
    };
    // offsets of a batch of 32 steps are fetched one step per lane, one batch ahead
    auto fetch = [&](int64_t q0, int32_t& a0, int32_t& a1, int32_t& c0, int32_t& c1) {
      a0 = a1 = c0 = c1 = 0;
      const int64_t q = q0 + lane;
      if (q < rg.e) {
        const int64_t u = q / p.TK, j = q - (q / p.TK) * p.TK;
        const int64_t t0 = 2 * u * p.TK + j;
        a0 = __ldg(p.tile_offsets + t0);
        a1 = __ldg(p.tile_offsets + t0 + 1);
        if (2 * u + 1 < p.TM) {
          c0 = __ldg(p.tile_offsets + t0 + p.TK);
          c1 = __ldg(p.tile_offsets + t0 + p.TK + 1);
        }
      }
    };
    int32_t a0, a1, c0, c1;
    fetch(rg.b, a0, a1, c0, c1);
    for (int64_t q0 = rg.b; q0 < rg.e && !stop; q0 += 32) {
      int32_t na0, na1, nc0, nc1;
      fetch(q0 + 32, na0, na1, nc0, nc1);
      const int cnt = static_cast<int>(min64(32, rg.e - q0));
      for (int i = 0; i < cnt; ++i) {
        const int32_t x0 = __shfl_sync(0xFFFFFFFFu, a0, i), x1 = __shfl_sync(0xFFFFFFFFu, a1, i);
        const int32_t y0 = __shfl_sync(0xFFFFFFFFu, c0, i), y1 = __shfl_sync(0xFFFFFFFFu, c1, i);
        int fail = 0;
        if (lane == 0) {
          int32_t n0 = x1 - x0, n1 = y1 - y0;
          const bool ok0 = x0 >= 0 && n0 >= 0 && !(x0 & 3) && !(n0 & 3) && n0 <= kMaxTileWords && x1 <= p.nwords;
          const bool ok1 = y0 >= 0 && n1 >= 0 && !(y0 & 3) && !(n1 & 3) && n1 <= kMaxTileWords && y1 <= p.nwords;
          if (!ok0 || !ok1) record_status(p.status, FLASHSPMM_ERR_CORRUPT_FORMAT);
          if (!ok0) n0 = 0;
          if (!ok1) n1 = 0;
          const uint32_t bytes = 4u * static_cast<uint32_t>(n0 + n1);
          const int s = static_cast<int>(n % Cf::kNumSlots);
          bool ok = true;
          while (ok && next_confirm <= n - Cf::kNumSlots) ok = confirm_next();
          while (ok && head + bytes - released > Cf::kRingBytes) ok = confirm_next();
          if (ok) {
            meta[s] = make_int4(static_cast<int>((head % Cf::kRingBytes) >> 2), n0, n1, 0);
            mbar_arrive_expect_tx(&words_full[s], bytes);
            const int32_t src_off[2] = {x0, y0};
            const int32_t src_cnt[2] = {n0, n1};
            for (int h = 0; h < 2; ++h) {
              const uint8_t* src = reinterpret_cast<const uint8_t*>(p.words + src_off[h]);
              uint32_t left = 4u * static_cast<uint32_t>(src_cnt[h]);
              while (left) {
                const uint32_t pos = static_cast<uint32_t>(head % Cf::kRingBytes);
                const uint32_t chunk = minu32(left, Cf::kRingBytes - pos);
                bulk_copy_g2s(ring + pos, src, chunk, &words_full[s], policy);
                src += chunk;
                left -= chunk;
                head += chunk;
              }
            }
            stage_end[s] = head;
            ++n;
          } else {
            fail = 1;
          }
        }
        if (__shfl_sync(0xFFFFFFFFu, fail, 0)) { stop = true; break; }
      }
      a0 = na0; a1 = na1; c0 = nc0; c1 = nc1;
    }
    // drain: wait (bounded) for copies still in flight before the CTA exits
    if (lane == 0) {
      for (int64_t k = max64(0, n - Cf::kNumSlots); k < n; ++k)
        mbar_wait(&words_full[k % Cf::kNumSlots], static_cast<uint32_t>((k / Cf::kNumSlots) & 1), abort_flag,
                  budget, p.status);
    }
  } else if (warp == kWarpB) {
    // ------------------------------------------------ dense B producer (TMA)
    if (lane == 0) {
      int64_t n = 0;
      for (int64_t q = rg.b; q < rg.e; ++q, ++n) {
        const int s = static_cast<int>(n % Cf::kNumB);
        if (!mbar_wait(&b_empty[s], static_cast<uint32_t>(((n / Cf::kNumB) & 1) ^ 1), abort_flag, budget, p.status)) break;
        const int32_t j = static_cast<int32_t>(q % p.TK);
        mbar_arrive_expect_tx(&b_full[s], Cf::kBSlabBytes);
        tma_load_2d(bslab + s * Cf::kBSlabBytes, &tmap_b, j * kTile, 0, &b_full[s]);
      }
      for (int64_t k = max64(0, n - Cf::kNumB); k < n; ++k)
        mbar_wait(&b_full[k % Cf::kNumB], static_cast<uint32_t>((k / Cf::kNumB) & 1), abort_flag, budget, p.status);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------ tcgen05 MMA issuer
    if (lane == 0) {
      int64_t n = 0, uc = 0;
      bool issued = false;
      for (int64_t q = rg.b; q < rg.e; ++q, ++n) {
        const int64_t j = q % p.TK;
        const bool first = (q == rg.b) || (j == 0);
        const bool last = (q == rg.e - 1) || (j == p.TK - 1);
        const int ab = static_cast<int>(uc & 1);
        if (first) {
          if (!mbar_wait(&acc_empty[ab], static_cast<uint32_t>(((uc >> 1) & 1) ^ 1), abort_flag, budget, p.status)) break;
          tc_fence_after_sync();
        }
        const int s = static_cast<int>(n % Cf::kNumB), d = static_cast<int>(n % Cf::kNumDense);
        if (!mbar_wait(&b_full[s], static_cast<uint32_t>((n / Cf::kNumB) & 1), abort_flag, budget, p.status)) break;
        if (!mbar_wait(&a_full[d], static_cast<uint32_t>((n / Cf::kNumDense) & 1), abort_flag, budget, p.status)) break;
        tc_fence_after_sync();
        const uint64_t adesc = smem_desc_k_sw128(smem_u32(dense + d * kDenseBytes));
        const uint64_t bdesc = smem_desc_k_sw128(smem_u32(bslab + s * Cf::kBSlabBytes));
        const uint32_t tmem_d = tmem_base + static_cast<uint32_t>(ab * N_MMA);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)  // K = 16 per MMA: advance 32 bytes inside the swizzle atom
          umma_f16_ss(tmem_d, adesc + 2 * kk, bdesc + 2 * kk, Cf::kIdesc, (first && kk == 0) ? 0u : 1u);
        issued = true;
        umma_commit(&b_empty[s]);
        umma_commit(&a_empty[d]);
        if (last) {
          umma_commit(&acc_full[ab]);
          ++uc;
        }
      }
      if (issued) {  // all MMAs retired before tensor memory is released
        umma_commit(mma_done);
        mbar_wait(mma_done, 0, abort_flag, budget, p.status);
      }
    }
    __syncwarp();
  } else if (warp >= kWarpEpi && warp < kWarpEpi + 4) {
    // ------------------------------------------------ epilogue
    const int etid = threadIdx.x - kWarpEpi * 32;
    const int quarter = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int64_t u_first = rg.b / p.TK, u_last = (rg.e - 1) / p.TK;
    for (int64_t u = u_first; u <= u_last && rg.e > rg.b; ++u) {
      const int64_t uc = u - u_first;
      const int ab = static_cast<int>(uc & 1);
      const bool ok = mbar_wait(&acc_full[ab], static_cast<uint32_t>((uc >> 1) & 1), abort_flag, budget, p.status);
      if (named_barrier_or(kBarEpi, kEpiThreads, !ok)) break;
      tc_fence_after_sync();
      const int64_t seg_b = max64(rg.b, u * p.TK), seg_e = min64(rg.e, (u + 1) * p.TK);
      const bool complete = seg_b == u * p.TK && seg_e == (u + 1) * p.TK;
      const int64_t m = u * kUnitRows + row;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(ab * N_MMA);
      float* part = nullptr;
      if (!complete) part = p.partials + partial_slot(p, blockIdx.x, u) * static_cast<int64_t>(p.N) * kUnitRows;
#pragma unroll 1
      for (int c = 0; c < N_MMA && c < p.N; c += 16) {
        uint32_t v[16];
        tmem_load_16(taddr + c, v);
        tmem_load_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int nn = c + i;
          if (nn < p.N) {
            const float x = __uint_as_float(v[i]);
            if (complete) {
              if (m < p.M) p.C[static_cast<int64_t>(nn) * p.M + m] = __float2half_rn(x);
            } else {
              part[static_cast<int64_t>(nn) * kUnitRows + row] = x;
            }
          }
        }
      }
      tc_fence_before_sync();
      named_barrier(kBarEpi, kEpiThreads);
      if (etid == 0) mbar_arrive(&acc_empty[ab]);
      if (!complete) {
        // last-arriver reduction of the unit's partial sums, in piece order
        int64_t first_pc, ncontrib;
        if (p.mode == 0) {
          first_pc = piece_of_step(p, u * p.TK);
          ncontrib = piece_of_step(p, u * p.TK + p.TK - 1) - first_pc + 1;
        } else {
          first_pc = u * p.split;
          ncontrib = p.split;
        }
        __threadfence();
        named_barrier(kBarEpi, kEpiThreads);
        if (etid == 0) *epi_last = (atomicAdd(p.counters + u, 1) == ncontrib - 1) ? 1 : 0;
        named_barrier(kBarEpi, kEpiThreads);
        if (*epi_last) {
          __threadfence();
          for (int nn = 0; nn < p.N; ++nn) {
            float acc = 0.0f;
            for (int64_t k = 0; k < ncontrib; ++k) {
              const int64_t sl = partial_slot(p, first_pc + k, u);
              acc += __ldcg(p.partials + (sl * p.N + nn) * kUnitRows + row);
            }
            if (m < p.M) p.C[static_cast<int64_t>(nn) * p.M + m] = __float2half_rn(acc);
          }
          if (etid == 0) p.counters[u] = 0;
        }
        named_barrier(kBarEpi, kEpiThreads);
      }
    }
  } else {
    // ------------------------------------------------ decompress (rst_smem + extract)
    const int dtid = threadIdx.x - kWarpDec * 32;
    const uint4* ring4 = reinterpret_cast<const uint4*>(ring);
    bool bad = false;
    int64_t n = 0;
    for (int64_t q = rg.b; q < rg.e; ++q, ++n) {
      const int d = static_cast<int>(n % Cf::kNumDense), s = static_cast<int>(n % Cf::kNumSlots);
      bool ok = mbar_wait(&a_empty[d], static_cast<uint32_t>(((n / Cf::kNumDense) & 1) ^ 1), abort_flag, budget, p.status);
      uint8_t* dbuf = dense + d * kDenseBytes;
      if (ok) {
        uint4* dz = reinterpret_cast<uint4*>(dbuf);
#pragma unroll
        for (int i = 0; i < kDenseBytes / 16 / kDecThreads; ++i) dz[i * kDecThreads + dtid] = make_uint4(0, 0, 0, 0);
        ok = mbar_wait(&words_full[s], static_cast<uint32_t>((n / Cf::kNumSlots) & 1), abort_flag, budget, p.status);
      }
      if (named_barrier_or(kBarDec, kDecThreads, !ok)) break;
      const int4 mt = meta[s];
      const int nvec = (mt.y + mt.z) >> 2;
      const uint32_t dense_u32 = smem_u32(dbuf);
      for (int v = dtid; v < nvec; v += kDecThreads) {
        const uint32_t widx = static_cast<uint32_t>(mt.x + 4 * v) % Cf::kRingWords;
        const uint4 w4 = ring4[widx >> 2];
        const uint32_t top = (4 * v < mt.y) ? 0u : 64u;
        scatter_word(dense_u32, w4.x, top, bad);
        scatter_word(dense_u32, w4.y, top, bad);
        scatter_word(dense_u32, w4.z, top, bad);
        scatter_word(dense_u32, w4.w, top, bad);
      }
      fence_proxy_async_smem();
      named_barrier(kBarDec, kDecThreads);
      if (dtid == 0) {
        mbar_arrive(&a_full[d]);
        mbar_arrive(&words_empty[s]);
      }
    }
    if (bad) record_status(p.status, FLASHSPMM_ERR_CORRUPT_FORMAT);
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, Cf::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

template <int N_MMA>
flashspmm_status launch_bucket(const flashspmm_tcsl* A, const void* B, void* C, int32_t M, int32_t K, int32_t N,
                               const SpmmPlan& plan, void* workspace, cudaStream_t s) {
  using Cf = Cfg<N_MMA>;
  EncodeTiledFn encode = get_encode_tiled();
  if (!encode) return FLASHSPMM_ERR_CUDA;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTile), static_cast<cuuint32_t>(N_MMA)};
  const cuuint32_t estride[2] = {1, 1};
  if (encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(B), dims, strides, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return FLASHSPMM_ERR_CUDA;

  static std::atomic<uint64_t> attr_set_mask{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLASHSPMM_ERR_CUDA;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(attr_set_mask.load() & bit)) {
    if (cudaFuncSetAttribute(spmm_lscd_sm100_kernel<N_MMA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cf::kSmemBytes) != cudaSuccess)
      return FLASHSPMM_ERR_CUDA;
    attr_set_mask.fetch_or(bit);
  }

  SpmmParams p{};
  p.tile_offsets = A->tile_offsets;
  p.words = A->words;
  p.nwords = A->nwords;
  p.C = static_cast<__half*>(C);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.partials = plan.partial_bytes ? reinterpret_cast<float*>(ws) : nullptr;
  p.counters = plan.counter_bytes ? reinterpret_cast<int32_t*>(ws + plan.partial_bytes) : nullptr;
  p.M = M; p.K = K; p.N = N;
  p.TM = plan.TM; p.TK = plan.TK; p.U = plan.U; p.T = plan.T;
  p.mode = plan.mode; p.split = plan.split; p.num_pieces = plan.num_pieces;
  p.timeout_ns = 1000000000ull;  // 1 s: far above any legitimate wait
  p.status = device_status_ptr();

  if (p.counters && cudaMemsetAsync(p.counters, 0, plan.counter_bytes, s) != cudaSuccess) return FLASHSPMM_ERR_CUDA;
  spmm_lscd_sm100_kernel<N_MMA><<<plan.num_pieces, kThreads, Cf::kSmemBytes, s>>>(tmap, p);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? FLASHSPMM_OK : FLASHSPMM_ERR_CUDA;
}

}  // namespace

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

SpmmPlan make_spmm_plan(int32_t M, int32_t K, int32_t N, int32_t split_k, int num_sms) {
  SpmmPlan pl{};
  pl.TM = (M + kTile - 1) / kTile;
  pl.TK = (K + kTile - 1) / kTile;
  pl.U = (pl.TM + 1) / 2;
  pl.T = static_cast<int64_t>(pl.U) * pl.TK;
  if (pl.T == 0) return pl;
  if (split_k <= 0) {
    pl.mode = 0;
    pl.split = 0;
    const int64_t want = (pl.T + kMinStepsPerPiece - 1) / kMinStepsPerPiece;
    pl.num_pieces = static_cast<int32_t>(max64(1, min64(want, num_sms > 1 ? num_sms : 1)));
    pl.partial_slots = pl.num_pieces > 1 ? 2 * static_cast<int64_t>(pl.num_pieces) : 0;
  } else {
    pl.mode = 1;
    pl.split = split_k < pl.TK ? split_k : pl.TK;
    pl.num_pieces = static_cast<int32_t>(static_cast<int64_t>(pl.U) * pl.split);
    pl.partial_slots = pl.split > 1 ? pl.num_pieces : 0;
  }
  pl.counters = pl.partial_slots ? pl.U : 0;
  pl.partial_bytes = align256(static_cast<size_t>(pl.partial_slots) * kUnitRows * N * sizeof(float));
  pl.counter_bytes = align256(static_cast<size_t>(pl.counters) * sizeof(int32_t));
  pl.workspace_bytes = pl.partial_bytes + pl.counter_bytes;
  return pl;
}

flashspmm_status launch_spmm_lscd(const flashspmm_tcsl* A, const void* B, void* C, int32_t M, int32_t K,
                                  int32_t N, const SpmmPlan& plan, void* workspace, cudaStream_t s) {
  if (N <= 16) return launch_bucket<16>(A, B, C, M, K, N, plan, workspace, s);
  if (N <= 32) return launch_bucket<32>(A, B, C, M, K, N, plan, workspace, s);
  if (N <= 64) return launch_bucket<64>(A, B, C, M, K, N, plan, workspace, s);
  if (N <= 128) return launch_bucket<128>(A, B, C, M, K, N, plan, workspace, s);
  return launch_bucket<256>(A, B, C, M, K, N, plan, workspace, s);
}

}  // namespace flashspmm
