// LSCD SpMM for sm_100a: C = A x B with A in Tiled-CSL (64 x 64 tiles), B a
// skinny fp16 K x N matrix, fp32 accumulation in tensor memory, fp16 C.
//
// Method (Flash-LLM paper review, xllm-io.github.io): the weights are loaded
// in their sparse form to cut HBM bytes, expanded on chip into dense tiles and
// multiplied densely on the tensor cores (section 2, "solution overview";
// section 3, pipeline stages gmem2reg / rst_smem / extract / ld_dense /
// smem2tc / TC_compute, overlapped across iterations).  The A100 kernel on the
// page (register-staged extraction, ldmatrix + mma.sync, cp.async double
// buffering) is prior art; this kernel keeps the stages and maps each one to
// sm_100a:
//
//   gmem2reg  -> decompress warps stream their tiles' word lists into a
//                per-warp shared-memory ring with cp.async (16 bytes per lane
//                per copy, three 256-word batches in flight per warp, no
//                registers held), then read each batch with conflict-free
//                32-bit shared loads; each warp's tiles are consecutive in
//                memory (see below), so its copies form one stream;
//   rst_smem  -> each warp zeroes its strip's half of a 128 x 64 dense A
//   + extract    buffer with 16-byte stores and scatters every word's value to its swizzled
//                position (UMMA K-major 128-byte layout);
//   ld_dense  -> each step's B slab (64 K x N_MMA) is loaded by TMA into the
//                step's buffer in the same swizzled layout, completing on the
//                barrier that hands the step to the MMA warps;
//   smem2tc   -> gone: tcgen05.mma reads both operands from shared memory;
//   TC_compute-> two MMA warps issue 4 x tcgen05.mma (M = 128, K = 16) per step
//                into double-buffered fp32 accumulators in tensor memory;
//   epilogue  -> 4 warps read the accumulator with tcgen05.ld and write fp16 C
//                (or fp32 partial sums, see below).
//
// A "unit" is 128 rows of A (two 64-row format strips stacked on the MMA M
// side); a "step" is one 64-wide K tile of one unit.  Each pair of decompress
// warps owns one buffer (16 KB dense A tile + B slab) and expands its share of
// the CTA's steps into it, one warp per strip: two mbarrier arrivals and the
// B slab's bytes hand the step to the MMA warps, one tcgen05.commit hands the
// buffer back.  No pair waits on another pair.
//
// The T = units x K-tiles steps are cut into contiguous pieces, one CTA each.
// When a unit is shared by several pieces, every piece writes its fp32
// partial sum to the workspace and the last piece to finish (atomic arrival
// counter) adds them in piece order and writes C: the split-K reduction of the
// page's Reduction kernel (section 5, "project structure"), fused and
// deterministic.
#include <cuda.h>
#include <cuda_fp16.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flashspmm {
namespace {

constexpr int kTile = 64;                           // format tile edge (rows and K)
constexpr int kUnitRows = 128;                      // MMA M
constexpr int kDenseBytes = kUnitRows * kTile * 2;  // 16 KB dense A buffer (one step)
constexpr int kHalfBytes = kDenseBytes / 2;         // one strip's 64 rows
constexpr int kMaxTileWords = kTile * kTile;        // 4096 words (already a multiple of 4)
// Warp roles: MMA issuers (warps 0 and 1), epilogue (2-5, one per
// tensor-memory lane quarter), decompress warps (6 and up, in pairs).
constexpr int kWarpMma = 0, kWarpMma1 = 1, kWarpEpi = 2, kWarpDec = 6;
constexpr int kEpiThreads = 128;
constexpr int kBarEpi = 1;                          // named barrier id of the epilogue warps
constexpr int kMinStepsPerPiece = 4;

// Decompress-warp word streaming: a batch is kRB rounds of 32 words (one word
// per lane per round) of one tile.  Batches are copied from global memory into
// a per-warp shared-memory ring of kStage slots with cp.async (16 bytes per
// lane per copy, no registers held while in flight); kStage - 1 batches are in
// flight while one is expanded.
constexpr int kRB = 8;
constexpr int kBatchWords = kRB * 32;
constexpr int kStage = 4;
constexpr int kStageBytes = kStage * kBatchWords * 4;  // 4 KB per decompress warp

// A batch descriptor packed in 32 bits: its word count (bits 0-8), the K tile
// of its step (bits 9-28, used to load the step's B slab) and three flags.
constexpr uint32_t kDescCountMask = (1u << 9) - 1u;
constexpr int kDescTileShift = 9;
constexpr uint32_t kDescTileMask = (1u << 20) - 1u;
constexpr uint32_t kDescValid = 1u << 29, kDescFirst = 1u << 30, kDescLast = 1u << 31;
constexpr int32_t kMaxKTiles = 1 << 20;             // K tiles a descriptor can name

template <int N_MMA>
struct Bufs {  // dense buffers (decompress pairs) per CTA for an N bucket
  static constexpr int value = N_MMA <= 32 ? 8 : (N_MMA == 64 ? 6 : (N_MMA == 128 ? 5 : 4));
};

template <int N_MMA, int ND>
struct Cfg {
  static_assert(N_MMA == 16 || N_MMA == 32 || N_MMA == 64 || N_MMA == 128 || N_MMA == 256, "N bucket");
  static constexpr int kThreads = (kWarpDec + 2 * ND) * 32;  // two decompress warps per dense buffer
  // Two MMA warps take the pairs by parity, each into its own accumulator (summed
  // in a fixed order by the epilogue), so two issue chains and two
  // accumulation chains run side by side; at N = 256 one accumulator pair
  // already fills tensor memory and a single MMA warp is used.
  static constexpr int kMmaWarps = N_MMA <= 128 ? 2 : 1;
  static constexpr int kBSlabBytes = N_MMA * kTile * 2;   // one 64-wide K tile of B (N_MMA rows)
  static constexpr int kPairBytes = kDenseBytes + kBSlabBytes;  // a pair's dense A tile + its B slab
  static constexpr int kTmemCols = 2 * kMmaWarps * N_MMA < 32 ? 32 : 2 * kMmaWarps * N_MMA;
  static constexpr uint32_t kIdesc = umma_idesc_f16_f32(kUnitRows, N_MMA);
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int kOffStage = ND * kPairBytes;              // word staging rings
  static constexpr int kOffBars = kOffStage + 2 * ND * kStageBytes;
  static constexpr int kNumBars = 2 * ND + 4 + 1;
  static constexpr int kOffMisc = kOffBars + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct SpmmParams {
  const int32_t* tile_offsets;
  const uint32_t* words;
  int64_t nwords;
  __half* C;
  float* partials;    // [slot][N][128]
  int32_t* counters;  // mode 0: one per piece (the first piece of a shared unit); mode 1: one per unit
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

__host__ __device__ __forceinline__ Range piece_range(const SpmmParams& p, int64_t pc) {
  if (p.mode == 0) return {pc * p.T / p.num_pieces, (pc + 1) * p.T / p.num_pieces};
  const int64_t u = pc / p.split, c = pc - (pc / p.split) * p.split;
  return {u * p.TK + c * p.TK / p.split, u * p.TK + (c + 1) * p.TK / p.split};
}

// Piece that owns step q in mode 0: the largest pc with floor(pc*T/P) <= q.
__host__ __device__ __forceinline__ int64_t piece_of_step(const SpmmParams& p, int64_t q) {
  return ((q + 1) * p.num_pieces + p.T - 1) / p.T - 1;
}

// Workspace slot of piece pc's partial sum for unit u.
__host__ __device__ __forceinline__ int64_t partial_slot(const SpmmParams& p, int64_t pc, int64_t u) {
  if (p.mode == 1) return pc;
  return 2 * pc + ((piece_range(p, pc).b / p.TK) != u ? 1 : 0);
}

// A piece is walked unit by unit: its segment in unit u covers K tiles
// [j0, j1), and pair b of the CTA expands the contiguous run
// [j0 + b*L/ND, j0 + (b+1)*L/ND) of it (L = j1 - j0), so each decompress warp
// streams a contiguous range of its strip's words.  The MMA warps take the
// pairs' steps round robin (round r: the r-th step of pairs 0, 1, ...), a
// fixed order, so results are deterministic.
struct Segment {
  int64_t u;
  int j0, len;
};

__device__ __forceinline__ Segment segment_at(const SpmmParams& p, const Range& rg, int64_t q) {
  Segment sg;
  sg.u = q / p.TK;
  sg.j0 = static_cast<int>(q - sg.u * p.TK);
  sg.len = static_cast<int>(min64(rg.e - sg.u * p.TK, p.TK)) - sg.j0;
  return sg;
}

template <int ND>
__host__ __device__ __forceinline__ int chunk_begin(int len, int b) {
  return b * len / ND;
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

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xFFFFFFFF;\n\tselp.b32 %0, 1, 0, P;\n\t}" : "=r"(pred));
  return pred != 0;
}

// Words are read with streaming loads (ld.global.cs: evict-first, every word
// is used exactly once).

// Writes one word's value into a strip's 64 x 64 half of the dense buffer at
// its swizzled place.  loc = r*64 + c; the unswizzled byte offset is
// 2*loc = r*128 + 2c, and the 128-byte swizzle XORs the 16-byte chunk index
// (bits 4-6) with r mod 8 (bits 7-9 of the same offset).  Only words with
// loc < 4096 are written: the sentinel (loc 0xFFFF) and any corrupt loc
// beyond the tile are skipped by the same test, so no write leaves the half.
__device__ __forceinline__ void scatter_word(uint32_t half_u32, uint32_t w) {
  // half_u32 is 1024-aligned, so the swizzle XOR may be applied after adding it
  const uint32_t addr = (half_u32 + 2u * (w >> 16)) ^ ((w >> 18) & 0x70u);
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.lt.u32 q, %1, 0x10000000;\n\t"
      "@q st.shared.u16 [%0], %1;\n\t}" ::"r"(addr),
      "r"(w));
}

// A word range [b, e) from the tile offsets is usable iff it lies inside the
// word array, starts on a 16-byte boundary and holds at most one tile.
__device__ __forceinline__ bool range_ok(int32_t b, int32_t e, int64_t nwords) {
  const int32_t n = e - b;
  return b >= 0 && n >= 0 && !(b & 3) && !(n & 3) && n <= kMaxTileWords && e <= nwords;
}

template <int N_MMA, int ND>
__global__ void __launch_bounds__(Cfg<N_MMA, ND>::kThreads, 1)
    spmm_lscd_sm100_kernel(const __grid_constant__ CUtensorMap tmap_b, const SpmmParams p) {
  using Cf = Cfg<N_MMA, ND>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bufs = smem;  // ND x (dense A tile, B slab)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::kOffBars);
  uint64_t* full = bars;             // [ND]: step expanded (one arrival per strip + the B slab's bytes)
  uint64_t* empty = full + ND;       // [ND]: step consumed (one commit)
  uint64_t* acc_full = empty + ND;   // [2]: accumulators of a unit complete (one commit per MMA warp)
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cf::kOffMisc + 4);
  volatile int* epi_last = reinterpret_cast<volatile int*>(smem + Cf::kOffMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Range rg = piece_range(p, blockIdx.x);
  const uint64_t budget = p.timeout_ns;

  griddep_launch_dependents();
  if (warp == kWarpMma1) {
    if (lane < ND) {
      mbar_init(&full[lane], 2);  // both strips of the step (the B slab adds its bytes)
      mbar_init(&empty[lane], 1);
    }
    if (lane < 2) {
      mbar_init(&acc_full[lane], Cf::kMmaWarps);  // one commit per MMA warp
      mbar_init(&acc_empty[lane], 1);
    }
    if (lane == 0) {
      mbar_init(mma_done, Cf::kMmaWarps);
      *abort_flag = 0;
      *epi_last = 0;
      prefetch_tensor_map(&tmap_b);
    }
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, Cf::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touched no global memory; from here on the inputs (which
  // the previous kernel in the stream may have written) are read.
  griddep_wait();

  if (warp == kWarpMma || warp == kWarpMma1) {
    // ------------------------------------------------ tcgen05 MMA issuers
    // MMA warp m issues the steps of pairs b with b % kMmaWarps == m, in the
    // round-robin order, into its own accumulator of the unit.  Every lane
    // tests the barriers itself (no broadcast needed) and one elected lane
    // issues the MMAs and commits (issue from a converged warp is markedly
    // cheaper than from a lone divergent thread).
    const int m = warp == kWarpMma ? 0 : 1;
    if (m < Cf::kMmaWarps) {
      const bool leader = elect_one();
      int ac = 0;          // accumulator pair of the current unit
      uint32_t acph = 1;   // parity to wait on acc_empty[ac]
      uint32_t fph = 0;    // bit b: parity to wait on full[b]
      const uint64_t desc0 = smem_desc_k_sw128(smem_u32(bufs));
      const uint32_t tmem_m = tmem_base + static_cast<uint32_t>(m * N_MMA);
      bool ok = true;
      for (int64_t q = rg.b; q < rg.e && ok;) {
        const Segment sg = segment_at(p, rg, q);
        if (!mbar_wait(&acc_empty[ac], acph, abort_flag, budget, p.status)) break;
        tc_fence_after_sync();  // accumulator handed back by the epilogue's tcgen05.ld
        const uint32_t tmem_d = tmem_m + static_cast<uint32_t>(ac * Cf::kMmaWarps * N_MMA);
        uint32_t acc_flag = 0u;  // 0 until this warp's first MMA of the unit
        const int rounds = (sg.len + ND - 1) / ND;
        for (int r = 0; r < rounds && ok; ++r) {
#pragma unroll
          for (int b = m; b < ND; b += Cf::kMmaWarps) {
            if (r < chunk_begin<ND>(sg.len, b + 1) - chunk_begin<ND>(sg.len, b)) {
              if (!mbar_wait(&full[b], (fph >> b) & 1u, abort_flag, budget, p.status)) {
                ok = false;
                break;
              }
              fph ^= 1u << b;
              if (leader) {
                // descriptor start addresses advance in 16-byte units; K = 16
                // per MMA advances 32 bytes (2 units) inside the swizzle atom
                const uint64_t adesc = desc0 + static_cast<uint64_t>((b * Cf::kPairBytes) >> 4);
                const uint64_t bdesc = adesc + static_cast<uint64_t>(kDenseBytes >> 4);
                umma_f16_ss(tmem_d, adesc, bdesc, Cf::kIdesc, acc_flag);
#pragma unroll
                for (int kk = 1; kk < kTile / 16; ++kk)
                  umma_f16_ss(tmem_d, adesc + 2 * kk, bdesc + 2 * kk, Cf::kIdesc, 1u);
                umma_commit(&empty[b]);
              }
              acc_flag = 1u;
            }
          }
        }
        if (!ok) break;
        if (leader) umma_commit(&acc_full[ac]);
        __syncwarp();
        if (ac == 1) acph ^= 1u;
        ac ^= 1;
        q = (sg.u + 1) * p.TK;
      }
      // all MMAs of both warps retired before tensor memory is released
      if (leader) umma_commit(mma_done);
      __syncwarp();
      if (lane == 0) mbar_wait_drain(mma_done, 0, budget, p.status);
      __syncwarp();
    }
  } else if (warp >= kWarpEpi && warp < kWarpEpi + 4) {
    // ------------------------------------------------ epilogue
    const int etid = threadIdx.x - kWarpEpi * 32;
    const int quarter = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int64_t u_first = rg.b / p.TK, u_last = (rg.e - 1) / p.TK;
    for (int64_t u = u_first; u <= u_last && rg.e > rg.b; ++u) {
      const int64_t uc = u - u_first;
      const int ab = static_cast<int>(uc & 1);
      bool ok = true;
      if (etid == 0) ok = mbar_wait(&acc_full[ab], static_cast<uint32_t>((uc >> 1) & 1), abort_flag, budget, p.status);
      if (named_barrier_or(kBarEpi, kEpiThreads, !ok)) break;  // the other threads sleep here
      tc_fence_after_sync();
      const int64_t seg_b = max64(rg.b, u * p.TK), seg_e = min64(rg.e, (u + 1) * p.TK);
      const bool complete = seg_b == u * p.TK && seg_e == (u + 1) * p.TK;
      const int64_t m = u * kUnitRows + row;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(ab * Cf::kMmaWarps * N_MMA);
      // MMA warp w wrote its accumulator iff one of its pairs (b % kMmaWarps
      // == w) had a step in the segment
      const int len = static_cast<int>(seg_e - seg_b);
      bool has0 = false, has1 = false;
#pragma unroll
      for (int b = 0; b < ND; ++b) {
        const bool any = chunk_begin<ND>(len, b + 1) > chunk_begin<ND>(len, b);
        if (Cf::kMmaWarps == 1 || (b & 1) == 0) has0 |= any;
        else has1 |= any;
      }
      float* part = nullptr;
      if (!complete) part = p.partials + partial_slot(p, blockIdx.x, u) * static_cast<int64_t>(p.N) * kUnitRows;
#pragma unroll 1
      for (int c = 0; c < N_MMA && c < p.N; c += 8) {
        uint32_t v[8], w[8];
        if (has0) tmem_load_8(taddr + c, v);
        if (has1) tmem_load_8(taddr + N_MMA + c, w);
        tmem_load_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int nn = c + i;
          if (nn < p.N) {
            const float x = has0 && has1 ? __uint_as_float(v[i]) + __uint_as_float(w[i])
                                         : __uint_as_float(has0 ? v[i] : w[i]);
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
        int32_t* const counter = p.counters + (p.mode == 0 ? first_pc : u);
        __threadfence();
        named_barrier(kBarEpi, kEpiThreads);
        if (etid == 0) *epi_last = (atomicAdd(counter, 1) == ncontrib - 1) ? 1 : 0;
        named_barrier(kBarEpi, kEpiThreads);
        if (*epi_last) {
          __threadfence();
#pragma unroll 1
          for (int nc = 0; nc < p.N; nc += 8) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll 1
            for (int64_t k = 0; k < ncontrib; ++k) {
              const float* src = p.partials + (partial_slot(p, first_pc + k, u) * p.N + nc) * kUnitRows + row;
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if (nc + i < p.N) acc[i] += __ldcg(src + i * kUnitRows);
            }
            if (m < p.M) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if (nc + i < p.N) p.C[static_cast<int64_t>(nc + i) * p.M + m] = __float2half_rn(acc[i]);
            }
          }
          if (etid == 0) *counter = 0;  // zero again for the next call
        }
        named_barrier(kBarEpi, kEpiThreads);
      }
    }
  } else {
    // ------------------------------------------------ decompress (gmem2reg + rst_smem + extract)
    // Pair b owns buffer b (dense A tile + B slab); warp h of the pair expands
    // strip h (rows 64h .. 64h + 63) of each of the pair's steps.  The pair's
    // steps are, unit segment by unit segment, its contiguous run of K tiles,
    // so a warp's tiles follow one another in memory and its loads stream.
    // Word lists are copied in batches of up to kBatchWords words into the
    // warp's staging ring, kStage - 1 batches ahead of the one being expanded,
    // and expanded word w of a batch on lane w % 32, round w / 32; a batch
    // never straddles two tiles, so every 32-word round
    // starts on a 32-word boundary from its tile's start (the windows the
    // bank-balanced word order is built for).  The first batch of a step waits
    // until the MMAs of the buffer's previous step have retired, starts the
    // TMA load of the step's B slab (warp 0 of the pair) and zeroes the warp's
    // half; the last one publishes the half to the MMA warps.
    const int dw = warp - kWarpDec;
    const int pair = dw >> 1, h = dw & 1;
    uint8_t* const pbuf = bufs + pair * Cf::kPairBytes;
    const uint32_t hb = smem_u32(pbuf + h * kHalfBytes);
    // k-th step of this pair: its unit and K tile (false past the last step)
    auto step_of = [&](int k, int64_t& u, int& j) -> bool {
      for (int64_t q = rg.b; q < rg.e;) {
        const Segment sg = segment_at(p, rg, q);
        const int c0 = chunk_begin<ND>(sg.len, pair), c1 = chunk_begin<ND>(sg.len, pair + 1);
        if (k < c1 - c0) {
          u = sg.u;
          j = sg.j0 + c0 + k;
          return true;
        }
        k -= c1 - c0;
        q = (sg.u + 1) * p.TK;
      }
      return false;
    };
    int my_steps = 0;
    for (int64_t q = rg.b; q < rg.e;) {
      const Segment sg = segment_at(p, rg, q);
      my_steps += chunk_begin<ND>(sg.len, pair + 1) - chunk_begin<ND>(sg.len, pair);
      q = (sg.u + 1) * p.TK;
    }
    // Raw tile offsets (begin, end) and K tile of 32 consecutive steps of this
    // warp, one step per lane.
    auto load_tab = [&](int k0, int32_t& ob, int32_t& oe, int32_t& oj) {
      ob = oe = oj = 0;
      int64_t u;
      int j;
      if (step_of(k0 + lane, u, j)) {
        oj = j;
        if (2 * u + h < p.TM) {
          const int64_t t = (2 * u + h) * p.TK + j;
          ob = __ldg(p.tile_offsets + t);
          oe = __ldg(p.tile_offsets + t + 1);
        }
      }
    };
    // Turns a raw (begin, end) into (start, length); a range that breaks the
    // format is reported and replaced by an empty tile.
    auto validate = [&](int32_t ob, int32_t oe, int32_t& ca, int32_t& cn) {
      const bool ok = range_ok(ob, oe, p.nwords);
      ca = ok ? ob : 0;
      cn = ok ? oe - ob : 0;
      if (!ok) record_status(p.status, FLASHSPMM_ERR_CORRUPT_FORMAT);
    };
    int32_t cur_a, cur_n, cur_j, nxt_b, nxt_e, nxt_j;
    {
      int32_t ob, oe;
      load_tab(0, ob, oe, cur_j);
      load_tab(32, nxt_b, nxt_e, nxt_j);
      validate(ob, oe, cur_a, cur_n);
    }
    int tab_base = 0;

    // ---- issue side: walks the warp's tiles and batches, copying each batch
    // into its staging slot
    const uint32_t stage = smem_u32(bufs + Cf::kOffStage + dw * kStageBytes);
    const uint32_t* const stage_w = reinterpret_cast<const uint32_t*>(bufs + Cf::kOffStage + dw * kStageBytes);
    int ij = 0, ipos = 0;
    int32_t ia = 0, in = 0;
    uint32_t itile = 0;
    auto issue = [&](uint32_t& desc, int slot) {
      if (ij < my_steps) {
        uint32_t flags = kDescValid;
        if (ipos == 0) {
          if (ij - tab_base == 32) {
            tab_base += 32;
            validate(nxt_b, nxt_e, cur_a, cur_n);
            cur_j = nxt_j;
            load_tab(tab_base + 32, nxt_b, nxt_e, nxt_j);
          }
          const int li = ij - tab_base;
          ia = __shfl_sync(0xFFFFFFFFu, cur_a, li);
          in = __shfl_sync(0xFFFFFFFFu, cur_n, li);
          itile = static_cast<uint32_t>(__shfl_sync(0xFFFFFFFFu, cur_j, li));
          flags |= kDescFirst;
        }
        const int cnt = min(in - ipos, kBatchWords);  // a multiple of 4 words
        // lane l copies the 16-byte groups l and l + 32 of the batch (words 4g .. 4g + 3)
        const uint32_t* src = p.words + (static_cast<int64_t>(ia) + ipos + 4 * lane);
        const uint32_t dst = stage + static_cast<uint32_t>(slot * kBatchWords * 4 + lane * 16);
        if (4 * lane < cnt) cp_async_16(dst, src);
        if (4 * (lane + 32) < cnt) cp_async_16(dst + 512, src + 128);
        ipos += kBatchWords;
        if (ipos >= in) {
          flags |= kDescLast;
          ++ij;
          ipos = 0;
        }
        desc = static_cast<uint32_t>(cnt) | ((itile & kDescTileMask) << kDescTileShift) | flags;
      } else {
        desc = 0u;
      }
      cp_async_commit();  // one group per batch slot, empty ones included, so the counting stays uniform
    };

    // ---- expand side
    int pj = 0;  // index (among this pair's steps) of the step being expanded
    auto process = [&](uint32_t desc, int slot) -> bool {
      if (desc & kDescFirst) {
        // the buffer is free once the MMAs of its previous step have retired
        if (!mbar_wait(&empty[pair], static_cast<uint32_t>((pj & 1) ^ 1), abort_flag, budget, p.status)) return false;
        if (h == 0 && lane == 0) {
          // the step's B slab: 64 K values x N_MMA rows (rows past N read as zero)
          mbar_expect_tx(&full[pair], static_cast<uint32_t>(Cf::kBSlabBytes));
          tma_load_2d(pbuf + kDenseBytes, &tmap_b, static_cast<int32_t>((desc >> kDescTileShift) & kDescTileMask) * kTile,
                      0, &full[pair]);
        }
#pragma unroll
        for (int i = 0; i < kHalfBytes / 16 / 32; ++i) st_shared_zero16(hb + static_cast<uint32_t>((i * 32 + lane) * 16));
        __syncwarp();
      }
      const int cnt = static_cast<int>(desc & kDescCountMask);
      const uint32_t* sw = stage_w + slot * kBatchWords + lane;
      if (cnt == kBatchWords) {
#pragma unroll
        for (int i = 0; i < kRB; ++i) scatter_word(hb, sw[32 * i]);
      } else {
#pragma unroll
        for (int i = 0; i < kRB; ++i)
          if (32 * i < cnt) scatter_word(hb, 32 * i + lane < cnt ? sw[32 * i] : kSentinel);
      }
      if (desc & kDescLast) {
        fence_proxy_async_smem();  // generic-proxy stores -> tensor-core (async proxy) reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[pair]);
        ++pj;
      }
      return true;
    };

    uint32_t dsc[kStage];
#pragma unroll
    for (int s = 0; s < kStage - 1; ++s) issue(dsc[s], s);
    bool run = true;
    while (run) {
#pragma unroll
      for (int s = 0; s < kStage; ++s) {
        if (run) {
          __syncwarp();  // every lane is done reading the slot about to be refilled
          issue(dsc[(s + kStage - 1) % kStage], (s + kStage - 1) % kStage);
          cp_async_wait<kStage - 1>();  // this lane's copies of slot s have landed
          __syncwarp();                 // ... and every other lane's
          if (!(dsc[s] & kDescValid) || !process(dsc[s], s)) run = false;
        }
      }
    }
    cp_async_wait<0>();  // no copy into shared memory outlives the CTA
    // every B slab this pair requested has landed before shared memory is
    // released (its last step's full barrier phase completed, or the wait ran
    // out of budget)
    if (h == 0 && lane == 0 && pj > 0) mbar_wait_drain(&full[pair], static_cast<uint32_t>((pj - 1) & 1), budget, p.status);
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
  constexpr int ND = Bufs<N_MMA>::value;
  using Cf = Cfg<N_MMA, ND>;
  EncodeTiledFn encode = get_encode_tiled();
  if (!encode) return FLASHSPMM_ERR_CUDA;
  // B (K x N column-major, i.e. N rows of K) as a 2-D tensor; one request
  // loads one 64-wide K tile of N_MMA rows, and elements past K or N read as
  // zero.
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTile), static_cast<cuuint32_t>(N_MMA)};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult rc = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(B), dims, strides, box,
                             estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (rc != CUDA_SUCCESS) return FLASHSPMM_ERR_CUDA;

  auto kernel = spmm_lscd_sm100_kernel<N_MMA, ND>;
  static std::atomic<uint64_t> attr_set_mask{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLASHSPMM_ERR_CUDA;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(attr_set_mask.load() & bit)) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kSmemBytes) != cudaSuccess)
      return FLASHSPMM_ERR_CUDA;
    attr_set_mask.fetch_or(bit);
  }

  SpmmParams p{};
  p.tile_offsets = A->tile_offsets;
  p.words = A->words;
  p.nwords = A->nwords;
  p.C = static_cast<__half*>(C);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.partials = plan.partial_bytes ? reinterpret_cast<float*>(ws + plan.partial_offset) : nullptr;
  p.counters = plan.counter_bytes ? reinterpret_cast<int32_t*>(ws + plan.counter_offset) : nullptr;
  p.M = M; p.K = K; p.N = N;
  p.TM = plan.TM; p.TK = plan.TK; p.U = plan.U; p.T = plan.T;
  p.mode = plan.mode; p.split = plan.split; p.num_pieces = plan.num_pieces;
  p.timeout_ns = 1000000000ull;  // 1 s: far above any legitimate wait
  p.status = device_status_ptr();

  // The arrival counters must start at zero.  Counters in the fixed region at
  // the start of the workspace are left zero by every completed call (the
  // last arriver resets its own); the rare plans whose counters do not fit
  // there keep them after the partial sums and clear them here.
  if (plan.counters_cleared && cudaMemsetAsync(p.counters, 0, plan.counter_bytes, s) != cudaSuccess)
    return FLASHSPMM_ERR_CUDA;

  // Programmatic stream serialisation: this kernel's prologue (barrier init,
  // tensor-memory allocation) may overlap the tail of the previous kernel in
  // the stream; the kernel reads no global memory before griddepcontrol.wait.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.num_pieces));
  cfg.blockDim = dim3(Cf::kThreads);
  cfg.dynamicSmemBytes = Cf::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, tmap, p);
  note_launch();
  return err == cudaSuccess ? FLASHSPMM_OK : FLASHSPMM_ERR_CUDA;
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
    // Partial sums exist only if some piece boundary cuts a unit; the kernel
    // touches the workspace only for such shared units.
    bool shared = false;
    for (int64_t pc = 1; pc < pl.num_pieces && !shared; ++pc) shared = (pc * pl.T / pl.num_pieces) % pl.TK != 0;
    pl.partial_slots = shared ? 2 * static_cast<int64_t>(pl.num_pieces) : 0;
  } else {
    pl.mode = 1;
    pl.split = split_k < pl.TK ? split_k : pl.TK;
    pl.num_pieces = static_cast<int32_t>(static_cast<int64_t>(pl.U) * pl.split);
    pl.partial_slots = pl.split > 1 ? pl.num_pieces : 0;
  }
  // counters: mode 0 indexes them by the first piece of a shared unit (unique
  // per shared unit, at most one per CTA), mode 1 by unit
  pl.counters = pl.partial_slots ? (pl.mode == 0 ? pl.num_pieces : pl.U) : 0;
  pl.partial_bytes = align256(static_cast<size_t>(pl.partial_slots) * kUnitRows * N * sizeof(float));
  if (pl.partial_slots == 0) {
    pl.workspace_bytes = 0;
    return pl;
  }
  pl.partial_offset = kCounterRegionBytes;
  pl.counters_cleared = pl.counters > kCounterRegionSlots;
  pl.counter_offset = pl.counters_cleared ? pl.partial_offset + pl.partial_bytes : 0;
  pl.counter_bytes = pl.counters_cleared ? align256(static_cast<size_t>(pl.counters) * sizeof(int32_t))
                                         : kCounterRegionBytes;
  pl.workspace_bytes = pl.partial_offset + pl.partial_bytes + (pl.counters_cleared ? pl.counter_bytes : 0);
  return pl;
}

// The plan fields the kernel's partition helpers read, filled on the host.
static SpmmParams plan_params(const SpmmPlan& pl) {
  SpmmParams p{};
  p.TM = pl.TM; p.TK = pl.TK; p.U = pl.U; p.T = pl.T;
  p.mode = pl.mode; p.split = pl.split; p.num_pieces = pl.num_pieces;
  return p;
}

static bool plan_args_ok(int32_t M, int32_t K, int32_t N, int32_t num_sms) {
  return M > 0 && K > 0 && N > 0 && N <= 256 && num_sms > 0;
}

flashspmm_status launch_spmm_lscd(const flashspmm_tcsl* A, const void* B, void* C, int32_t M, int32_t K,
                                  int32_t N, const SpmmPlan& plan, void* workspace, cudaStream_t s) {
  if (static_cast<int64_t>(plan.TK) > kMaxKTiles) return FLASHSPMM_ERR_UNSUPPORTED;
  if (N <= 16) return launch_bucket<16>(A, B, C, M, K, N, plan, workspace, s);
  if (N <= 32) return launch_bucket<32>(A, B, C, M, K, N, plan, workspace, s);
  if (N <= 64) return launch_bucket<64>(A, B, C, M, K, N, plan, workspace, s);
  if (N <= 128) return launch_bucket<128>(A, B, C, M, K, N, plan, workspace, s);
  return launch_bucket<256>(A, B, C, M, K, N, plan, workspace, s);
}

}  // namespace flashspmm

using flashspmm::make_spmm_plan;

extern "C" int flashspmm_plan_query(int32_t M, int32_t K, int32_t N, int32_t split_k, int32_t num_sms, int64_t* info,
                                    int64_t* ranges) {
  if (!flashspmm::plan_args_ok(M, K, N, num_sms) || !info) return -1;
  const flashspmm::SpmmPlan pl = make_spmm_plan(M, K, N, split_k, num_sms);
  const int64_t vals[9] = {pl.TM, pl.TK, pl.U, pl.T, pl.mode, pl.split, pl.num_pieces, pl.partial_slots,
                           static_cast<int64_t>(pl.workspace_bytes)};
  for (int i = 0; i < 9; ++i) info[i] = vals[i];
  if (ranges) {
    const flashspmm::SpmmParams p = flashspmm::plan_params(pl);
    for (int64_t pc = 0; pc < pl.num_pieces; ++pc) {
      const flashspmm::Range r = flashspmm::piece_range(p, pc);
      ranges[2 * pc] = r.b;
      ranges[2 * pc + 1] = r.e;
    }
  }
  return 0;
}

extern "C" int64_t flashspmm_plan_owner(int32_t M, int32_t K, int32_t N, int32_t split_k, int32_t num_sms,
                                        int64_t q) {
  if (!flashspmm::plan_args_ok(M, K, N, num_sms)) return -1;
  const flashspmm::SpmmPlan pl = make_spmm_plan(M, K, N, split_k, num_sms);
  if (pl.mode != 0 || q < 0 || q >= pl.T) return -1;
  return flashspmm::piece_of_step(flashspmm::plan_params(pl), q);
}

extern "C" int64_t flashspmm_plan_slot(int32_t M, int32_t K, int32_t N, int32_t split_k, int32_t num_sms,
                                       int64_t pc, int64_t u) {
  if (!flashspmm::plan_args_ok(M, K, N, num_sms)) return -1;
  const flashspmm::SpmmPlan pl = make_spmm_plan(M, K, N, split_k, num_sms);
  if (pc < 0 || pc >= pl.num_pieces || u < 0 || u >= pl.U || pl.partial_slots == 0) return -1;
  return flashspmm::partial_slot(flashspmm::plan_params(pl), pc, u);
}
