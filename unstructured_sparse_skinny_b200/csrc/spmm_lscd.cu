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
//   gmem2reg  -> 8 decompress warps stream their tiles' word lists from HBM
//                straight into registers (coalesced 32-bit loads, L1
//                bypassed, L2 evict-first), one round (1024 words, or 512
//                for very sparse matrices) always in flight per warp while
//                the previous round is expanded;
//   rst_smem  -> each warp zeroes its half (64 rows) of a 128 x 64 dense A
//   + extract    buffer with 16-byte stores and scatters every word's value
//                to its swizzled position (UMMA K-major 128-byte layout);
//   ld_dense  -> warp 1 loads B slabs (64 K x N_MMA) with TMA tensor copies in
//                the same swizzled layout, several K tiles per request;
//   smem2tc   -> gone: tcgen05.mma reads both operands from shared memory;
//   TC_compute-> warp 0 issues 4 x tcgen05.mma (M = 128, K = 16) per step into
//                a double-buffered fp32 accumulator in tensor memory;
//   epilogue  -> 4 warps read the accumulator with tcgen05.ld and write fp16 C
//                (or fp32 partial sums, see below).
//
// A "unit" is 128 rows of A (two 64-row format strips stacked on the MMA M
// side); a "step" is one 64-wide K tile of one unit, expanded by a pair of
// decompress warps (one per strip) into a dense buffer.  The CTA's steps are
// taken in groups of 4; pair p expands step p of every group, and the groups
// alternate between two sets of 4 dense buffers.  A group costs one mbarrier
// hand-off (8 arrivals) to the MMA warp and one commit back, which the MMA
// warp answers with 16 MMAs: per-step synchronisation, not data, is what
// limits a skinny SpMM, so it is paid once per group.
//
// The T = units x K-tiles steps are cut into contiguous pieces, one CTA each.
// When a unit is shared by several pieces, every piece writes its fp32
// partial sum to the workspace and the last piece to finish (atomic arrival
// counter) adds them in piece order and writes C: the split-K reduction of the
// page's Reduction kernel (section 5, "project structure"), fused and
// deterministic.  The last piece also resets the unit's arrival counter.
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
constexpr int kDenseBytes = kUnitRows * kTile * 2;  // 16 KB dense A buffer
constexpr int kHalfBytes = kDenseBytes / 2;         // one strip's 64 rows
constexpr int kMaxTileWords = kTile * kTile;        // 4096 words (already a multiple of 4)
constexpr int kWarpMma = 0, kWarpB = 1, kWarpEpi = 2, kWarpDec = 6;
constexpr int kDecWarps = 8;                        // 4 pairs, one warp per strip
constexpr int kPairs = kDecWarps / 2;
constexpr int kThreads = (kWarpDec + kDecWarps) * 32;
constexpr int kEpiThreads = 128;
constexpr int kNumDense = 2 * kPairs;               // two sets of one buffer per pair
constexpr int kBarEpi = 1;                          // named barrier id of the epilogue warps
// Words per lane per load round (a round is 32x that per warp): 32 for most
// matrices, 16 when a tile averages at most kSmallRoundMaxWords words, where
// 32-word rounds would be mostly sentinel slots that still cost instructions.
constexpr int kRoundRegsLarge = 32, kRoundRegsSmall = 16;
constexpr int kSmallRoundMaxWords = 448;
constexpr int kMinStepsPerPiece = 4;
constexpr int kTableBytes = (kMaxTablePieces + 1) * 8;  // a CTA's checked copy of the piece table


template <int N_MMA>
struct Cfg {
  static_assert(N_MMA == 16 || N_MMA == 32 || N_MMA == 64 || N_MMA == 128 || N_MMA == 256, "N bucket");
  static constexpr int kBSlabBytes = N_MMA * kTile * 2;  // one 64-wide K tile of B
  static constexpr int kSlabsPerReq = kBSlabBytes >= 16384 ? 1 : 16384 / kBSlabBytes;  // K tiles per TMA request
  static constexpr int kReqBytes = kSlabsPerReq * kBSlabBytes;
  static constexpr int kNumReq = N_MMA <= 128 ? 3 : 2;   // B requests in flight
  static constexpr int kTmemCols = 2 * N_MMA < 32 ? 32 : 2 * N_MMA;
  static constexpr uint32_t kIdesc = umma_idesc_f16_f32(kUnitRows, N_MMA);
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int kOffDense = 0;
  static constexpr int kOffB = kOffDense + kNumDense * kDenseBytes;
  static constexpr int kOffBars = kOffB + kNumReq * kReqBytes;
  static constexpr int kNumBars = 2 * 2 + 2 * kNumReq + 4 + 1;
  static constexpr int kOffMisc = kOffBars + kNumBars * 8;
  static constexpr int kOffTable = kOffMisc + 64;  // piece-table copy (table instances only)
  static constexpr int kSmemBytes = kOffTable + 1024;                 // + alignment slack
  static constexpr int kSmemBytesTable = kOffTable + kTableBytes + 1024;
  static_assert(kSmemBytesTable <= 232448, "shared memory budget");
};

struct SpmmParams {
  const int32_t* tile_offsets;
  const uint32_t* words;
  int64_t nwords;
  void* C;           // fp16, or fp32 when c_f32
  float* partials;    // [slot][N][128]
  int32_t* counters;  // mode 0: one per piece (the first piece of a shared unit); mode 1: one per unit
  int32_t M, K, N;
  int32_t TM, TK, U;
  int64_t T;
  int32_t mode, split, num_pieces;
  int32_t b_kb;    // K tiles of B per TMA request (1 with the 2-D map)
  int32_t b_3d;    // B tensor map is 3-D (64 x N x K/64)
  uint64_t timeout_ns;
  int* status;
  const int64_t* bounds;  // word-balanced piece table (mode 0), or null for even pieces
  int64_t ld;             // tile_offsets entries between consecutive strips
  int32_t c_f32;          // C holds fp32 instead of fp16
};

struct Range {
  int64_t b, e;
};

// First step of piece pc.  `tab` is the CTA's checked copy of a word-balanced
// piece table (mode 0 only), or null for the closed forms: even pieces of the
// whole step space (mode 0) or split equal K-chunks per unit (mode 1).
__host__ __device__ __forceinline__ int64_t piece_begin(const SpmmParams& p, const int64_t* tab, int64_t pc) {
  if (p.mode == 0) return tab ? tab[pc] : pc * p.T / p.num_pieces;
  const int64_t u = pc / p.split, c = pc - (pc / p.split) * p.split;
  return u * p.TK + c * p.TK / p.split;
}

__host__ __device__ __forceinline__ Range piece_range(const SpmmParams& p, const int64_t* tab, int64_t pc) {
  return {piece_begin(p, tab, pc), piece_begin(p, tab, pc + 1)};
}

// Piece that owns step q in mode 0: the largest pc with piece_begin(pc) <= q.
__host__ __device__ __forceinline__ int64_t piece_of_step(const SpmmParams& p, const int64_t* tab, int64_t q) {
  if (!tab) return ((q + 1) * p.num_pieces + p.T - 1) / p.T - 1;
  int64_t lo = 0, hi = p.num_pieces - 1;  // tab[0] = 0 <= q
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) >> 1;
    if (tab[mid] <= q) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Workspace slot of piece pc's partial sum for unit u: in mode 0 a piece has
// two, one for the unit it starts in and one for the unit it ends in (the
// units in between are whole and never shared).
__host__ __device__ __forceinline__ int64_t partial_slot(const SpmmParams& p, const int64_t* tab, int64_t pc,
                                                         int64_t u) {
  if (p.mode == 1) return pc;
  return 2 * pc + ((piece_begin(p, tab, pc) / p.TK) != u ? 1 : 0);
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

// Word `slot` of this lane in a load round, or the sentinel when the slot is
// past the lane's `nvalid` words (the address is then not dereferenced).
// Read-only path, no L1 allocation, evict-first in L2: every word is used
// exactly once.
__device__ __forceinline__ uint32_t ldg_word(const uint32_t* ptr, int slot, int nvalid, uint64_t policy) {
  uint32_t v = kSentinel;
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.lt.s32 q, %2, %3;\n\t"
      "@q ld.global.nc.L1::no_allocate.L2::cache_hint.b32 %0, [%1], %4;\n\t}"
      : "+r"(v)
      : "l"(ptr), "r"(slot), "r"(nvalid), "l"(policy));
  return v;
}

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

// One element of C: fp16 (round to nearest even), or the fp32 accumulator.
__device__ __forceinline__ void store_c(const SpmmParams& p, int64_t idx, float x) {
  if (p.c_f32) static_cast<float*>(p.C)[idx] = x;
  else static_cast<__half*>(p.C)[idx] = __float2half_rn(x);
}

// A load round of a decompress warp: words [base, end) of one strip tile,
// at most 32 * RR of them.
struct Round {
  int k;      // index of the step among the warp's steps
  bool first, last, valid;
};

// kTable: the instance that takes its pieces from a word-balanced table (the
// plain instance has none of that code and none of its shared memory).
template <int N_MMA, int RR, bool kTable>
__global__ void __launch_bounds__(kThreads, 1)
    spmm_lscd_sm100_kernel(const __grid_constant__ CUtensorMap tmap_b, const SpmmParams p) {
  using Cf = Cfg<N_MMA>;
  constexpr int kRoundRegs = RR;
  constexpr int kRoundWords = RR * 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* dense = smem + Cf::kOffDense;
  uint8_t* bslab = smem + Cf::kOffB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::kOffBars);
  uint64_t* a_full = bars;          // [2]: buffer set filled (8 arrivals)
  uint64_t* a_empty = a_full + 2;   // [2]: buffer set consumed (one commit)
  uint64_t* b_full = a_empty + 2;
  uint64_t* b_empty = b_full + Cf::kNumReq;
  uint64_t* acc_full = b_empty + Cf::kNumReq;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cf::kOffMisc + 4);
  volatile int* epi_last = reinterpret_cast<volatile int*>(smem + Cf::kOffMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t budget = p.timeout_ns;
  Range rg = piece_range(p, nullptr, blockIdx.x);  // even pieces (closed form; replaced by a table's below)

  griddep_launch_dependents();
  if (warp == kWarpB) {
    if (lane < 2) {
      mbar_init(&a_full[lane], kDecWarps);  // every decompress warp, once per group
      mbar_init(&a_empty[lane], 1);
    }
    if (lane < Cf::kNumReq) {
      mbar_init(&b_full[lane], 1);
      mbar_init(&b_empty[lane], 1);
    }
    if (lane < 2) {
      mbar_init(&acc_full[lane], 1);
      mbar_init(&acc_empty[lane], 1);
    }
    if (lane == 0) {
      mbar_init(mma_done, 1);
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

  // A word-balanced piece table is copied whole into every CTA and checked
  // there (strictly increasing from 0 to T), so all CTAs take the same
  // decision: the table's pieces, or even pieces when it is malformed.
  const int64_t* tab = nullptr;
  if (kTable && p.bounds) {
    int64_t* st = reinterpret_cast<int64_t*>(smem + Cf::kOffTable);
    const int np = p.num_pieces;  // <= kMaxTablePieces (checked on the host)
    for (int i = threadIdx.x; i <= np; i += kThreads) st[i] = __ldg(p.bounds + i);
    __syncthreads();
    bool bad = false;
    for (int i = threadIdx.x; i <= np; i += kThreads) {
      bad |= i == 0 ? st[0] != 0 : st[i] <= st[i - 1];
      if (i == np) bad |= st[np] != p.T;
    }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0 && blockIdx.x == 0) record_status(p.status, FLASHSPMM_ERR_CORRUPT_FORMAT);
    } else {
      tab = st;
      rg = piece_range(p, tab, blockIdx.x);
    }
  }

  if (warp == kWarpB) {
    // ------------------------------------------------ dense B producer (TMA)
    // A request loads b_kb consecutive 64-wide K tiles of B (one group); the
    // requests of the piece are the (unit, group) pairs it touches, and lane r
    // issues every kNumReq-th request into request slot r.
    if (lane < Cf::kNumReq) {
      const int kb = p.b_kb;
      const int ngroups = (p.TK + kb - 1) / kb;
      int64_t u = rg.b / p.TK;
      int g = static_cast<int>(rg.b - u * p.TK) / kb;
      int64_t k = 0, uses = 0;
      while (u * p.TK + static_cast<int64_t>(g) * kb < rg.e) {
        if (static_cast<int>(k % Cf::kNumReq) == lane) {
          if (!mbar_wait(&b_empty[lane], static_cast<uint32_t>((uses & 1) ^ 1), abort_flag, budget, p.status)) break;
          mbar_arrive_expect_tx(&b_full[lane], static_cast<uint32_t>(kb * Cf::kBSlabBytes));
          uint8_t* dst = bslab + lane * Cf::kReqBytes;
          if (p.b_3d) tma_load_3d(dst, &tmap_b, 0, 0, g * kb, &b_full[lane]);
          else tma_load_2d(dst, &tmap_b, g * kTile, 0, &b_full[lane]);
          ++uses;
        }
        ++k;
        if (++g == ngroups) { g = 0; ++u; }
      }
      // every issued copy lands before the CTA's shared memory is released
      if (uses > 0) mbar_wait_drain(&b_full[lane], static_cast<uint32_t>((uses - 1) & 1), budget, p.status);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------ tcgen05 MMA issuer
    // The whole warp runs one uniform loop, one group of up to 4 steps per
    // iteration; every lane tests the barriers itself (so no broadcast is
    // needed) and one elected lane issues the MMAs and commits (issue from a
    // converged warp is markedly cheaper than from a lone divergent thread).
    // Before a step that starts a B request or an accumulator the warp waits
    // for that too, never earlier: a request slot or accumulator may only be
    // freed by this group's own earlier MMAs.  Step bookkeeping is kept in
    // 32-bit counters: this loop is latency-bound, one iteration per group.
    const int kb = p.b_kb;
    int nleft = static_cast<int>(rg.e - rg.b);        // steps left in the piece
    int to_unit = p.TK - static_cast<int>(rg.b % p.TK);  // steps left in the current unit
    int jk = (p.TK - to_unit) % kb;                   // slab of the current step in its B request
    bool pfirst = true;
    int r = Cf::kNumReq - 1;  // B request slot of the current step
    uint32_t rph = 1;         // its phase parity (flips when the slot index wraps to 0)
    int ac = 0;               // accumulator of the current unit
    uint32_t acph = 1;        // parity to wait on acc_empty[ac]
    const uint32_t a_base = smem_u32(dense);
    const uint32_t b_base = smem_u32(bslab);
    bool issued = false, dead = false;
    for (int64_t k = 0; nleft > 0 && !dead; ++k) {
      const int set = static_cast<int>(k & 1);
      if (!mbar_wait(&a_full[set], static_cast<uint32_t>((k >> 1) & 1), abort_flag, budget, p.status)) break;
      const bool leader = elect_one();
      const int gsteps = nleft < kPairs ? nleft : kPairs;
#pragma unroll
      for (int i = 0; i < kPairs; ++i) {
        if (i >= gsteps) break;
        const bool first = pfirst || to_unit == p.TK;
        const bool last = nleft == 1 || to_unit == 1;
        const bool new_req = pfirst || jk == 0;
        if (new_req) {
          if (++r == Cf::kNumReq) { r = 0; rph ^= 1u; }
          if (!mbar_wait(&b_full[r], rph, abort_flag, budget, p.status)) { dead = true; break; }
        }
        if (first) {
          if (!mbar_wait(&acc_empty[ac], acph, abort_flag, budget, p.status)) { dead = true; break; }
          tc_fence_after_sync();  // accumulator handed back by the epilogue's tcgen05.ld
        }
        const uint64_t adesc = smem_desc_k_sw128(a_base + static_cast<uint32_t>((i + kPairs * set) * kDenseBytes));
        const uint64_t bdesc =
            smem_desc_k_sw128(b_base + static_cast<uint32_t>(r * Cf::kReqBytes + jk * Cf::kBSlabBytes));
        const uint32_t tmem_d = tmem_base + static_cast<uint32_t>(ac * N_MMA);
        uint64_t ad[kTile / 16], bd[kTile / 16];  // K = 16 per MMA: advance 32 bytes inside the swizzle atom
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) { ad[kk] = adesc + 2 * kk; bd[kk] = bdesc + 2 * kk; }
        const uint32_t acc0 = first ? 0u : 1u;
        if (leader) {
          umma_f16_ss(tmem_d, ad[0], bd[0], Cf::kIdesc, acc0);
#pragma unroll
          for (int kk = 1; kk < kTile / 16; ++kk) umma_f16_ss(tmem_d, ad[kk], bd[kk], Cf::kIdesc, 1u);
          if (jk == kb - 1 || last) umma_commit(&b_empty[r]);  // request fully used
          if (last) umma_commit(&acc_full[ac]);
        }
        issued = true;
        pfirst = false;
        --nleft;
        if (last) {
          if (ac == 1) acph ^= 1u;
          ac ^= 1;
        }
        if (--to_unit == 0) {
          to_unit = p.TK;
          jk = 0;
        } else if (++jk == kb) {
          jk = 0;
        }
      }
      if (dead) break;
      if (leader) umma_commit(&a_empty[set]);
      __syncwarp();
    }
    if (issued) {  // all MMAs retired before tensor memory is released
      if (elect_one()) umma_commit(mma_done);
      __syncwarp();
      if (lane == 0) mbar_wait_drain(mma_done, 0, budget, p.status);
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
      bool ok = true;
      if (etid == 0) ok = mbar_wait(&acc_full[ab], static_cast<uint32_t>((uc >> 1) & 1), abort_flag, budget, p.status);
      if (named_barrier_or(kBarEpi, kEpiThreads, !ok)) break;  // the other threads sleep here
      tc_fence_after_sync();
      const int64_t seg_b = max64(rg.b, u * p.TK), seg_e = min64(rg.e, (u + 1) * p.TK);
      const bool complete = seg_b == u * p.TK && seg_e == (u + 1) * p.TK;
      const int64_t m = u * kUnitRows + row;
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(ab * N_MMA);
      float* part = nullptr;
      if (!complete) part = p.partials + partial_slot(p, tab, blockIdx.x, u) * static_cast<int64_t>(p.N) * kUnitRows;
#pragma unroll 1
      for (int c = 0; c < N_MMA && c < p.N; c += 16) {
        uint32_t v[16];
        tmem_load_16(taddr + c, v);
        tmem_load_wait();
        if (!complete) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c + i < p.N) part[static_cast<int64_t>(c + i) * kUnitRows + row] = __uint_as_float(v[i]);
        } else if (m < p.M) {
          if (p.c_f32) {
            float* cc = static_cast<float*>(p.C) + m;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c + i < p.N) cc[static_cast<int64_t>(c + i) * p.M] = __uint_as_float(v[i]);
          } else {
            __half* cc = static_cast<__half*>(p.C) + m;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c + i < p.N) cc[static_cast<int64_t>(c + i) * p.M] = __float2half_rn(__uint_as_float(v[i]));
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
          first_pc = piece_of_step(p, tab, u * p.TK);
          ncontrib = piece_of_step(p, tab, u * p.TK + p.TK - 1) - first_pc + 1;
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
          for (int nc = 0; nc < p.N; nc += 16) {
            float acc[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
#pragma unroll 1
            for (int64_t k = 0; k < ncontrib; ++k) {
              const float* src = p.partials + (partial_slot(p, tab, first_pc + k, u) * p.N + nc) * kUnitRows + row;
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (nc + i < p.N) acc[i] += __ldcg(src + i * kUnitRows);
            }
            if (m < p.M) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (nc + i < p.N) store_c(p, static_cast<int64_t>(nc + i) * p.M + m, acc[i]);
            }
          }
          if (etid == 0) *counter = 0;  // zero again for the next call
        }
        named_barrier(kBarEpi, kEpiThreads);
      }
    }
  } else {
    // ------------------------------------------------ decompress (gmem2reg + rst_smem + extract)
    // Warp (pair, h) expands strip h of step `pair` of every group, i.e. the
    // steps pair, pair + 4, ... of the piece, into buffer pair of the group's
    // buffer set.  Its word lists are streamed in rounds of up to 32 * RR words
    // (RR per lane, consecutive words on consecutive lanes); the loads of the next
    // round are issued before the current round is expanded, so one round is
    // always in flight.  The first round of a step waits until the MMAs of
    // the buffer's previous step have retired and zeroes the warp's half of
    // the buffer; the last round publishes the half to the MMA warp.
    const int dw = warp - kWarpDec;
    const int pair = dw >> 1, h = dw & 1;
    const int64_t piece_steps = rg.e - rg.b;
    const int64_t my_steps = piece_steps > pair ? (piece_steps - pair + kPairs - 1) / kPairs : 0;
    const uint64_t policy = l2_policy_evict_first();
    // Tile offsets of 32 consecutive steps of this warp, one step per lane:
    // the current table (validated) and the next one (loads in flight).
    auto load_tab = [&](int64_t k0, int32_t& ta, int32_t& tb) {
      ta = 0;
      tb = 0;
      const int64_t k = k0 + lane;
      if (k < my_steps) {
        const int64_t q = rg.b + pair + k * kPairs;
        const int64_t u = q / p.TK, j = q - (q / p.TK) * p.TK;
        const int64_t strip = 2 * u + h;
        if (strip < p.TM) {
          const int64_t t = strip * p.ld + j;
          ta = __ldg(p.tile_offsets + t);
          tb = __ldg(p.tile_offsets + t + 1);
        }
      }
    };
    auto validate = [&](int32_t& ta, int32_t& tb) {
      const int32_t n = tb - ta;
      const bool ok = ta >= 0 && n >= 0 && !(ta & 3) && !(n & 3) && n <= kMaxTileWords && tb <= p.nwords;
      if (!ok) {
        record_status(p.status, FLASHSPMM_ERR_CORRUPT_FORMAT);
        ta = 0;
        tb = 0;
      }
    };
    int32_t ca, cb, na, nb;
    int tab_base = 0, ik = 0;  // steps of this warp: at most a piece's steps, far below 2^31
    uint32_t ipos = 0;
    const int my_steps32 = static_cast<int>(my_steps);
    load_tab(0, ca, cb);
    load_tab(32, na, nb);
    validate(ca, cb);
    auto issue = [&](uint32_t (&v)[kRoundRegs], Round& rd) {
      rd.valid = ik < my_steps32;
      if (!rd.valid) return;
      if (ik - tab_base == 32) {
        tab_base += 32;
        ca = na;
        cb = nb;
        validate(ca, cb);
        load_tab(tab_base + 32, na, nb);
      }
      const int li = ik - tab_base;
      const uint32_t a0 = static_cast<uint32_t>(__shfl_sync(0xFFFFFFFFu, ca, li));
      const uint32_t a1 = static_cast<uint32_t>(__shfl_sync(0xFFFFFFFFu, cb, li));
      const uint32_t base = a0 + ipos;
      const int rem = min(static_cast<int>(a1 - base), kRoundWords);
      rd.k = ik;
      rd.first = ipos == 0;
      rd.last = base + kRoundWords >= a1;
      // lane l holds words base + l + 32 i, i < nvalid
      const int nvalid = rem > lane ? (rem - lane + 31) >> 5 : 0;
      const uint32_t* src = p.words + base + lane;
#pragma unroll
      for (int i = 0; i < kRoundRegs; ++i) v[i] = ldg_word(src + 32 * i, i, nvalid, policy);
      if (rd.last) {
        ++ik;
        ipos = 0;
      } else {
        ipos += kRoundWords;
      }
    };
    // Buffer set k & 1 is free once the MMAs of group k - 2 have retired.
    auto wait_set = [&](int k) -> bool {  // every lane tests the barrier: no broadcast needed
      return mbar_wait(&a_empty[k & 1], static_cast<uint32_t>(((k >> 1) & 1) ^ 1), abort_flag, budget, p.status);
    };
    auto process = [&](const uint32_t (&v)[kRoundRegs], const Round& rd) -> bool {
      const int set = static_cast<int>(rd.k & 1);
      uint8_t* half = dense + (pair + kPairs * set) * kDenseBytes + h * kHalfBytes;
      if (rd.first) {
        if (!wait_set(rd.k)) return false;
        uint4* dz = reinterpret_cast<uint4*>(half);
#pragma unroll
        for (int i = 0; i < kHalfBytes / 16 / 32; ++i) dz[i * 32 + lane] = make_uint4(0, 0, 0, 0);
        __syncwarp();
      }
      const uint32_t hb = smem_u32(half);
#pragma unroll
      for (int i = 0; i < kRoundRegs; ++i) scatter_word(hb, v[i]);
      if (rd.last) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[set]);
      }
      return true;
    };
    uint32_t va[kRoundRegs], vb[kRoundRegs];
    Round ra, rb;
    bool ok = true;
    issue(va, ra);
    while (ra.valid) {
      issue(vb, rb);
      if (!(ok = process(va, ra)) || !rb.valid) break;
      issue(va, ra);
      if (!(ok = process(vb, rb))) break;
    }
    // A pair without a step in the piece's last (partial) group still
    // completes that group's arrival count, once the set is free (so the
    // arrival cannot count towards the set's previous group).
    const int64_t ngroups = (piece_steps + kPairs - 1) / kPairs;
    if (ok && my_steps < ngroups && wait_set(my_steps32)) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[my_steps32 & 1]);
    }
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
flashspmm_status launch_bucket(const flashspmm_tcsl* A, const void* B, void* C, bool c_f32, int32_t M, int32_t K,
                               int32_t N, const SpmmPlan& plan, void* workspace, cudaStream_t s) {
  using Cf = Cfg<N_MMA>;
  EncodeTiledFn encode = get_encode_tiled();
  if (!encode) return FLASHSPMM_ERR_CUDA;
  // B as a 3-D tensor (64 x N x K/64) lets one TMA request load several
  // consecutive K tiles; a ragged K keeps the 2-D map (one tile per request)
  // so no box element can fall past the end of B.
  const int TK = (K + kTile - 1) / kTile;
  const bool b3d = (K % kTile == 0) && Cf::kSlabsPerReq > 1 && TK >= Cf::kSlabsPerReq;
  CUtensorMap tmap;
  CUresult rc;
  if (b3d) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kTile), static_cast<cuuint64_t>(N),
                                static_cast<cuuint64_t>(TK)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, static_cast<cuuint64_t>(kTile) * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kTile), static_cast<cuuint32_t>(N_MMA),
                               static_cast<cuuint32_t>(Cf::kSlabsPerReq)};
    const cuuint32_t estride[3] = {1, 1, 1};
    rc = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(B), dims, strides, box, estride,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTile), static_cast<cuuint32_t>(N_MMA)};
    const cuuint32_t estride[2] = {1, 1};
    rc = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(B), dims, strides, box, estride,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (rc != CUDA_SUCCESS) return FLASHSPMM_ERR_CUDA;

  static std::atomic<uint64_t> attr_set_mask{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLASHSPMM_ERR_CUDA;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(attr_set_mask.load() & bit)) {
    if (cudaFuncSetAttribute(spmm_lscd_sm100_kernel<N_MMA, kRoundRegsLarge, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(spmm_lscd_sm100_kernel<N_MMA, kRoundRegsSmall, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(spmm_lscd_sm100_kernel<N_MMA, kRoundRegsLarge, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kSmemBytesTable) != cudaSuccess ||
        cudaFuncSetAttribute(spmm_lscd_sm100_kernel<N_MMA, kRoundRegsSmall, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kSmemBytesTable) != cudaSuccess)
      return FLASHSPMM_ERR_CUDA;
    attr_set_mask.fetch_or(bit);
  }
  const int64_t num_tiles = static_cast<int64_t>(plan.TM) * plan.TK;
  const bool small_rounds = num_tiles > 0 && A->nwords <= static_cast<int64_t>(kSmallRoundMaxWords) * num_tiles;

  SpmmParams p{};
  p.tile_offsets = A->tile_offsets;
  p.words = A->words;
  p.nwords = A->nwords;
  p.C = C;
  p.c_f32 = c_f32 ? 1 : 0;
  p.bounds = plan.table ? A->piece_bounds : nullptr;
  p.ld = A->offsets_ld > 0 ? A->offsets_ld : plan.TK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.partials = plan.partial_bytes ? reinterpret_cast<float*>(ws + plan.partial_offset) : nullptr;
  p.counters = plan.counter_bytes ? reinterpret_cast<int32_t*>(ws + plan.counter_offset) : nullptr;
  p.M = M; p.K = K; p.N = N;
  p.TM = plan.TM; p.TK = plan.TK; p.U = plan.U; p.T = plan.T;
  p.mode = plan.mode; p.split = plan.split; p.num_pieces = plan.num_pieces;
  p.b_kb = b3d ? Cf::kSlabsPerReq : 1;
  p.b_3d = b3d ? 1 : 0;
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
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = plan.table ? Cf::kSmemBytesTable : Cf::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err;
  if (plan.table)
    err = small_rounds ? cudaLaunchKernelEx(&cfg, spmm_lscd_sm100_kernel<N_MMA, kRoundRegsSmall, true>, tmap, p)
                       : cudaLaunchKernelEx(&cfg, spmm_lscd_sm100_kernel<N_MMA, kRoundRegsLarge, true>, tmap, p);
  else
    err = small_rounds ? cudaLaunchKernelEx(&cfg, spmm_lscd_sm100_kernel<N_MMA, kRoundRegsSmall, false>, tmap, p)
                       : cudaLaunchKernelEx(&cfg, spmm_lscd_sm100_kernel<N_MMA, kRoundRegsLarge, false>, tmap, p);
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

SpmmPlan make_spmm_plan(int32_t M, int32_t K, int32_t N, int32_t split_k, int num_sms, bool table) {
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
    // touches the workspace only for such shared units.  A piece table's
    // boundaries are known only on the device, so it may cut any unit.
    pl.table = table && pl.num_pieces <= kMaxTablePieces;
    bool shared = pl.table && pl.num_pieces > 1;
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

flashspmm_status launch_spmm_lscd(const flashspmm_tcsl* A, const void* B, void* C, bool c_f32, int32_t M,
                                  int32_t K, int32_t N, const SpmmPlan& plan, void* workspace, cudaStream_t s) {
  if (N <= 16) return launch_bucket<16>(A, B, C, c_f32, M, K, N, plan, workspace, s);
  if (N <= 32) return launch_bucket<32>(A, B, C, c_f32, M, K, N, plan, workspace, s);
  if (N <= 64) return launch_bucket<64>(A, B, C, c_f32, M, K, N, plan, workspace, s);
  if (N <= 128) return launch_bucket<128>(A, B, C, c_f32, M, K, N, plan, workspace, s);
  return launch_bucket<256>(A, B, C, c_f32, M, K, N, plan, workspace, s);
}

}  // namespace flashspmm

using flashspmm::make_spmm_plan;

// Dense/sparse choice (the page's integration picks dense or sparse per MatMul
// through its GEMM wrapper; "N dimension" study: sparse wins for skinny N).
// Per-call time models fitted to this library's kernel and to dense cuBLAS
// fp16 GEMMs of the same shapes on B200 (inputs in HBM, CUDA-graph launches,
// 12288^2 at 50-95 % zeros x N 8-128 and the OPT-66B / OPT-175B layers):
//   sparse(us) = 26.97 + 0.085 s + 0.0415 s (N_MMA / 16) + 0.030 w
//     s = steps per CTA of the automatic plan, w = KB of words per CTA;
//   dense(us)  = 5.47 + 153.2 x (2 M K bytes in GB)   (about 6.5 TB/s).
// They agree with the measured faster path in 115 of 126 calls; the rest
// are within a few per cent of parity.
static bool predict_us(int32_t M, int32_t K, int32_t N, int64_t nnz, int32_t num_sms, double* t_sparse,
                       double* t_dense) {
  if (M <= 0 || K <= 0 || N <= 0 || N > 256 || nnz < 0 || num_sms <= 0) return false;
  const flashspmm::SpmmPlan pl = make_spmm_plan(M, K, N, 0, num_sms);
  const double s = static_cast<double>(pl.T) / pl.num_pieces;
  const int n_mma = N <= 16 ? 16 : (N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256)));
  const double w_kb = 4.0 * static_cast<double>(nnz) / pl.num_pieces / 1e3;
  *t_sparse = 26.97 + 0.085 * s + 0.0415 * s * (n_mma / 16.0) + 0.030 * w_kb;
  *t_dense = 5.47 + 153.2 * (2.0 * M * static_cast<double>(K) / 1e9);
  return true;
}

extern "C" int flashspmm_predict_us(int32_t M, int32_t K, int32_t N, int64_t nnz, int32_t num_sms, double* t_sparse,
                                    double* t_dense) {
  double a = 0, b = 0;
  if (!predict_us(M, K, N, nnz, num_sms, &a, &b)) return -1;
  if (t_sparse) *t_sparse = a;
  if (t_dense) *t_dense = b;
  return 0;
}

extern "C" int flashspmm_prefer_sparse(int32_t M, int32_t K, int32_t N, int64_t nnz, int32_t num_sms) {
  double a = 0, b = 0;
  if (!predict_us(M, K, N, nnz, num_sms, &a, &b)) return -1;
  return a < b ? 1 : 0;
}

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
      const flashspmm::Range r = flashspmm::piece_range(p, nullptr, pc);
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
  return flashspmm::piece_of_step(flashspmm::plan_params(pl), nullptr, q);
}

extern "C" int64_t flashspmm_plan_slot(int32_t M, int32_t K, int32_t N, int32_t split_k, int32_t num_sms,
                                       int64_t pc, int64_t u) {
  if (!flashspmm::plan_args_ok(M, K, N, num_sms)) return -1;
  const flashspmm::SpmmPlan pl = make_spmm_plan(M, K, N, split_k, num_sms);
  if (pc < 0 || pc >= pl.num_pieces || u < 0 || u >= pl.U || pl.partial_slots == 0) return -1;
  return flashspmm::partial_slot(flashspmm::plan_params(pl), nullptr, pc, u);
}
