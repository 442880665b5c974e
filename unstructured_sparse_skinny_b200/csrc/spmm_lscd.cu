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

constexpr int kTile = 64;                           // format tile edge (rows and K)
constexpr int kUnitRows = 128;                      // MMA M
constexpr int kDenseBytes = kUnitRows * kTile * 2;  // 16 KB dense A buffer
constexpr int kMaxTileWords = kTile * kTile;        // 4096 words (already a multiple of 4)
constexpr int kThreads = 480;                       // 15 warps
constexpr int kWarpWords = 0, kWarpB = 1, kWarpMma = 2, kWarpEpi = 3, kWarpDec = 7;
constexpr int kEpiThreads = 128;
constexpr int kGroups = 2;                          // independent decompress groups
constexpr int kGroupWarps = 4, kGroupThreads = kGroupWarps * 32;
constexpr int kNumDenseBufs = 4;                    // step n uses dense buffer n % 4 (group n % 2)
constexpr int kBarEpi = 1, kBarGroup0 = 2;          // named barrier ids (groups use 2..5)
constexpr int kNumSlots = 128;                      // per-step metadata / barrier slots (< 256: 8-bit field)
constexpr int kBatch = 32;                          // steps published per producer batch (one per lane)
constexpr int kMinStepsPerPiece = 4;
static_assert(kWarpDec + kGroups * kGroupWarps == kThreads / 32, "warp roles");

template <int N_MMA>
struct Cfg {
  static_assert(N_MMA == 16 || N_MMA == 32 || N_MMA == 64 || N_MMA == 128 || N_MMA == 256, "N bucket");
  static constexpr int kNumDense = kNumDenseBufs;
  static constexpr int kBSlabBytes = N_MMA * kTile * 2;  // one 64-wide K tile of B
  static constexpr int kSlabsPerReq = kBSlabBytes >= 16384 ? 1 : 16384 / kBSlabBytes;  // K tiles per TMA request
  static constexpr int kReqBytes = kSlabsPerReq * kBSlabBytes;
  static constexpr int kNumReq = N_MMA <= 128 ? 3 : 2;   // B requests in flight
  static constexpr int kRingBytes = N_MMA <= 128 ? 96 * 1024 : 64 * 1024;
  static constexpr int kRingWords = kRingBytes / 4;
  static constexpr int kChunkTarget = 16 * 1024;  // bytes per published chunk
  static constexpr int kTmemCols = 2 * N_MMA < 32 ? 32 : 2 * N_MMA;
  static constexpr uint32_t kIdesc = umma_idesc_f16_f32(kUnitRows, N_MMA);
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int kOffDense = 0;
  static constexpr int kOffB = kOffDense + kNumDense * kDenseBytes;
  static constexpr int kOffRing = kOffB + kNumReq * kReqBytes;
  static constexpr int kOffMeta = kOffRing + kRingBytes;
  static constexpr int kOffEnd = kOffMeta + kNumSlots * 16;
  static constexpr int kOffBars = kOffEnd + kNumSlots * 8;
  static constexpr int kNumBars = 2 * kNumSlots + 2 * kNumReq + 2 * kNumDense + 4 + 1;
  static constexpr int kOffMisc = kOffBars + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // a chunk is at most the target plus one step with two dense tiles
  static_assert(kRingBytes >= kChunkTarget + 2 * kMaxTileWords * 4, "ring must hold the largest chunk");
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
  int32_t b_kb;    // K tiles of B per TMA request (1 with the 2-D map)
  int32_t b_3d;    // B tensor map is 3-D (64 x N x K/64)
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

// Writes one word's value into the dense 128 x 64 buffer at its swizzled place.
// loc = r*64 + c; the unswizzled byte offset is 2*loc = r*128 + 2c, and the
// 128-byte swizzle XORs the 16-byte chunk index (bits 4-6) with r mod 8
// (bits 7-9 of the same offset).  Sentinels are skipped; a corrupt loc >= 4096
// stays inside the tile (masked) and is reported through `seen`.
__device__ __forceinline__ void scatter_word(uint32_t base_u32, uint32_t w, uint32_t& seen) {
  if ((w >> 16) != 0xFFFFu) {
    const uint32_t x = (w >> 15) & 0x1FFEu;
    const uint32_t off = x ^ ((x >> 3) & 0x70u);
    const uint16_t v = static_cast<uint16_t>(w & 0xFFFFu);
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(base_u32 + off), "h"(v));
    seen |= w;
  }
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xFFFFFFFF;\n\tselp.b32 %0, 1, 0, P;\n\t}" : "=r"(pred));
  return pred != 0;
}

// Thread t of the group takes words 4t..4t+3, 4(t+T).. (T = group size) with
// one 16-byte load each (a tile's list and its ring position are multiples of
// 4 words, so a load never straddles the ring's end); two loads are in flight
// before the stores.
template <int RW>
__device__ __forceinline__ void scatter_range(const uint32_t* ring, uint32_t pos, int cnt, uint32_t base_u32,
                                              int gtid, uint32_t& seen) {
  const uint4* ring4 = reinterpret_cast<const uint4*>(ring);
  for (int i = 4 * gtid; i < cnt; i += 8 * kGroupThreads) {
    const int i2 = i + 4 * kGroupThreads;
    uint32_t idx = pos + static_cast<uint32_t>(i);
    if (idx >= static_cast<uint32_t>(RW)) idx -= RW;
    uint32_t idx2 = pos + static_cast<uint32_t>(i2);
    if (idx2 >= static_cast<uint32_t>(RW)) idx2 -= RW;
    const uint4 w = ring4[idx >> 2];
    const uint4 w2 = i2 < cnt ? ring4[idx2 >> 2] : make_uint4(0xFFFF0000u, 0xFFFF0000u, 0xFFFF0000u, 0xFFFF0000u);
    scatter_word(base_u32, w.x, seen);
    scatter_word(base_u32, w.y, seen);
    scatter_word(base_u32, w.z, seen);
    scatter_word(base_u32, w.w, seen);
    scatter_word(base_u32, w2.x, seen);
    scatter_word(base_u32, w2.y, seen);
    scatter_word(base_u32, w2.z, seen);
    scatter_word(base_u32, w2.w, seen);
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
  uint64_t* words_empty = words_full + kNumSlots;
  uint64_t* b_full = words_empty + kNumSlots;
  uint64_t* b_empty = b_full + Cf::kNumReq;
  uint64_t* a_full = b_empty + Cf::kNumReq;
  uint64_t* a_empty = a_full + Cf::kNumDense;
  uint64_t* acc_full = a_empty + Cf::kNumDense;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cf::kOffMisc + 4);
  volatile int* epi_last = reinterpret_cast<volatile int*>(smem + Cf::kOffMisc + 8);
  uint32_t* flush_word = reinterpret_cast<uint32_t*>(smem + Cf::kOffMisc + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Range rg = piece_range(p, blockIdx.x);
  const uint64_t budget = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumSlots; ++i) { mbar_init(&words_full[i], 1); mbar_init(&words_empty[i], 1); }
    for (int i = 0; i < Cf::kNumReq; ++i) { mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1); }
    for (int i = 0; i < Cf::kNumDense; ++i) { mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 1); }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    *epi_last = 0;
    *flush_word = 0;
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
    // The warp publishes up to 32 steps at once, one per lane.  Steps are
    // grouped into chunks of about kChunkTarget bytes; a chunk occupies
    // [strip-0 words of its steps][strip-1 words of its steps] in the ring and
    // is fetched with two bulk copies (a strip's consecutive K tiles are
    // adjacent in memory), which complete on the barrier of the chunk's first
    // step.  The other steps' barriers only publish their metadata, and their
    // consumers also wait on the chunk's first barrier.  Whole chunks are
    // published only once the ring has room for them, so copies stay large.
    const uint64_t policy = l2_policy_evict_first();
    const uint32_t lane_le = (lane == 31) ? 0xFFFFFFFFu : ((2u << lane) - 1u);
    int64_t n = 0, next_confirm = 0, head = 0, rel = 0;
    int32_t prev_end0 = -1, prev_end1 = -1;
    int prev_ok = 1;
    bool stop = false;
    auto confirm_next = [&]() -> bool {  // lane 0 only
      const int s = static_cast<int>(next_confirm & (kNumSlots - 1));
      if (!mbar_wait(&words_empty[s], static_cast<uint32_t>((next_confirm / kNumSlots) & 1), abort_flag, budget,
                     p.status))
        return false;
      rel = stage_end[s];
      ++next_confirm;
      return true;
    };
    auto copy_to_ring = [&](int64_t pos, int32_t src_word, uint32_t bytes, uint64_t* bar) {
      const uint8_t* src = reinterpret_cast<const uint8_t*>(p.words + src_word);
      while (bytes) {
        const uint32_t at = static_cast<uint32_t>(pos % Cf::kRingBytes);
        const uint32_t len = minu32(bytes, Cf::kRingBytes - at);
        bulk_copy_g2s(ring + at, src, len, bar, policy);
        src += len;
        bytes -= len;
        pos += len;
      }
    };
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
    auto sync_state = [&]() {
      rel = __shfl_sync(0xFFFFFFFFu, rel, 0);
      next_confirm = __shfl_sync(0xFFFFFFFFu, next_confirm, 0);
    };
    int32_t a0, a1, c0, c1;
    fetch(rg.b, a0, a1, c0, c1);
    for (int64_t q0 = rg.b; q0 < rg.e && !stop; q0 += 32) {
      int32_t na0, na1, nc0, nc1;
      fetch(q0 + 32, na0, na1, nc0, nc1);
      const int cnt = static_cast<int>(min64(32, rg.e - q0));
      const bool active = lane < cnt;
      int j = static_cast<int>(q0 % p.TK) + lane;
      while (j >= p.TK) j -= p.TK;
      int32_t n0 = a1 - a0, n1 = c1 - c0;
      const bool ok0 = a0 >= 0 && n0 >= 0 && !(a0 & 3) && !(n0 & 3) && n0 <= kMaxTileWords && a1 <= p.nwords;
      const bool ok1 = c0 >= 0 && n1 >= 0 && !(c0 & 3) && !(n1 & 3) && n1 <= kMaxTileWords && c1 <= p.nwords;
      if (active && !(ok0 && ok1)) record_status(p.status, FLASHSPMM_ERR_CORRUPT_FORMAT);
      if (!ok0 || !active) n0 = 0;
      if (!ok1 || !active) n1 = 0;
      const int ok = ok0 && ok1;
      // batch-local byte prefixes (strip 0, strip 1, both)
      int32_t in0 = 4 * n0, in1 = 4 * n1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y0 = __shfl_up_sync(0xFFFFFFFFu, in0, o), y1 = __shfl_up_sync(0xFFFFFFFFu, in1, o);
        if (lane >= o) { in0 += y0; in1 += y1; }
      }
      const int32_t ex0 = in0 - 4 * n0, ex1 = in1 - 4 * n1, in = in0 + in1, ex = ex0 + ex1;
      // a chunk starts at unit starts, around invalid tiles, where the offsets
      // are not contiguous, and each time the running byte count crosses a
      // multiple of the chunk target
      int32_t pe0 = __shfl_up_sync(0xFFFFFFFFu, a0 + n0, 1), pe1 = __shfl_up_sync(0xFFFFFFFFu, c0 + n1, 1);
      int pok = __shfl_up_sync(0xFFFFFFFFu, ok, 1);
      const int32_t pex = __shfl_up_sync(0xFFFFFFFFu, ex, 1);
      if (lane == 0) { pe0 = prev_end0; pe1 = prev_end1; pok = prev_ok; }
      const bool start = lane == 0 || j == 0 || !ok || !pok || a0 != pe0 || c0 != pe1 ||
                         (ex / Cf::kChunkTarget) != (pex / Cf::kChunkTarget);
      const uint32_t start_mask = __ballot_sync(0xFFFFFFFFu, start);
      int L0 = 0;
      while (L0 < cnt) {
        // Slots of the steps about to be published must be free.  A step's
        // barrier is also waited on (by parity) by the consumers of the later
        // steps of its chunk, so slot s - kNumSlots is reused only once every
        // step that may share its chunk (chunks never leave a batch, hence
        // the next kBatch - 1 steps) has been consumed.
        int fail = 0;
        if (lane == 0) {
          const int64_t need = n + (cnt - L0) - 1 - kNumSlots + (kBatch - 1);
          while (!fail && next_confirm <= need) fail = !confirm_next();
        }
        if (__shfl_sync(0xFFFFFFFFu, fail, 0)) { stop = true; break; }
        sync_state();
        const uint32_t range = (cnt == 32 ? 0xFFFFFFFFu : ((1u << cnt) - 1u)) & ~((1u << L0) - 1u);
        const uint32_t sm = (start_mask | (1u << L0)) & range;
        const int first = 31 - __clz(sm & lane_le);  // chunk start at or below this lane
        const uint32_t above = sm & ~lane_le;
        const int last = (above ? __ffs(above) - 1 : cnt) - 1;
        const int fl = first & 31, ll = last & 31;
        const int32_t base_ex = __shfl_sync(0xFFFFFFFFu, ex, L0);
        const int32_t chunk_end = __shfl_sync(0xFFFFFFFFu, in, ll);
        const bool mine = lane >= L0 && lane < cnt;
        const bool fits = mine && head + (chunk_end - base_ex) - rel <= Cf::kRingBytes;
        const int L1 = L0 + __popc(__ballot_sync(0xFFFFFFFFu, fits));
        if (L1 == L0) {  // wait until the next chunk fits in the ring
          const int32_t need = __shfl_sync(0xFFFFFFFFu, chunk_end, L0) - base_ex;
          if (lane == 0)
            while (!fail && head + need - rel > Cf::kRingBytes) fail = !confirm_next();
          if (__shfl_sync(0xFFFFFFFFu, fail, 0)) { stop = true; break; }
          sync_state();
          continue;
        }
        const int32_t f_ex = __shfl_sync(0xFFFFFFFFu, ex, fl), f_ex0 = __shfl_sync(0xFFFFFFFFu, ex0, fl);
        const int32_t f_ex1 = __shfl_sync(0xFFFFFFFFu, ex1, fl);
        const int32_t l_in0 = __shfl_sync(0xFFFFFFFFu, in0, ll), l_in1 = __shfl_sync(0xFFFFFFFFu, in1, ll);
        if (lane >= L0 && lane < L1) {
          const int64_t step = n + (lane - L0), fstep = n + (first - L0);
          const int s = static_cast<int>(step & (kNumSlots - 1));
          const int fslot = static_cast<int>(fstep & (kNumSlots - 1));
          const int fpar = static_cast<int>((fstep / kNumSlots) & 1);
          const int64_t cp = head + (f_ex - base_ex);  // ring position of the chunk
          const uint32_t cb0 = static_cast<uint32_t>(l_in0 - f_ex0), cb1 = static_cast<uint32_t>(l_in1 - f_ex1);
          const int64_t pos0 = cp + (ex0 - f_ex0), pos1 = cp + cb0 + (ex1 - f_ex1);
          meta[s] = make_int4(static_cast<int>((pos0 % Cf::kRingBytes) >> 2) | (n0 << 16),
                              static_cast<int>((pos1 % Cf::kRingBytes) >> 2) | (n1 << 16), fslot | (fpar << 8), 0);
          stage_end[s] = (lane == last) ? cp + cb0 + cb1 : cp;  // a chunk is freed by its last step
          uint64_t* bar = &words_full[s];
          if (lane == first) {
            mbar_arrive_expect_tx(bar, cb0 + cb1);
            copy_to_ring(cp, a0, cb0, bar);
            copy_to_ring(cp + cb0, c0, cb1, bar);
          } else {
            mbar_arrive(bar);
          }
        }
        // Measured on B200: one shared-memory reduction from the producer warp
        // after each published batch makes its bulk copies start markedly
        // sooner (about 2x kernel throughput); memory and proxy fences, plain
        // stores or sleeps at this point do not have that effect.
        if (lane == 0) red_shared_add(flush_word, 1u);
        const int tail = L1 - 1;
        head += __shfl_sync(0xFFFFFFFFu, in, tail) - base_ex;
        prev_end0 = __shfl_sync(0xFFFFFFFFu, a0 + n0, tail);
        prev_end1 = __shfl_sync(0xFFFFFFFFu, c0 + n1, tail);
        prev_ok = __shfl_sync(0xFFFFFFFFu, ok, tail);
        n += L1 - L0;
        L0 = L1;
      }
      a0 = na0; a1 = na1; c0 = nc0; c1 = nc1;
    }
    // drain: wait (bounded) for copies still in flight before the CTA exits
    if (lane == 0) {
      for (int64_t k = max64(0, n - kNumSlots); k < n; ++k)
        mbar_wait(&words_full[k & (kNumSlots - 1)], static_cast<uint32_t>((k / kNumSlots) & 1), abort_flag, budget,
                  p.status);
    }
  } else if (warp == kWarpB) {
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
      if (uses > 0)
        mbar_wait(&b_full[lane], static_cast<uint32_t>((uses - 1) & 1), abort_flag, budget, p.status);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------ tcgen05 MMA issuer
    // The whole warp runs the loop; lane 0 waits on the barriers, and one
    // elected lane issues the MMAs and commits (issue from a converged warp is
    // markedly cheaper than from a lone divergent thread).
    const int kb = p.b_kb;
    int64_t uc = 0;
    int d = 0, r = -1;
    uint32_t dph = 0, rph = 1;
    int j = static_cast<int>(rg.b % p.TK);
    bool issued = false;
    for (int64_t q = rg.b; q < rg.e; ++q) {
      const bool first = (q == rg.b) || (j == 0);
      const bool last = (q == rg.e - 1) || (j == p.TK - 1);
      const int ab = static_cast<int>(uc & 1);
      const int jk = j % kb;
      const bool new_req = (q == rg.b) || jk == 0;  // first step served by a new B request
      if (new_req) {
        if (++r == Cf::kNumReq) r = 0;
        if (r == 0) rph ^= 1u;
      }
      int ok = 1;
      if (lane == 0) {
        if (first) ok = mbar_wait(&acc_empty[ab], static_cast<uint32_t>(((uc >> 1) & 1) ^ 1), abort_flag, budget, p.status);
        if (ok && new_req) ok = mbar_wait(&b_full[r], rph, abort_flag, budget, p.status);
        if (ok) ok = mbar_wait(&a_full[d], dph, abort_flag, budget, p.status);
      }
      if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;
      if (first) tc_fence_after_sync();  // accumulator handed back by the epilogue's tcgen05.ld
      const uint64_t adesc = smem_desc_k_sw128(smem_u32(dense + d * kDenseBytes));
      const uint64_t bdesc = smem_desc_k_sw128(smem_u32(bslab + r * Cf::kReqBytes + jk * Cf::kBSlabBytes));
      const uint32_t tmem_d = tmem_base + static_cast<uint32_t>(ab * N_MMA);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)  // K = 16 per MMA: advance 32 bytes inside the swizzle atom
          umma_f16_ss(tmem_d, adesc + 2 * kk, bdesc + 2 * kk, Cf::kIdesc, (first && kk == 0) ? 0u : 1u);
        umma_commit(&a_empty[d]);
        if (jk == kb - 1 || last) umma_commit(&b_empty[r]);  // request fully used
        if (last) umma_commit(&acc_full[ab]);
      }
      __syncwarp();
      issued = true;
      if (last) ++uc;
      if (++d == Cf::kNumDense) { d = 0; dph ^= 1u; }
      if (++j == p.TK) j = 0;
    }
    if (issued) {  // all MMAs retired before tensor memory is released
      if (elect_one()) umma_commit(mma_done);
      __syncwarp();
      if (lane == 0) mbar_wait(mma_done, 0, abort_flag, budget, p.status);
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
#pragma unroll 1
          for (int nc = 0; nc < p.N; nc += 16) {
            float acc[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
#pragma unroll 1
            for (int64_t k = 0; k < ncontrib; ++k) {
              const float* src = p.partials + (partial_slot(p, first_pc + k, u) * p.N + nc) * kUnitRows + row;
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (nc + i < p.N) acc[i] += __ldcg(src + i * kUnitRows);
            }
            if (m < p.M) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (nc + i < p.N) p.C[static_cast<int64_t>(nc + i) * p.M + m] = __float2half_rn(acc[i]);
            }
          }
          if (etid == 0) p.counters[u] = 0;
        }
        named_barrier(kBarEpi, kEpiThreads);
      }
    }
  } else {
    // ------------------------------------------------ decompress (rst_smem + extract)
    // Group g takes every kGroups-th step and alternates between dense
    // buffers g and g + 2, so the buffer it zeroes for its next step was last
    // read by the MMAs of two steps earlier.  Two group barriers per step: one
    // after the words have landed (which also orders the zero-fill), one
    // after the scatter.
    const int g = (warp - kWarpDec) / kGroupWarps;
    const int gtid = threadIdx.x - (kWarpDec + g * kGroupWarps) * 32;
    const uint32_t bar_id = kBarGroup0 + g;
    const uint32_t* rw = reinterpret_cast<const uint32_t*>(ring);
    uint32_t seen = 0;
    auto zero_buffer = [&](int dbi) {
      uint4* dz = reinterpret_cast<uint4*>(dense + dbi * kDenseBytes);
#pragma unroll
      for (int i = 0; i < kDenseBytes / 16 / kGroupThreads; ++i) dz[i * kGroupThreads + gtid] = make_uint4(0, 0, 0, 0);
    };
    bool next_ok = true;
    if (rg.b + g < rg.e) zero_buffer(g);  // first use of the buffer: nothing to wait for
    for (int64_t q = rg.b + g, n = g; q < rg.e; q += kGroups, n += kGroups) {
      const int s = static_cast<int>(n % kNumSlots);
      const int dbi = static_cast<int>(n % kNumDenseBufs);
      const uint32_t dense_u32 = smem_u32(dense + dbi * kDenseBytes);
      // the group leader waits for the words; the others sleep in the barrier
      bool ok = next_ok;
      if (gtid == 0 && ok) {
        ok = mbar_wait(&words_full[s], static_cast<uint32_t>((n / kNumSlots) & 1), abort_flag, budget, p.status);
        if (ok) {
          const int fz = meta[s].z;  // chunk whose copy carries this step's words
          ok = mbar_wait(&words_full[fz & 0xFF], static_cast<uint32_t>((fz >> 8) & 1), abort_flag, budget, p.status);
        }
      }
      if (named_barrier_or(bar_id, kGroupThreads, !ok)) break;
      const int4 mt = meta[s];
      scatter_range<Cf::kRingWords>(rw, static_cast<uint32_t>(mt.x & 0xFFFF), mt.x >> 16, dense_u32, gtid, seen);
      scatter_range<Cf::kRingWords>(rw, static_cast<uint32_t>(mt.y & 0xFFFF), mt.y >> 16, dense_u32 + 8192u, gtid,
                                    seen);
      fence_proxy_async_smem();
      named_barrier(bar_id, kGroupThreads);
      if (gtid == 0) {
        mbar_arrive(&a_full[dbi]);
        mbar_arrive(&words_empty[s]);
      }
      // zero the buffer of this group's next step once its previous MMAs retired
      const int64_t n2 = n + kGroups;
      if (q + kGroups < rg.e) {
        const int d2 = static_cast<int>(n2 % kNumDenseBufs);
        next_ok = mbar_wait(&a_empty[d2], static_cast<uint32_t>(((n2 / kNumDenseBufs) & 1) ^ 1), abort_flag, budget,
                            p.status);
        if (next_ok) zero_buffer(d2);
      }
    }
    if (seen >> 28) record_status(p.status, FLASHSPMM_ERR_CORRUPT_FORMAT);
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
  p.b_kb = b3d ? Cf::kSlabsPerReq : 1;
  p.b_3d = b3d ? 1 : 0;
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
