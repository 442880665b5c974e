/*
 * libflashspmm: Load-as-Sparse / Compute-as-Dense (LSCD) SpMM for B200 (sm_100a).
 *
 * Computes C = A x B where A is an unstructured-pruned fp16 weight matrix
 * (M x K) held in the Tiled-CSL format and B is a skinny fp16 activation
 * matrix (K x N, N <= 256), with fp32 accumulation and fp16 output.
 *
 * Sources: the Flash-LLM paper review page ("Flash-LLM: Enabling
 * Cost-Effective and Highly-Efficient Large Generative Model Inference with
 * Unstructured Sparsity", xllm-io.github.io paper review):
 *   [core-formulas]  section 3, "core formulas": C = A x B with A in R^{M x K}
 *                    the sparse weights and B in R^{K x N} the dense features.
 *   [tiled-csl]      section 3, "sparse encoding format: Tiled-CSL":
 *                    NonZeros[] grouped by tile, one 32-bit word per nonzero
 *                    = [16-bit value | 16-bit in-tile index], TileOffsets[]
 *                    locating each tile, 128-bit vectorised loads.
 *   [lscd]           section 2, "solution overview": load the weights in
 *                    sparse form, expand on chip, multiply densely on tensor
 *                    cores.
 *   [code-layout]    section 5, "project structure": SpMM_API (host wrapper),
 *                    SpMM kernel and Reduction kernel (split-K partial sums).
 *
 * Format (Tiled-CSL as this library reads it):
 *   - tiles of tile_m x tile_k, enumerated row-major over the tile grid
 *     (t = i * ceil(K/tile_k) + j); edge tiles may be ragged;
 *   - loc = r * tile_k + c inside the tile (row-major, full tile_k pitch);
 *   - word = fp16 bits | (loc << 16); stored iff the fp16 bits are not 0x0000;
 *   - words of a tile in ascending loc (or, after flashspmm_tcsl_reorder_banks,
 *     the bank-balanced order; the SpMM accepts either), padded to a multiple
 *     of 4 words with the sentinel 0xFFFF0000; tile_m * tile_k <= 65535;
 *   - tile_offsets: int32[num_tiles + 1], in words, tile_offsets[0] = 0.
 *
 * Views (tensor-parallel shards without copying; the Flash-LLM review,
 * section 5 item 5, distributed inference).  The SpMM reads tile offsets as
 * absolute indices into `words` and addresses tile (i, j) of its operand as
 * tile_offsets[i * ld + j], so:
 *   - rows: a run of whole strips of a larger matrix is the view whose
 *     tile_offsets point at the run's first tile, with that matrix's ld,
 *     words and nwords;
 *   - K range: K tiles [j0, j1) of every strip are the view whose
 *     tile_offsets point at entry j0, with that matrix's ld (its tiles per
 *     strip), words and nwords, and K = the range's width.  Tile j1 - 1 of a
 *     strip ends where tile j1 (or the next strip) begins, so no extra entry
 *     is needed.
 * flashspmm_tcsl_validate checks whole matrices only (ld equal to the tiles
 * per strip and offsets starting at 0).
 *
 * Conventions for every call:
 *   - Array arguments are DEVICE pointers owned by the caller (the only host
 *     pointers are B_host / C_host of flashspmm_spmm_lscd_host); the library
 *     allocates no device memory and keeps no pointer after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream.
 *   - Argument errors detectable on the host return synchronously and launch
 *     nothing.  Errors found by a kernel (corrupt format, timeout) are recorded
 *     in a device status word read by flashspmm_get_device_status().
 *   - No call throws; none synchronises except flashspmm_get_device_status().
 */
#ifndef FLASHSPMM_H
#define FLASHSPMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FLASHSPMM_ABI_VERSION 2

/* Bytes of the fixed device scratch behind flashspmm_spmm_lscd_noalloc. */
#define FLASHSPMM_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

typedef enum {
  FLASHSPMM_OK = 0,
  FLASHSPMM_ERR_INVALID_ARG = 1,    /* null pointer, negative size, mismatched view */
  FLASHSPMM_ERR_UNSUPPORTED = 2,    /* shape or tile outside what the kernels handle */
  FLASHSPMM_ERR_ALIGNMENT = 3,      /* a pointer or leading dimension breaks 16-byte alignment */
  FLASHSPMM_ERR_CAPACITY = 4,       /* output buffer / workspace too small, or > 2^31 words */
  FLASHSPMM_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
  FLASHSPMM_ERR_CORRUPT_FORMAT = 6, /* tile offsets or words violate the format */
  FLASHSPMM_ERR_TIMEOUT = 7,        /* a bounded in-kernel wait ran out (kernel exited early) */
  FLASHSPMM_ERR_NO_DEVICE = 8       /* no usable sm_100 device is current */
} flashspmm_status;

/* A read-only view of a Tiled-CSL matrix in device memory.  The library owns
 * nothing it points to. */
typedef struct {
  int32_t M, K;                 /* dense shape of A (of the view) */
  int32_t tile_m, tile_k;       /* format tile; the SpMM kernel needs 64 x 64 */
  int64_t nnz;                  /* stored entries excluding padding (informational; -1 = not counted) */
  int64_t nwords;               /* words reachable through `words` (a whole matrix: tile_offsets[num_tiles]) */
  const int32_t* tile_offsets;  /* device; tile (i, j) spans words [tile_offsets[i*ld + j], tile_offsets[i*ld + j + 1]) */
  const uint32_t* words;        /* device, nwords entries, 16-byte aligned */
  int64_t offsets_ld;           /* ld above: entries from one strip's first tile to the next strip's.
                                   0 means ceil(K / tile_k), a whole matrix.  A K-range shard of a
                                   larger matrix keeps that matrix's ld and points tile_offsets at
                                   its first K tile (see "Views" above). */
  const int64_t* piece_bounds;  /* optional, device: word-balanced work partition written by
                                   flashspmm_tcsl_partition for this view; NULL = even pieces */
  int32_t bounds_pieces;        /* pieces that table describes (it holds bounds_pieces + 1 entries) */
  int32_t reserved;             /* must be 0 */
} flashspmm_tcsl;

/* ABI version of the loaded library (FLASHSPMM_ABI_VERSION at build time). */
int flashspmm_abi_version(void);

/* Static, human-readable name of a status code (never NULL). */
const char* flashspmm_status_string(int status);

/* Number of format tiles: ceil(M / tile_m) * ceil(K / tile_k); -1 on bad args. */
int64_t flashspmm_num_tiles(int32_t M, int32_t K, int32_t tile_m, int32_t tile_k);

/* Encoder, pass 1 of 2 [tiled-csl]: counts the nonzero bit patterns of every
 * tile of A and writes the padded running offsets.
 *   A             device fp16, M x K row-major, 16-byte aligned, K % 8 == 0.
 *   tile_m/tile_k tile_m >= 1, tile_k % 8 == 0, tile_m * tile_k <= 65535.
 *   tile_offsets  device int32[num_tiles + 1]; receives the Tiled-CSL offsets.
 *   nnz           device int64[1]; receives the number of stored entries.
 * Read tile_offsets[num_tiles] (the word count) after the stream reaches this
 * point to size the words buffer for pass 2.  A total above 2^31 - 1 words
 * records FLASHSPMM_ERR_CAPACITY in the device status word. */
flashspmm_status flashspmm_tcsl_count(const void* A, int32_t M, int32_t K, int32_t tile_m, int32_t tile_k,
                                      int32_t* tile_offsets, int64_t* nnz, void* stream);

/* Encoder, pass 2 of 2 [tiled-csl]: writes every tile's words in ascending loc
 * followed by sentinel padding, at the offsets from pass 1.  Output is
 * bit-identical to the format definition above.
 *   words           device uint32[words_capacity], 16-byte aligned.
 * A tile whose entries do not fit its offset range (A changed since pass 1) or
 * an offset beyond words_capacity records FLASHSPMM_ERR_CAPACITY and that tile
 * is left unwritten. */
flashspmm_status flashspmm_tcsl_fill(const void* A, int32_t M, int32_t K, int32_t tile_m, int32_t tile_k,
                                     const int32_t* tile_offsets, uint32_t* words, int64_t words_capacity,
                                     void* stream);

/* Optional encoder pass [tiled-csl] (page's ahead-of-time reordering of each
 * tile's nonzeros, restated for this library's dense tile): rewrites, in
 * place, the words of every 64 x 64 tile of an ascending-loc encoding into
 * the bank-balanced order ("word order v2").  The value at loc lands in the
 * SpMM's shared-memory tile at byte x = 2*loc swizzled as x ^ ((x >> 3) & 0x70),
 * i.e. in bank (that offset >> 2) & 31.  A tile's real words (those before its
 * first sentinel) are placed window by window, a window being 32 consecutive
 * positions from the tile start: at each window's start the banks are ranked
 * by unplaced words (most first, ties to the lower bank) and the window takes
 * the lowest-loc unplaced word of each bank in rank order, round after round,
 * until it is full.  Offsets, the set of words, padding and the decoded
 * matrix are unchanged; a 32-word store of the SpMM then hits as many
 * distinct banks as possible.
 *   tile_offsets  device int32[num_tiles + 1] of an M x K matrix, 64 x 64 tiles.
 *   words         device uint32[nwords], rewritten in place, 16-byte aligned.
 * A tile longer than 4096 words or holding a real word with loc >= 4096
 * records FLASHSPMM_ERR_CORRUPT_FORMAT and is left unchanged.  Tiles other
 * than 64 x 64 return FLASHSPMM_ERR_UNSUPPORTED. */
flashspmm_status flashspmm_tcsl_reorder_banks(const int32_t* tile_offsets, uint32_t* words, int64_t nwords, int32_t M,
                                              int32_t K, int32_t tile_m, int32_t tile_k, void* stream);

/* Checked mode: verifies a whole Tiled-CSL matrix on the GPU (offsets start at 0,
 * non-decreasing, multiples of 4, end at nwords, segment <= roundup4(area);
 * each tile holds real words with distinct in-range locs and nonzero value
 * bits, in any order (ascending or bank-balanced), then fewer than four exact
 * sentinels).  Any violation records FLASHSPMM_ERR_CORRUPT_FORMAT in the
 * device status word.  A view with offsets_ld other than 0 or ceil(K/tile_k)
 * returns FLASHSPMM_ERR_UNSUPPORTED (validate the whole matrix instead). */
flashspmm_status flashspmm_tcsl_validate(const flashspmm_tcsl* A, void* stream);

/* Pieces (CTAs) of the automatic plan (split_k = 0) for an M x K operand on
 * num_sms SMs: min(num_sms, ceil(T / 4)) with T = ceil(M / 128) * ceil(K / 64)
 * steps.  flashspmm_tcsl_partition writes that many pieces plus one entry.
 * -1 on bad arguments (M, K, num_sms > 0).  Host only. */
int32_t flashspmm_partition_pieces(int32_t M, int32_t K, int32_t num_sms);

/* Word-balanced work partition for the automatic plan [code-layout].  The
 * plan cuts the step space (step q = u * ceil(K/64) + j: 128-row unit u, K
 * tile j) into P pieces of consecutive steps, one CTA each.  Without a table
 * every piece holds the same number of steps, and a piece over denser rows or
 * columns takes longer.  This call computes pieces of about equal cost
 * instead, where a step costs 1024 plus its words (both strips' tiles,
 * padding included): 1024 words is the fixed per-step cost, measured in word
 * equivalents on B200.  With c(q) the cost of steps [0, q) and c(T) the total,
 * bounds[pc] is the smallest q with P * c(q) >= pc * c(T).  The entries are
 * then raised to at least bounds[pc-1] + 1 (from pc = 1 up) and lowered to at
 * most bounds[pc+1] - 1 (from pc = P - 1 down), so every piece keeps at least
 * one step.  bounds[0] = 0 and bounds[P] = T.
 *   A                view with 64 x 64 tiles (any ld); its offsets are read on
 *                    the device.
 *   num_sms          SMs of the device that will run the SpMM; 0 = the
 *                    current device's.
 *   bounds           device int64[bounds_capacity]; receives P + 1 entries,
 *                    P = flashspmm_partition_pieces(M, K, num_sms).
 * To use it, set A->piece_bounds = bounds and A->bounds_pieces = P.  The SpMM
 * uses a table only when split_k = 0 and P equals its plan's pieces (P <=
 * 512); otherwise it cuts even pieces.  A table that is not strictly
 * increasing from 0 to T makes the SpMM record FLASHSPMM_ERR_CORRUPT_FORMAT
 * and cut even pieces.  More than 16384 units (M > 2,097,152) or P > 512
 * returns FLASHSPMM_ERR_UNSUPPORTED; bounds_capacity < P + 1 returns
 * FLASHSPMM_ERR_CAPACITY. */
flashspmm_status flashspmm_tcsl_partition(const flashspmm_tcsl* A, int32_t num_sms, int64_t* bounds,
                                          int32_t bounds_capacity, void* stream);

/* Host diagnostic of flashspmm_tcsl_partition: the same rule, run on the host
 * over a host copy of a view's offsets (tile (i, j) at tile_offsets[i*ld + j];
 * offsets_ld 0 = ceil(K/64)), for num_pieces pieces.  Writes num_pieces + 1
 * entries to the host array `bounds`.  0, or -1 on bad arguments. */
int flashspmm_partition_host(const int32_t* tile_offsets, int64_t offsets_ld, int32_t M, int32_t K,
                             int32_t num_pieces, int64_t* bounds);

/* Bytes of workspace flashspmm_spmm_lscd needs on the CURRENT device for this
 * problem (0 when no partial sums are needed).  split_k as below.  With
 * split_k = 0 the size also covers a word-balanced piece table, whose piece
 * boundaries may fall anywhere (so with more than one piece it is never 0). */
size_t flashspmm_spmm_workspace_bytes(int32_t M, int32_t K, int32_t N, int32_t split_k);

/* LSCD SpMM [lscd][core-formulas]: C = A x B.
 *   A          Tiled-CSL view with tile_m = tile_k = 64; A->M == M, A->K == K.
 *              Tile offsets that break the format (negative, unaligned, past
 *              nwords, a tile longer than 4096 words) record
 *              FLASHSPMM_ERR_CORRUPT_FORMAT and those tiles are skipped.  Word
 *              contents are not checked here: a word whose loc lies outside
 *              the tile (other than the sentinel) is ignored, so the result is
 *              unspecified but no memory outside the call's buffers is touched;
 *              flashspmm_tcsl_validate finds such words.
 *   B          device fp16, K x N column-major (a contiguous [N][K] array),
 *              16-byte aligned, K % 8 == 0.  B must be finite: the product is
 *              computed densely per tile, so a non-finite B value meets the
 *              tile's stored zeros.
 *   C          device fp16, M x N column-major (a contiguous [N][M] array).
 *   N          1 <= N <= 256.
 *   split_k    0: automatic, the step space (units of 128 rows x 64-wide K
 *              tiles) is cut into one contiguous piece per SM (even in steps,
 *              or from A->piece_bounds when it holds a table for this plan,
 *              see flashspmm_tcsl_partition) and units shared by several
 *              pieces are reduced by the last CTA to finish ([code-layout]
 *              Reduction kernel, fused here); >= 1: each 128-row unit is cut
 *              into min(split_k, ceil(K/64)) K-chunks.
 *              Results are deterministic for a given (problem, split_k, device).
 *   workspace  device, >= flashspmm_spmm_workspace_bytes(...), 16-byte aligned;
 *              may be NULL when that size is 0.  Holds fp32 partial sums and
 *              arrival counters.  Zero it once when it is allocated: every
 *              call that completes leaves the counters zero again (the last
 *              arriving CTA of a unit resets its counter), so one workspace
 *              serves any sequence of calls ordered on a stream without a
 *              clearing step between them.  After FLASHSPMM_ERR_TIMEOUT zero
 *              it again before reuse.  Calls that may run concurrently need
 *              separate workspaces.
 * The kernel is launched with programmatic stream serialisation: its
 * prologue may overlap the tail of the previous kernel in the stream, and it
 * reads no input before that kernel has completed.
 * K == 0 writes zeros to C; M == 0 or N == 0 does nothing. */
flashspmm_status flashspmm_spmm_lscd(const flashspmm_tcsl* A, const void* B, void* C, int32_t M, int32_t K,
                                     int32_t N, int32_t split_k, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* flashspmm_spmm_lscd with fp32 output: C is device fp32, M x N column-major
 * (a contiguous [N][M] float array), holding the fp32 accumulators without
 * the fp16 rounding.  This is the partial product of a K-range shard that a
 * tensor-parallel caller sums across ranks (an all-reduce) before rounding
 * once.  Other arguments, workspace rules and errors as flashspmm_spmm_lscd;
 * K == 0 writes zeros. */
flashspmm_status flashspmm_spmm_lscd_f32(const flashspmm_tcsl* A, const void* B, float* C, int32_t M, int32_t K,
                                         int32_t N, int32_t split_k, void* workspace, size_t workspace_bytes,
                                         void* stream);

/* Rounds n fp32 values to fp16 (round to nearest even, overflow to +-Inf):
 * the last step of a tensor-parallel K split, once the ranks' fp32 partials
 * (flashspmm_spmm_lscd_f32) have been summed.  x and y are device arrays of n
 * elements, 16-byte aligned; they may not overlap. */
flashspmm_status flashspmm_round_f16(const float* x, void* y, int64_t n, void* stream);

/* End-to-end form of flashspmm_spmm_lscd for callers whose activations live
 * in host memory: on `stream` it copies B from B_host (K x N column-major fp16)
 * into the caller's device staging buffer B_dev, runs the SpMM into the
 * device buffer C_dev, and copies C back to C_host (M x N column-major fp16).
 * Host buffers should be pinned for the copies to overlap; the call returns
 * before the copies finish.  Same argument rules as flashspmm_spmm_lscd. */
flashspmm_status flashspmm_spmm_lscd_host(const flashspmm_tcsl* A, const void* B_host, void* C_host, void* B_dev,
                                          void* C_dev, int32_t M, int32_t K, int32_t N, int32_t split_k,
                                          void* workspace, size_t workspace_bytes, void* stream);

/* flashspmm_spmm_lscd without a workspace argument.  The paper has no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory on demand, such as a plugin running inside an engine that owns all
 * device memory and forbids allocation while it executes, or a
 * latency-critical path that cannot accept cudaMalloc's implicit device
 * synchronisation.  The call allocates nothing.
 *   - Its scratch (split-K partial sums and arrival counters) is one
 *     FLASHSPMM_NOALLOC_SCRATCH_BYTES (16 MiB) array that the library places in
 *     the memory of every GPU that loads it, held until the process exits.
 *   - A problem whose flashspmm_spmm_workspace_bytes(M, K, N, split_k) exceeds
 *     that size returns FLASHSPMM_ERR_CAPACITY and launches nothing (with
 *     split_k = 0 on a 148-SM B200, every N <= 96 fits).
 *   - The first call in a device's context looks up the array's device
 *     address (cudaGetSymbolAddress, with that device current) and caches it
 *     for that context; make that first call before any stream capture.  After
 *     a device reset the next call looks it up again.
 *   - All calls on a device share the one array; each call clears its
 *     arrival counters on `stream` (cudaMemsetAsync) before its kernel.
 *     Calls that can overlap on the GPU (unordered streams) race on the array
 *     and give wrong results.
 *   - Other arguments and errors as flashspmm_spmm_lscd. */
flashspmm_status flashspmm_spmm_lscd_noalloc(const flashspmm_tcsl* A, const void* B, void* C, int32_t M, int32_t K,
                                             int32_t N, int32_t split_k, void* stream);

/* Failure-path diagnostic: launches one thread that waits on an mbarrier
 * nothing completes, bounded by timeout_us (1 .. 1e6) microseconds, exactly as
 * the SpMM pipeline's waits are bounded.  When the budget runs out the kernel
 * records FLASHSPMM_ERR_TIMEOUT in the device status word and returns; the
 * context stays usable.  Returns FLASHSPMM_ERR_INVALID_ARG outside the range. */
flashspmm_status flashspmm_selftest_wait_timeout(uint32_t timeout_us, void* stream);

/* Diagnostics of the work partition [code-layout], computed on the host with
 * the same functions the SpMM kernel uses (no device needed), for num_sms SMs:
 *   flashspmm_plan_query  info[0..8] = TM, TK, units U, steps T, mode (0 even
 *                         pieces, 1 split-K per unit), split, pieces, partial
 *                         slots, workspace bytes; `ranges` (may be NULL, else
 *                         2 * pieces int64) receives each piece's [begin, end)
 *                         in steps (step = unit * TK + K tile).  0, or -1 on
 *                         bad arguments (M, K, N, num_sms > 0, N <= 256).
 *   flashspmm_plan_owner  mode 0: the piece holding step q, else -1.
 *   flashspmm_plan_slot   the workspace slot piece pc writes its partial sum
 *                         of unit u to, -1 when the plan has no partial sums
 *                         or the arguments are out of range. */
int flashspmm_plan_query(int32_t M, int32_t K, int32_t N, int32_t split_k, int32_t num_sms, int64_t* info,
                         int64_t* ranges);
int64_t flashspmm_plan_owner(int32_t M, int32_t K, int32_t N, int32_t split_k, int32_t num_sms, int64_t q);
int64_t flashspmm_plan_slot(int32_t M, int32_t K, int32_t N, int32_t split_k, int32_t num_sms, int64_t pc, int64_t u);

/* Dense or sparse, per MatMul [lscd] (the Flash-LLM review, section 5 item 5:
 * the integration's GEMM wrapper picks dense or sparse per weight; section 6,
 * "N dimension": the sparse kernel wins only for skinny N).  From time models
 * fitted to this library's SpMM and to dense fp16 cuBLAS GEMMs of the same
 * shapes on B200 (inputs resident in HBM, CUDA-graph launches):
 *   flashspmm_predict_us     predicted microseconds of this library's SpMM
 *                            (automatic split) and of a dense GEMM for an
 *                            M x K weight with nnz stored entries and N
 *                            columns on num_sms SMs; 0, or -1 on bad
 *                            arguments (M, K, N, num_sms > 0, N <= 256,
 *                            nnz >= 0).  Either output pointer may be NULL.
 *   flashspmm_prefer_sparse  1 when the SpMM is predicted faster, 0 when the
 *                            dense GEMM is, -1 on bad arguments.
 * Host only, no device needed; running the dense GEMM stays the caller's job. */
int flashspmm_predict_us(int32_t M, int32_t K, int32_t N, int64_t nnz, int32_t num_sms, double* t_sparse,
                         double* t_dense);
int flashspmm_prefer_sparse(int32_t M, int32_t K, int32_t N, int64_t nnz, int32_t num_sms);

/* Synchronises `stream`, then reads and clears the library's device status
 * word for the current device: FLASHSPMM_OK or the first error a kernel
 * recorded since the last read. */
flashspmm_status flashspmm_get_device_status(void* stream);

/* Number of kernels this library has launched in this process (diagnostic). */
uint64_t flashspmm_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FLASHSPMM_H */
