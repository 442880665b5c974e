// extern "C" entry points of libflashspmm: argument checks, then the kernel
// launchers.  This is the host wrapper the Flash-LLM review lists as
// SpMM_API (section 5, "project structure"), reshaped as a plain C ABI that
// takes device pointers, sizes and a stream and never allocates.
#include <cuda.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "common.cuh"

namespace flashspmm {

__device__ int g_device_status = 0;

static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

struct SymbolCache {
  std::mutex mu;
  CUcontext ctx[64][2] = {};
  void* ptr[64][2] = {};
};

SymbolCache& symbol_cache() {
  static SymbolCache c;
  return c;
}

}  // namespace

void* symbol_address_cached(int slot, const void* symbol) {
  int dev = 0;
  if (slot < 0 || slot > 1 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return nullptr;
  CUcontext ctx = nullptr;  // null until the runtime has made the device's context current
  if (get(&ctx) != CUDA_SUCCESS) return nullptr;
  SymbolCache& c = symbol_cache();
  std::lock_guard<std::mutex> lock(c.mu);
  if (!ctx || c.ctx[dev][slot] != ctx || !c.ptr[dev][slot]) {
    void* a = nullptr;
    // the lookup also creates and binds the device's primary context if needed
    if (cudaGetSymbolAddress(&a, symbol) != cudaSuccess || !a) return nullptr;
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
    c.ctx[dev][slot] = ctx;
    c.ptr[dev][slot] = a;
  }
  return c.ptr[dev][slot];
}

int* device_status_ptr() { return static_cast<int*>(symbol_address_cached(0, &g_device_status)); }

}  // namespace flashspmm

using namespace flashspmm;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

flashspmm_status check_encoder_args(const void* A, int32_t M, int32_t K, int32_t tile_m, int32_t tile_k) {
  if (M < 0 || K < 0 || tile_m <= 0 || tile_k <= 0) return FLASHSPMM_ERR_INVALID_ARG;
  if (static_cast<int64_t>(tile_m) * tile_k > 65535) return FLASHSPMM_ERR_UNSUPPORTED;
  if (tile_k % 8 != 0 || K % 8 != 0) return FLASHSPMM_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(M) * K > 0 && A == nullptr) return FLASHSPMM_ERR_INVALID_ARG;
  if (A && !aligned16(A)) return FLASHSPMM_ERR_ALIGNMENT;
  return FLASHSPMM_OK;
}

flashspmm_status check_view(const flashspmm_tcsl* A) {
  if (!A) return FLASHSPMM_ERR_INVALID_ARG;
  if (A->M < 0 || A->K < 0 || A->tile_m <= 0 || A->tile_k <= 0 || A->nwords < 0 || A->nwords > INT32_MAX)
    return FLASHSPMM_ERR_INVALID_ARG;
  if (static_cast<int64_t>(A->tile_m) * A->tile_k > 65535) return FLASHSPMM_ERR_UNSUPPORTED;
  if (!A->tile_offsets) return FLASHSPMM_ERR_INVALID_ARG;
  if (A->nwords > 0 && !A->words) return FLASHSPMM_ERR_INVALID_ARG;
  if (A->words && !aligned16(A->words)) return FLASHSPMM_ERR_ALIGNMENT;
  if ((A->nwords & 3) != 0) return FLASHSPMM_ERR_CORRUPT_FORMAT;
  const int64_t tk = A->tile_k > 0 ? (static_cast<int64_t>(A->K) + A->tile_k - 1) / A->tile_k : 0;
  if (A->offsets_ld < 0 || (A->offsets_ld > 0 && A->offsets_ld < tk)) return FLASHSPMM_ERR_INVALID_ARG;
  if (A->reserved != 0 || A->bounds_pieces < 0 || (A->piece_bounds && A->bounds_pieces == 0))
    return FLASHSPMM_ERR_INVALID_ARG;
  return FLASHSPMM_OK;
}

bool have_device() {
  int n = 0;
  return cudaGetDeviceCount(&n) == cudaSuccess && n > 0;
}

}  // namespace

extern "C" {

int flashspmm_abi_version(void) { return FLASHSPMM_ABI_VERSION; }

const char* flashspmm_status_string(int status) {
  switch (status) {
    case FLASHSPMM_OK: return "ok";
    case FLASHSPMM_ERR_INVALID_ARG: return "invalid argument";
    case FLASHSPMM_ERR_UNSUPPORTED: return "unsupported shape or tile";
    case FLASHSPMM_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case FLASHSPMM_ERR_CAPACITY: return "buffer or workspace too small";
    case FLASHSPMM_ERR_CUDA: return "CUDA runtime error";
    case FLASHSPMM_ERR_CORRUPT_FORMAT: return "corrupt Tiled-CSL data";
    case FLASHSPMM_ERR_TIMEOUT: return "bounded in-kernel wait timed out";
    case FLASHSPMM_ERR_NO_DEVICE: return "no usable CUDA device";
    default: return "unknown status";
  }
}

int64_t flashspmm_num_tiles(int32_t M, int32_t K, int32_t tile_m, int32_t tile_k) {
  if (M < 0 || K < 0 || tile_m <= 0 || tile_k <= 0) return -1;
  return static_cast<int64_t>((M + tile_m - 1) / tile_m) * ((K + tile_k - 1) / tile_k);
}

flashspmm_status flashspmm_tcsl_count(const void* A, int32_t M, int32_t K, int32_t tile_m, int32_t tile_k,
                                      int32_t* tile_offsets, int64_t* nnz, void* stream) {
  flashspmm_status st = check_encoder_args(A, M, K, tile_m, tile_k);
  if (st != FLASHSPMM_OK) return st;
  if (!tile_offsets || !nnz) return FLASHSPMM_ERR_INVALID_ARG;
  if (!have_device()) return FLASHSPMM_ERR_NO_DEVICE;
  return launch_tcsl_count(A, M, K, tile_m, tile_k, tile_offsets, nnz, as_stream(stream)) == cudaSuccess
             ? FLASHSPMM_OK
             : FLASHSPMM_ERR_CUDA;
}

flashspmm_status flashspmm_tcsl_fill(const void* A, int32_t M, int32_t K, int32_t tile_m, int32_t tile_k,
                                     const int32_t* tile_offsets, uint32_t* words, int64_t words_capacity,
                                     void* stream) {
  flashspmm_status st = check_encoder_args(A, M, K, tile_m, tile_k);
  if (st != FLASHSPMM_OK) return st;
  if (!tile_offsets || words_capacity < 0 || (words_capacity > 0 && !words)) return FLASHSPMM_ERR_INVALID_ARG;
  if (words && !aligned16(words)) return FLASHSPMM_ERR_ALIGNMENT;
  if (!have_device()) return FLASHSPMM_ERR_NO_DEVICE;
  return launch_tcsl_fill(A, M, K, tile_m, tile_k, tile_offsets, words, words_capacity, as_stream(stream)) ==
                 cudaSuccess
             ? FLASHSPMM_OK
             : FLASHSPMM_ERR_CUDA;
}

flashspmm_status flashspmm_tcsl_reorder_banks(const int32_t* tile_offsets, uint32_t* words, int64_t nwords, int32_t M,
                                               int32_t K, int32_t tile_m, int32_t tile_k, void* stream) {
  if (M < 0 || K < 0 || tile_m <= 0 || tile_k <= 0 || nwords < 0 || nwords > INT32_MAX || !tile_offsets ||
      (nwords > 0 && !words))
    return FLASHSPMM_ERR_INVALID_ARG;
  if (tile_m != 64 || tile_k != 64) return FLASHSPMM_ERR_UNSUPPORTED;
  if (words && !aligned16(words)) return FLASHSPMM_ERR_ALIGNMENT;
  if (!have_device()) return FLASHSPMM_ERR_NO_DEVICE;
  const int64_t nt = static_cast<int64_t>((M + 63) / 64) * ((K + 63) / 64);
  return launch_tcsl_reorder_banks(tile_offsets, words, nt, nwords, as_stream(stream)) == cudaSuccess
             ? FLASHSPMM_OK
             : FLASHSPMM_ERR_CUDA;
}

flashspmm_status flashspmm_tcsl_validate(const flashspmm_tcsl* A, void* stream) {
  flashspmm_status st = check_view(A);
  if (st != FLASHSPMM_OK) return st;
  if (A->offsets_ld != 0 && A->offsets_ld != (static_cast<int64_t>(A->K) + A->tile_k - 1) / A->tile_k)
    return FLASHSPMM_ERR_UNSUPPORTED;
  if (!have_device()) return FLASHSPMM_ERR_NO_DEVICE;
  return launch_tcsl_validate(A, as_stream(stream)) == cudaSuccess ? FLASHSPMM_OK : FLASHSPMM_ERR_CUDA;
}

size_t flashspmm_spmm_workspace_bytes(int32_t M, int32_t K, int32_t N, int32_t split_k) {
  if (M <= 0 || K <= 0 || N <= 0 || N > 256) return 0;
  const int sms = device_sm_count();
  const size_t even = make_spmm_plan(M, K, N, split_k, sms).workspace_bytes;
  if (split_k > 0) return even;
  const size_t table = make_spmm_plan(M, K, N, split_k, sms, true).workspace_bytes;
  return table > even ? table : even;
}

int32_t flashspmm_partition_pieces(int32_t M, int32_t K, int32_t num_sms) {
  if (M <= 0 || K <= 0 || num_sms <= 0) return -1;
  return make_spmm_plan(M, K, 8, 0, num_sms).num_pieces;
}

flashspmm_status flashspmm_tcsl_partition(const flashspmm_tcsl* A, int32_t num_sms, int64_t* bounds,
                                          int32_t bounds_capacity, void* stream) {
  flashspmm_status st = check_view(A);
  if (st != FLASHSPMM_OK) return st;
  if (A->tile_m != 64 || A->tile_k != 64) return FLASHSPMM_ERR_UNSUPPORTED;
  if (A->M <= 0 || A->K <= 0 || num_sms < 0 || !bounds) return FLASHSPMM_ERR_INVALID_ARG;
  if (!have_device()) return FLASHSPMM_ERR_NO_DEVICE;
  const int sms = num_sms > 0 ? num_sms : device_sm_count();
  if (sms <= 0) return FLASHSPMM_ERR_NO_DEVICE;
  const int32_t pieces = flashspmm_partition_pieces(A->M, A->K, sms);
  if (pieces > kMaxTablePieces) return FLASHSPMM_ERR_UNSUPPORTED;  // the SpMM would not use the table
  if (bounds_capacity < pieces + 1) return FLASHSPMM_ERR_CAPACITY;
  if ((static_cast<int64_t>(A->M) + 127) / 128 > kMaxPartitionUnits) return FLASHSPMM_ERR_UNSUPPORTED;
  return launch_tcsl_partition(A, pieces, bounds, as_stream(stream)) == cudaSuccess ? FLASHSPMM_OK
                                                                                      : FLASHSPMM_ERR_CUDA;
}

int flashspmm_partition_host(const int32_t* tile_offsets, int64_t offsets_ld, int32_t M, int32_t K,
                             int32_t num_pieces, int64_t* bounds) {
  if (!tile_offsets || !bounds || M <= 0 || K <= 0 || num_pieces <= 0 || offsets_ld < 0) return -1;
  return partition_host(tile_offsets, offsets_ld, M, K, num_pieces, bounds) ? 0 : -1;
}

}  // extern "C"

namespace flashspmm {

flashspmm_status prepare_spmm(const flashspmm_tcsl* A, const void* B, void* C, bool c_f32, int32_t M, int32_t K,
                              int32_t N, int32_t split_k, cudaStream_t s, SpmmPlan* plan, bool* done) {
  *done = true;
  flashspmm_status st = check_view(A);
  if (st != FLASHSPMM_OK) return st;
  if (M < 0 || K < 0 || N < 0 || A->M != M || A->K != K) return FLASHSPMM_ERR_INVALID_ARG;
  if (A->tile_m != 64 || A->tile_k != 64) return FLASHSPMM_ERR_UNSUPPORTED;
  if (N > 256 || K % 8 != 0) return FLASHSPMM_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return FLASHSPMM_OK;
  if (!C) return FLASHSPMM_ERR_INVALID_ARG;
  if (!have_device()) return FLASHSPMM_ERR_NO_DEVICE;
  if (K == 0) {
    const size_t bytes = static_cast<size_t>(M) * N * (c_f32 ? 4 : 2);
    return cudaMemsetAsync(C, 0, bytes, s) == cudaSuccess ? FLASHSPMM_OK : FLASHSPMM_ERR_CUDA;
  }
  if (!B) return FLASHSPMM_ERR_INVALID_ARG;
  if (!aligned16(B)) return FLASHSPMM_ERR_ALIGNMENT;
  const int sms = device_sm_count();
  if (sms <= 0) return FLASHSPMM_ERR_NO_DEVICE;
  *plan = make_spmm_plan(M, K, N, split_k, sms);
  // a piece table is used when it was made for exactly this plan's pieces
  if (split_k <= 0 && A->piece_bounds && A->bounds_pieces == plan->num_pieces)
    *plan = make_spmm_plan(M, K, N, split_k, sms, true);
  *done = false;
  return FLASHSPMM_OK;
}

}  // namespace flashspmm

extern "C" {

static flashspmm_status spmm_with_workspace(const flashspmm_tcsl* A, const void* B, void* C, bool c_f32, int32_t M,
                                            int32_t K, int32_t N, int32_t split_k, void* workspace,
                                            size_t workspace_bytes, void* stream) {
  cudaStream_t s = as_stream(stream);
  SpmmPlan plan{};
  bool done = true;
  const flashspmm_status st = prepare_spmm(A, B, C, c_f32, M, K, N, split_k, s, &plan, &done);
  if (st != FLASHSPMM_OK || done) return st;
  if (plan.workspace_bytes > 0) {
    if (!workspace || workspace_bytes < plan.workspace_bytes) return FLASHSPMM_ERR_CAPACITY;
    if (!aligned16(workspace)) return FLASHSPMM_ERR_ALIGNMENT;
  }
  return launch_spmm_lscd(A, B, C, c_f32, M, K, N, plan, workspace, s);
}

flashspmm_status flashspmm_spmm_lscd(const flashspmm_tcsl* A, const void* B, void* C, int32_t M, int32_t K,
                                     int32_t N, int32_t split_k, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  return spmm_with_workspace(A, B, C, false, M, K, N, split_k, workspace, workspace_bytes, stream);
}

flashspmm_status flashspmm_spmm_lscd_f32(const flashspmm_tcsl* A, const void* B, float* C, int32_t M, int32_t K,
                                         int32_t N, int32_t split_k, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  return spmm_with_workspace(A, B, C, true, M, K, N, split_k, workspace, workspace_bytes, stream);
}

flashspmm_status flashspmm_round_f16(const float* x, void* y, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return FLASHSPMM_ERR_INVALID_ARG;
  if (n == 0) return FLASHSPMM_OK;
  if (!aligned16(x) || !aligned16(y)) return FLASHSPMM_ERR_ALIGNMENT;
  if (!have_device()) return FLASHSPMM_ERR_NO_DEVICE;
  return launch_round_f16(x, static_cast<__half*>(y), n, as_stream(stream)) == cudaSuccess ? FLASHSPMM_OK
                                                                                          : FLASHSPMM_ERR_CUDA;
}

flashspmm_status flashspmm_spmm_lscd_host(const flashspmm_tcsl* A, const void* B_host, void* C_host, void* B_dev,
                                          void* C_dev, int32_t M, int32_t K, int32_t N, int32_t split_k,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  if (M < 0 || K < 0 || N < 0) return FLASHSPMM_ERR_INVALID_ARG;
  const size_t b_bytes = static_cast<size_t>(K) * N * 2, c_bytes = static_cast<size_t>(M) * N * 2;
  if ((b_bytes && (!B_host || !B_dev)) || (c_bytes && (!C_host || !C_dev))) return FLASHSPMM_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  if (b_bytes && cudaMemcpyAsync(B_dev, B_host, b_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return FLASHSPMM_ERR_CUDA;
  const flashspmm_status st = flashspmm_spmm_lscd(A, B_dev, C_dev, M, K, N, split_k, workspace, workspace_bytes,
                                                  stream);
  if (st != FLASHSPMM_OK) return st;
  if (c_bytes && cudaMemcpyAsync(C_host, C_dev, c_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return FLASHSPMM_ERR_CUDA;
  return FLASHSPMM_OK;
}

flashspmm_status flashspmm_get_device_status(void* stream) {
  if (!have_device()) return FLASHSPMM_ERR_NO_DEVICE;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return FLASHSPMM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return FLASHSPMM_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return FLASHSPMM_ERR_CUDA;
  }
  return static_cast<flashspmm_status>(v);
}

uint64_t flashspmm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
