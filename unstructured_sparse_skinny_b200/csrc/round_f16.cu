// fp32 -> fp16 rounding for tensor-parallel K splits.
//
// Each rank of a K split (the Flash-LLM review, section 5 item 5: model
// parallelism across GPUs) computes its shard's product in fp32
// (flashspmm_spmm_lscd_f32); after the ranks' partials are summed (an
// all-reduce) this kernel rounds the sum to fp16 once.
#include "common.cuh"

// 8 values per thread per iteration (two 16-byte loads, one 16-byte store),
// at most 8 CTAs per SM in a grid-stride loop, then a scalar tail.
namespace flashspmm {
namespace {

__global__ void __launch_bounds__(256) round_f16_kernel(const float* __restrict__ x, __half* __restrict__ y,
                                                        int64_t n) {
  const int64_t n8 = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(x)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(x)[2 * i + 1];
    union {
      __half2 h[4];
      uint4 u;
    } o;
    o.h[0] = __floats2half2_rn(a.x, a.y);
    o.h[1] = __floats2half2_rn(a.z, a.w);
    o.h[2] = __floats2half2_rn(b.x, b.y);
    o.h[3] = __floats2half2_rn(b.z, b.w);
    reinterpret_cast<uint4*>(y)[i] = o.u;
  }
  if (blockIdx.x == 0)
    for (int64_t i = n8 * 8 + threadIdx.x; i < n; i += blockDim.x) y[i] = __float2half_rn(x[i]);
}

}  // namespace

cudaError_t launch_round_f16(const float* x, __half* y, int64_t n, cudaStream_t s) {
  const int sms = device_sm_count();
  const int64_t want = (n / 8 + 255) / 256;
  const int grid = static_cast<int>(max64(1, min64(want, static_cast<int64_t>(sms > 0 ? sms : 1) * 8)));
  round_f16_kernel<<<grid, 256, 0, s>>>(x, y, n);
  note_launch();
  return cudaGetLastError();
}

}  // namespace flashspmm
