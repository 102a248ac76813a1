// Weighted combine of the k expert outputs of each token.
//
// out[t, :] = sum_j w[t, j] * Z[inv[t*k + j], :], j ascending, accumulated in
// fp32 and rounded to bf16 once.  This is the weighted sum over a token's
// experts (experts4bit-qlora 0.22.0, "Which training path?", numerics
// paragraph); a per-token gather in slot order instead of scattered atomics
// keeps it deterministic.  HBM-bound: 16-byte loads of Z rows.
#include "common.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ z, const int32_t* __restrict__ inv,
                                                      const float* __restrict__ w, int64_t S, int k, int H,
                                                      uint16_t* __restrict__ out) {
  const int c4 = blockIdx.y * blockDim.x + threadIdx.x;  // 4 columns per thread
  const int64_t t = blockIdx.x;
  if (c4 * 4 >= H) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const int64_t pos = clampv<int64_t>(inv[t * k + j], 0, S - 1);
    const float wv = w[t * k + j];
    const float4 v = __ldcs(reinterpret_cast<const float4*>(z + pos * H) + c4);
    acc.x = fmaf(wv, v.x, acc.x);
    acc.y = fmaf(wv, v.y, acc.y);
    acc.z = fmaf(wv, v.z, acc.z);
    acc.w = fmaf(wv, v.w, acc.w);
  }
  uint2 o;
  o.x = pack_bf16x2(acc.x, acc.y);
  o.y = pack_bf16x2(acc.z, acc.w);
  reinterpret_cast<uint2*>(out + t * H)[c4] = o;
}

}  // namespace

cudaError_t launch_combine(const float* z, const int32_t* inv, const float* w, int64_t M, int k, int H,
                           uint16_t* out, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const int threads = 128;
  dim3 grid(static_cast<unsigned>(M), (H / 4 + threads - 1) / threads);
  LaunchScope ls("combine", stream);
  combine_kernel<<<grid, threads, 0, stream>>>(z, inv, w, M * k, k, H, out);
  return cudaGetLastError();
}

}  // namespace e4b
