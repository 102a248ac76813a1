// Weighted combine of the k expert outputs of each token.
//
// out[t, :] = sum_j w[t, j] * Z[inv[t*k + j], :], j ascending, accumulated in
// fp32 and rounded to bf16 once.  This is the weighted sum over a token's
// experts (experts4bit-qlora 0.22.0, "Which training path?", numerics
// paragraph); a per-token gather in slot order instead of scattered atomics
// keeps it deterministic.  Z holds the per-slot down-projection rows in bf16
// (one rounding of each expert's output, as the layer's bf16 activations
// have).  HBM-bound: 16-byte loads of Z rows, eight columns per thread.
#include "common.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

__global__ void __launch_bounds__(128) combine_kernel(const uint16_t* __restrict__ z, const int32_t* __restrict__ inv,
                                                      const float* __restrict__ w, int64_t S, int k, int H,
                                                      uint16_t* __restrict__ out) {
  const int c8 = blockIdx.y * blockDim.x + threadIdx.x;  // 8 columns per thread
  const int64_t t = blockIdx.x;
  if (c8 * 8 >= H) return;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < k; ++j) {
    const int64_t pos = clampv<int64_t>(inv[t * k + j], 0, S - 1);
    const float wv = w[t * k + j];
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(z + pos * H) + c8);
    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(wv, __uint_as_float(vw[i] << 16), acc[2 * i]);
      acc[2 * i + 1] = fmaf(wv, __uint_as_float(vw[i] & 0xffff0000u), acc[2 * i + 1]);
    }
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  reinterpret_cast<uint4*>(out + t * H)[c8] = o;
}

}  // namespace

cudaError_t launch_combine(const uint16_t* z, const int32_t* inv, const float* w, int64_t M, int k, int H,
                           uint16_t* out, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const int threads = 128;
  dim3 grid(static_cast<unsigned>(M), (H / 8 + threads - 1) / threads);
  LaunchScope ls("combine", stream);
  combine_kernel<<<grid, threads, 0, stream>>>(z, inv, w, M * k, k, H, out);
  return cudaGetLastError();
}

}  // namespace e4b
