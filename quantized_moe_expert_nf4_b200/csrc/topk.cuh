// Router top-k of one token by one warp (shared by the routing kernels and the
// fused small-M forward).  Experts are ordered by (logit descending, index
// ascending) through 64-bit keys (order-preserving bits of the logit, then the
// complemented index); the weights are the softmax over the selected logits
// (renormalised) or the full softmax over all experts.
#pragma once

#include "common.cuh"

namespace e4b {

__device__ __forceinline__ uint32_t ordered_bits(float v) {
  if (v == 0.0f) v = 0.0f;  // -0 and +0 compare equal: let the index decide
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One warp selects the top k of row `logits[0..E)`; lane j < k receives the
// j-th expert id and its logit.  MAXJ = ceil(E / 32) values held per lane.
template <int MAXJ>
__device__ __forceinline__ void warp_topk(const float* __restrict__ row, int E, int k, int* my_id,
                                          float* my_logit, float* full_max, float* full_sum,
                                          bool need_full) {
  const int lane = threadIdx.x & 31;
  float v[MAXJ];
  uint64_t key[MAXJ];
#pragma unroll
  for (int j = 0; j < MAXJ; ++j) {
    const int e = lane + 32 * j;
    v[j] = (e < E) ? row[e] : 0.0f;
    key[j] = (e < E) ? ((static_cast<uint64_t>(ordered_bits(v[j])) << 32) | static_cast<uint32_t>(~e)) : 0ull;
  }
  int sel_id = 0;
  float sel_v = 0.0f;
  for (int j = 0; j < k; ++j) {
    uint64_t best = 0;
    float bv = 0.0f;
#pragma unroll
    for (int q = 0; q < MAXJ; ++q) {
      if (key[q] > best) {
        best = key[q];
        bv = v[q];
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const uint64_t ob = __shfl_xor_sync(0xffffffffu, best, o);
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      if (ob > best) {
        best = ob;
        bv = ov;
      }
    }
    const int id = static_cast<int>(~static_cast<uint32_t>(best & 0xffffffffu));
#pragma unroll
    for (int q = 0; q < MAXJ; ++q)
      if (key[q] == best) key[q] = 0;  // taken
    if (lane == j) {
      sel_id = id;
      sel_v = bv;
    }
  }
  *my_id = sel_id;
  *my_logit = sel_v;
  if (need_full) {
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < MAXJ; ++q)
      if (lane + 32 * q < E) m = fmaxf(m, v[q]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.0f;
#pragma unroll
    for (int q = 0; q < MAXJ; ++q)
      if (lane + 32 * q < E) s += expf(v[q] - m);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    *full_max = m;
    *full_sum = s;
  }
}

// Top-k of token t by one warp; writes ids/w and returns the lane's id (lane < k).
template <int MAXJ>
__device__ __forceinline__ int route_token(const float* __restrict__ logits, int64_t t, int E, int k,
                                           bool renormalize, int32_t* __restrict__ ids,
                                           float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  int id;
  float lv, fmax = 0.0f, fsum = 1.0f;
  warp_topk<MAXJ>(logits + t * E, E, k, &id, &lv, &fmax, &fsum, !renormalize);
  const float l0 = __shfl_sync(0xffffffffu, lv, 0);
  float ex;
  if (renormalize) {
    ex = (lane < k) ? expf(lv - l0) : 0.0f;
    float s = ex;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    ex = ex / s;
  } else {
    ex = expf(lv - fmax) / fsum;
  }
  if (lane < k) {
    ids[t * k + lane] = id;
    w[t * k + lane] = ex;
  }
  return id;
}

}  // namespace e4b
