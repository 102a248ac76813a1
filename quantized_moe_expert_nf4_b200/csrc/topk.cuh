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

__device__ __forceinline__ float from_ordered_bits(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// One warp selects the top k of row `logits[0..E)`; lane j < k receives the
// j-th expert id and its logit.  Each lane holds MAXJ = ceil(E / 32) logits as
// order-preserving 32-bit keys.  Per selection: the warp maximum of the keys
// (__reduce_max_sync), then the lowest expert index holding that key
// (__reduce_min_sync) -- the (value descending, index ascending) order exactly.
template <int MAXJ>
__device__ __forceinline__ void warp_topk(const float* __restrict__ row, int E, int k, int* my_id,
                                          float* my_logit, float* full_max, float* full_sum,
                                          bool need_full) {
  const int lane = threadIdx.x & 31;
  uint32_t key[MAXJ];
  uint32_t live = 0;  // bit q: entry lane + 32q is a valid, not yet selected expert
#pragma unroll
  for (int q = 0; q < MAXJ; ++q) {
    const int e = lane + 32 * q;
    key[q] = (e < E) ? ordered_bits(row[e]) : 0u;
    if (e < E) live |= 1u << q;
  }
  int sel_id = 0;
  float sel_v = 0.0f;
  for (int j = 0; j < k; ++j) {
    uint32_t m = 0;
#pragma unroll
    for (int q = 0; q < MAXJ; ++q)
      if (((live >> q) & 1u) && key[q] > m) m = key[q];
    // A live entry can have key 0 only for a NaN pattern; it still takes part
    // through the index step below.
    const uint32_t wm = __reduce_max_sync(0xffffffffu, m);
    uint32_t idx = 0xffffffffu;
#pragma unroll
    for (int q = 0; q < MAXJ; ++q)
      if (((live >> q) & 1u) && key[q] == wm) {
        idx = static_cast<uint32_t>(lane + 32 * q);
        break;
      }
    const uint32_t wi = __reduce_min_sync(0xffffffffu, idx);
    if (static_cast<int>(wi & 31u) == lane) live &= ~(1u << (wi >> 5));
    if (lane == j) {
      sel_id = static_cast<int>(wi);
      sel_v = from_ordered_bits(wm);
    }
  }
  *my_id = sel_id;
  *my_logit = sel_v;
  if (need_full) {
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < MAXJ; ++q)
      if (lane + 32 * q < E) mx = fmaxf(mx, from_ordered_bits(key[q]));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float s = 0.0f;
#pragma unroll
    for (int q = 0; q < MAXJ; ++q)
      if (lane + 32 * q < E) s += expf(from_ordered_bits(key[q]) - mx);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    *full_max = mx;
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
