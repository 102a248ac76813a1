// Device helpers shared by the kernels of libe4b (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

// The NF4 codebook (QLoRA paper, Appendix E), ascending, entry 7 = 0.  One
// literal list serves the host table and the per-translation-unit device copy.
#define E4B_NF4_CODEBOOK_VALUES                                                             \
  -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,                 \
      -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,            \
      0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f,                     \
      0.33791524171829224f, 0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, \
      1.0f

// The FP4 codebook: code c is the e2m1 element (sign bit 3, exponent bits 2-1
// with bias 1, mantissa bit 0; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) divided by
// 6, each entry the float nearest to that ratio (the divisions below are
// correctly rounded).  Codes 0 and 8 are both zero.
#define E4B_FP4_CODEBOOK_VALUES                                                                          \
  0.0f, 0.5f / 6.0f, 1.0f / 6.0f, 1.5f / 6.0f, 2.0f / 6.0f, 3.0f / 6.0f, 4.0f / 6.0f, 1.0f, -0.0f,      \
      -0.5f / 6.0f, -1.0f / 6.0f, -1.5f / 6.0f, -2.0f / 6.0f, -3.0f / 6.0f, -4.0f / 6.0f, -1.0f

namespace e4b {

// The e2m1 element values themselves (MXFP4 codes, before their e8m0 block scale).
#define E4B_E2M1_VALUES \
  0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f, -0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f

// Indexed by storage: [0] NF4, [1] FP4 (the e4b_quant_type values), [2] MXFP4 e2m1.
static __device__ __constant__ float kCodebooksDev[3][16] = {
    {E4B_NF4_CODEBOOK_VALUES}, {E4B_FP4_CODEBOOK_VALUES}, {E4B_E2M1_VALUES}};

// Entry c (0..15) of the table of storage `quant` (0 NF4, 1 FP4, 2 MXFP4; others NF4).
__device__ __forceinline__ float codebook_entry(int quant, int c) {
  return kCodebooksDev[(quant == 1 || quant == 2) ? quant : 0][c & 15];
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Two floats -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + __expf(-z)); }

template <typename T>
__device__ __forceinline__ T clampv(T v, T lo, T hi) {
  return v < lo ? lo : (v > hi ? hi : v);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Inclusive warp scan of ints.
__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Locate the work tile `tile` among groups: group e owns ceil(cnt_e / rows_per_tile)
// consecutive tiles, cnt_e = clamp(offsets[e+1]) - clamp(offsets[e]).  Run by one
// full warp; every lane gets the same result.  Returns false if tile is past the end.
__device__ __forceinline__ bool find_group_tile(const int32_t* __restrict__ offsets, int E,
                                                int64_t total_rows, int rows_per_tile, int64_t tile,
                                                int* group, int64_t* row_begin, int64_t* row_end) {
  const int lane = threadIdx.x & 31;
  int64_t carry = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    int64_t lo = 0, hi = 0;
    if (e < E) {
      lo = clampv<int64_t>(offsets[e], 0, total_rows);
      hi = clampv<int64_t>(offsets[e + 1], 0, total_rows);
      if (hi < lo) hi = lo;
    }
    const int t = static_cast<int>((hi - lo + rows_per_tile - 1) / rows_per_tile);
    const int incl = warp_inclusive_scan(t);
    const int excl = incl - t;
    const bool mine = (e < E) && (tile >= carry + excl) && (tile < carry + incl);
    const uint32_t b = __ballot_sync(0xffffffffu, mine);
    if (b) {
      const int src = __ffs(b) - 1;
      const int64_t first = carry + __shfl_sync(0xffffffffu, excl, src);
      const int64_t glo = __shfl_sync(0xffffffffu, lo, src);
      const int64_t ghi = __shfl_sync(0xffffffffu, hi, src);
      *group = base + src;
      *row_begin = glo + (tile - first) * rows_per_tile;
      *row_end = min(ghi, *row_begin + rows_per_tile);
      return true;
    }
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  return false;
}

}  // namespace e4b
