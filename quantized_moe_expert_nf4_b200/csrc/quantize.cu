// Blockwise 4-bit quantisation of a fused expert stack (load time): NF4, or FP4
// (e2m1 codes over 6) on the same layout.
//
// Follows "Why does load_in_4bit still OOM on a Mixture-of-Experts model?",
// section "Which project solves it": the stack is quantised expert by expert
// with blocks that never cross an expert boundary.  Because every expert holds
// N*K elements with (N*K) % 64 == 0, cutting the flattened [E, N*K] stack into
// consecutive blocks of 64 gives exactly the per-expert blocks.  The storage
// modes nf4 and fp4 are the two 4-bit packed ones of experts4bit-qlora 0.22.0
// (opening section).
//
// Per block: absmax a = max |w| (exact in fp32); s = w / a as one IEEE fp32
// division; level = number of decision thresholds T[l] <= s, where T[l] is the
// smallest float above the exact midpoint of the ascending distinct codebook
// values l and l+1 (so a value exactly on a midpoint takes the lower level);
// the code written is the level's code (NF4: the level itself; FP4: the
// sign-magnitude code, +0 for zero); a = 0 gives the code of 0.
//
// The kernel finds the level of s by one lookup in a table of 128 cells over
// [-1, 1] (the threshold inside the cell and the codes on either side of it)
// and decides most weights on w * fl32(1 / a), keeping the exact division for
// the few that fall within 2^-22 of a threshold (see code_of).
//
// HBM-bound: 4 B (fp32) or 2 B (bf16) read + 0.5625 B written per weight.  One
// warp handles 8 blocks (512 weights) per step with 16-byte loads; each block
// is reduced by a 16-lane shuffle tree.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>

#include "common.cuh"
#include "e4b_internal.h"

namespace e4b {

const float kCodebooks[2][16] = {{E4B_NF4_CODEBOOK_VALUES}, {E4B_FP4_CODEBOOK_VALUES}};

QuantTables quant_tables(int quant) {
  QuantTables qt{};
  const float* cb = kCodebooks[quant];
  // Distinct values, ascending; each keeps the lowest code that holds it
  // (+0 and -0 compare equal, so FP4 zero is code 0).
  float lv[16];
  uint32_t lc[16];
  int n = 0;
  for (int c = 0; c < 16; ++c) {
    bool seen = false;
    for (int i = 0; i < n; ++i) seen = seen || lv[i] == cb[c];
    if (!seen) {
      lv[n] = cb[c] == 0.0f ? 0.0f : cb[c];
      lc[n] = static_cast<uint32_t>(c);
      ++n;
    }
  }
  for (int i = 1; i < n; ++i)  // insertion sort by value
    for (int j = i; j > 0 && lv[j - 1] > lv[j]; --j) {
      std::swap(lv[j - 1], lv[j]);
      std::swap(lc[j - 1], lc[j]);
    }
  for (int l = 0; l < 16; ++l) {
    qt.code[l] = l < n ? lc[l] : lc[n - 1];
    qt.t[l] = std::numeric_limits<float>::infinity();
  }
  for (int l = 0; l + 1 < n; ++l) {
    // Exact in double: sum of two floats, then an exact halving.
    const double mid = (static_cast<double>(lv[l]) + static_cast<double>(lv[l + 1])) * 0.5;
    float f = static_cast<float>(mid);
    if (static_cast<double>(f) <= mid) f = std::nextafter(f, std::numeric_limits<float>::infinity());
    qt.t[l] = f;
  }
  qt.zero_code = 0;
  for (int l = 0; l < n; ++l)
    if (lv[l] == 0.0f) qt.zero_code = lc[l];
  return qt;
}

QuantCellTable quant_cell_table(int quant) {
  const QuantTables qt = quant_tables(quant);
  int nthr = 0;
  while (nthr < 16 && std::isfinite(qt.t[nthr])) ++nthr;
  QuantCellTable ct{};
  ct.ok = 1;
  for (int c = 0; c < kQuantCells; ++c) {
    const double lo = c / 64.0 - 1.0 - kQuantCellSlack, hi = (c + 1) / 64.0 - 1.0 + kQuantCellSlack;
    int base = 0;  // thresholds at or below every s of the cell
    while (base < nthr && static_cast<double>(qt.t[base]) <= lo) ++base;
    float t = std::numeric_limits<float>::infinity();
    if (base < nthr && static_cast<double>(qt.t[base]) <= hi) {
      t = qt.t[base];
      if (base + 1 < nthr && static_cast<double>(qt.t[base + 1]) <= hi) ct.ok = 0;
    }
    uint32_t tb;
    std::memcpy(&tb, &t, sizeof tb);
    ct.cell[c] = make_uint2(tb, qt.code[base] | (qt.code[std::min(base + 1, nthr)] << 4));
  }
  ct.zero_code = qt.zero_code;
  return ct;
}

namespace {

// The code of weight w in a block with absmax a > 0.  The method's scaled value
// is s = fl32(w / a) (one IEEE division).  For a in [2^-125, 2^125] the kernel
// first forms s' = fl32(w * y) with y = fl32(1 / a) computed once per block:
// |s' - w/a| <= 2^-23 |w/a| + 2^-48 and |s - w/a| <= 2^-25, so |s' - s| < 2^-22
// for |w| <= a.  When s' lies farther than 2^-22 from the cell's threshold
// (tested on the rounded difference, which only errs towards the exact path),
// s and s' fall on the same side of it and s' decides the code; otherwise, and
// for absmax outside that range, the code is decided on s itself.  The cell
// index is only a hint: every s and s' of a cell lies inside its widened range.
__device__ __forceinline__ uint32_t code_of(float w, float a, float y, bool fast, const uint2* cells) {
  float s = fast ? __fmul_rn(w, y) : __fdiv_rn(w, a);
  const int c = min(max(__float2int_rd((s + 1.0f) * 64.0f), 0), kQuantCells - 1);
  const uint2 e = cells[c];
  const float t = __uint_as_float(e.x);
  if (fast && !(fabsf(__fsub_rn(s, t)) > 0x1p-22f)) s = __fdiv_rn(w, a);
  return (s >= t ? e.y >> 4 : e.y) & 15u;
}

template <bool kBf16>
__device__ __forceinline__ void load4(const void* W, int64_t elem, float v[4]) {
  if constexpr (kBf16) {
    const uint2 raw = __ldcs(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(W) + elem));
    v[0] = __uint_as_float(raw.x << 16);
    v[1] = __uint_as_float(raw.x & 0xffff0000u);
    v[2] = __uint_as_float(raw.y << 16);
    v[3] = __uint_as_float(raw.y & 0xffff0000u);
  } else {
    const float4 f = __ldcs(reinterpret_cast<const float4*>(static_cast<const float*>(W) + elem));
    v[0] = f.x;
    v[1] = f.y;
    v[2] = f.z;
    v[3] = f.w;
  }
}

template <bool kBf16>
__global__ void __launch_bounds__(256) nf4_quantize_kernel(const void* __restrict__ W, int64_t nblocks,
                                                           uint8_t* __restrict__ packed,
                                                           float* __restrict__ absmax, QuantCellTable ct) {
  __shared__ uint2 cells_s[kQuantCells];
  for (int i = threadIdx.x; i < kQuantCells; i += blockDim.x) cells_s[i] = ct.cell[i];
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t ngroups = (nblocks + 7) / 8;  // 8 blocks = 512 weights per warp step

  for (int64_t g = warp; g < ngroups; g += nwarps) {
    float v[4][4];
    bool valid[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // Step i covers blocks 2i (lanes 0-15) and 2i+1 (lanes 16-31).
      const int64_t blk = g * 8 + 2 * i + (lane >> 4);
      valid[i] = blk < nblocks;
      const int64_t elem = g * 512 + 128 * i + 4 * lane;
      if (valid[i]) {
        load4<kBf16>(W, elem, v[i]);
      } else {
        v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0.0f;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float m = fmaxf(fmaxf(fabsf(v[i][0]), fabsf(v[i][1])), fmaxf(fabsf(v[i][2]), fabsf(v[i][3])));
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const bool fast = m >= 0x1p-125f && m <= 0x1p125f;
      const float y = __frcp_rn(m);  // IEEE reciprocal, used on the fast path only
      uint32_t q[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) q[j] = (m > 0.0f) ? code_of(v[i][j], m, y, fast, cells_s) : ct.zero_code;
      const int64_t blk = g * 8 + 2 * i + (lane >> 4);
      const int64_t elem = g * 512 + 128 * i + 4 * lane;
      if (valid[i]) {
        const uint16_t two = static_cast<uint16_t>(((q[0] << 4) | q[1]) | (((q[2] << 4) | q[3]) << 8));
        *reinterpret_cast<uint16_t*>(packed + elem / 2) = two;
        if ((lane & 15) == 0) absmax[blk] = m;
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize(const void* W, bool bf16, int64_t nblocks, int quant, uint8_t* packed, float* absmax,
                            cudaStream_t stream) {
  if (nblocks == 0) return cudaSuccess;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int64_t ngroups = (nblocks + 7) / 8;
  const int threads = 256;
  const int64_t want = (ngroups + (threads / 32) - 1) / (threads / 32);
  const int64_t cap = static_cast<int64_t>(di.sm_count) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  const QuantCellTable ct = quant_cell_table(quant);
  if (!ct.ok) return cudaErrorInvalidValue;
  LaunchScope ls("quantize", stream);
  if (bf16)
    nf4_quantize_kernel<true><<<grid, threads, 0, stream>>>(W, nblocks, packed, absmax, ct);
  else
    nf4_quantize_kernel<false><<<grid, threads, 0, stream>>>(W, nblocks, packed, absmax, ct);
  return cudaGetLastError();
}

}  // namespace e4b
