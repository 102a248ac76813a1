// Grouped GEMM straight from MXFP4 expert bytes (e2m1 codes, e8m0 block scales).
//
// The pages multiply released MXFP4 experts (gpt-oss- and Kimi-class) on their
// e2m1 blocks and e8m0 scales, with no requantisation to NF4 and no bf16 copy
// of the weights (Solutions -- one page per problem, the gemm_mxfp4_grouped row
// of grouped-nf4-gemm).  Format (OCP microscaling): an e2m1 code is sign, two
// exponent bits (bias 1) and one mantissa bit (magnitudes 0, 0.5, 1, 1.5, 2,
// 3, 4, 6); one e8m0 byte x scales a block of 32 consecutive elements of a row
// by 2^(x - 127) (x = 255: NaN).  Layout per expert: row n of the [N, K]
// matrix holds K/2 code bytes (element 2i in the low nibble of byte i) and
// K/32 scale bytes.
//
// Warp-MMA kernel (mma.sync m16n8k16), the same "swap AB" tiling as the NF4
// one: 64 weight rows (the MMA's M, 16 per warp) by 64 routed rows (N), K in
// steps of 64.  Lane t of a quad owns physical k [8t, 8t+8) of each 32-wide
// chunk, so a chunk is exactly one scale block: the chunk's two MMAs
// accumulate the unscaled e2m1 values (exact in bf16) and the product is
// folded into the accumulator times the row's block scale in fp32.
#include "common.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

constexpr int kTileW = 64;     // weight rows per CTA tile
constexpr int kTileT = 64;     // routed rows per CTA tile
constexpr int kXStride = 96;   // bf16 per shared row of the routed-row tile (192 B: conflict-free)
constexpr int kThreads = 128;  // 4 warps x 16 weight rows

__device__ __forceinline__ void mma_16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async_16(void* smem, const void* gmem, bool pred) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int src_size = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_size));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }

// The value of an e2m1 code from its fields.
__device__ __forceinline__ float e2m1_value(int c) {
  const int e = (c >> 1) & 3, m = c & 1;
  const float mag = e == 0 ? 0.5f * m : __uint_as_float(static_cast<uint32_t>(126 + e) << 23) * (1.0f + 0.5f * m);
  return (c & 8) ? -mag : mag;
}

// 2^(x - 127) for an e8m0 byte (x = 0: the float32 subnormal 2^-127; x = 255: NaN).
__device__ __forceinline__ float e8m0_value(uint32_t x) {
  if (x == 255u) return __uint_as_float(0x7fc00000u);
  if (x == 0u) return __uint_as_float(0x00400000u);
  return __uint_as_float(x << 23);
}

__device__ __forceinline__ int weight_row(bool swiglu, int tile_y, int warp, int i, int N) {
  if (swiglu) {
    const int n = tile_y * (kTileW / 2) + warp * 8 + (i & 7);
    return (i < 8) ? n : (N / 2 + n);
  }
  return tile_y * kTileW + warp * 16 + i;
}

__global__ void __launch_bounds__(kThreads) grouped_mxfp4_mma_kernel(Mxfp4Args a) {
  __shared__ uint32_t lut[256];  // byte -> bf16x2 (low nibble's value, high nibble's value)
  __shared__ __align__(16) uint16_t xs[2][kTileT * kXStride];
  __shared__ int32_t rows_s[kTileT];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const bool swiglu = a.epi == E4B_EPI_SWIGLU;

  int e;
  int64_t row_begin, row_end;
  if (!find_group_tile(a.offsets, a.E, a.total_rows, kTileT, blockIdx.x, &e, &row_begin, &row_end)) return;

  for (int b = tid; b < 256; b += kThreads) lut[b] = pack_bf16x2(e2m1_value(b & 15), e2m1_value(b >> 4));
  const int nrows = static_cast<int>(row_end - row_begin);
  for (int i = tid; i < kTileT; i += kThreads) {
    int64_t src = row_begin + i;
    if (i < nrows) {
      if (a.row_index) src = a.row_index[src];
      src = clampv<int64_t>(src, 0, a.a_rows - 1);
    } else {
      src = -1;
    }
    rows_s[i] = static_cast<int32_t>(src);
  }
  __syncthreads();

  const int K = a.K, N = a.N;
  const int ksteps = K / 64, sblocks = K / 32;
  const int64_t expert_row0 = static_cast<int64_t>(e) * N;
  const int wr0 = weight_row(swiglu, blockIdx.y, warp, g, N);
  const int wr1 = weight_row(swiglu, blockIdx.y, warp, g + 8, N);
  const uint8_t* p0 = a.blocks + (expert_row0 + wr0) * (K / 2) + 4 * t;
  const uint8_t* p1 = a.blocks + (expert_row0 + wr1) * (K / 2) + 4 * t;
  const uint8_t* s0p = a.scales + (expert_row0 + wr0) * sblocks;
  const uint8_t* s1p = a.scales + (expert_row0 + wr1) * sblocks;

  auto load_x = [&](int kb, int buf) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = tid + j * kThreads;
      const int r = c >> 3, ch = c & 7;
      const int src = rows_s[r];
      const uint16_t* gp = a.A + (src < 0 ? 0 : static_cast<int64_t>(src) * a.lda) + kb * 64 + ch * 8;
      cp_async_16(&xs[buf][r * kXStride + ch * 8], gp, src >= 0);
    }
    cp_async_commit();
  };

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

  uint32_t wq[2][2];  // [row g / g+8][32-k chunk]
  float sc[2][2];     // [row][chunk]
  auto load_w = [&](int kb, uint32_t q[2][2], float s[2][2]) {
    const int off = kb * 32;
    q[0][0] = __ldg(reinterpret_cast<const uint32_t*>(p0 + off));
    q[0][1] = __ldg(reinterpret_cast<const uint32_t*>(p0 + off + 16));
    q[1][0] = __ldg(reinterpret_cast<const uint32_t*>(p1 + off));
    q[1][1] = __ldg(reinterpret_cast<const uint32_t*>(p1 + off + 16));
    s[0][0] = e8m0_value(__ldg(s0p + 2 * kb));
    s[0][1] = e8m0_value(__ldg(s0p + 2 * kb + 1));
    s[1][0] = e8m0_value(__ldg(s1p + 2 * kb));
    s[1][1] = e8m0_value(__ldg(s1p + 2 * kb + 1));
  };
  load_w(0, wq, sc);
  load_x(0, 0);

  for (int kb = 0; kb < ksteps; ++kb) {
    const int buf = kb & 1;
    cp_async_wait_all();
    __syncthreads();  // routed-row tile kb visible; buffer buf^1 free
    uint32_t nq[2][2] = {{0, 0}, {0, 0}};
    float nsc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    if (kb + 1 < ksteps) {
      load_x(kb + 1, buf ^ 1);
      load_w(kb + 1, nq, nsc);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint32_t w0 = wq[0][c], w1 = wq[1][c];
      // bytes of the word: physical k pairs (8t,8t+1), (8t+2,8t+3), (8t+4,8t+5), (8t+6,8t+7)
      const uint32_t afr0[4] = {lut[w0 & 0xff], lut[w1 & 0xff], lut[(w0 >> 8) & 0xff], lut[(w1 >> 8) & 0xff]};
      const uint32_t afr1[4] = {lut[(w0 >> 16) & 0xff], lut[(w1 >> 16) & 0xff], lut[w0 >> 24], lut[w1 >> 24]};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        float tmp[4] = {0.f, 0.f, 0.f, 0.f};
        const uint4 xv = *reinterpret_cast<const uint4*>(&xs[buf][(nt * 8 + g) * kXStride + c * 32 + 8 * t]);
        mma_16816(tmp, afr0, xv.x, xv.y);
        mma_16816(tmp, afr1, xv.z, xv.w);
        acc[nt][0] = fmaf(tmp[0], sc[0][c], acc[nt][0]);
        acc[nt][1] = fmaf(tmp[1], sc[0][c], acc[nt][1]);
        acc[nt][2] = fmaf(tmp[2], sc[1][c], acc[nt][2]);
        acc[nt][3] = fmaf(tmp[3], sc[1][c], acc[nt][3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        wq[i][c] = nq[i][c];
        sc[i][c] = nsc[i][c];
      }
  }

  // Epilogue.  acc[nt][0..1]: row g, routed rows 8nt+2t, +1; acc[nt][2..3]: row g+8.
  const int outN = swiglu ? N / 2 : N;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int tok = nt * 8 + 2 * t + q;
      if (tok >= nrows) continue;
      const int64_t p = row_begin + tok;
      const float v0 = acc[nt][q], v1 = acc[nt][2 + q];
      if (swiglu) {
        const float h = silu_f32(v0) * v1;
        if (a.out_bf16)
          static_cast<uint16_t*>(a.out)[p * outN + wr0] = float_to_bf16_bits(h);
        else
          static_cast<float*>(a.out)[p * outN + wr0] = h;
      } else if (a.out_bf16) {
        static_cast<uint16_t*>(a.out)[p * outN + wr0] = float_to_bf16_bits(v0);
        static_cast<uint16_t*>(a.out)[p * outN + wr1] = float_to_bf16_bits(v1);
      } else {
        static_cast<float*>(a.out)[p * outN + wr0] = v0;
        static_cast<float*>(a.out)[p * outN + wr1] = v1;
      }
    }
  }
}

}  // namespace

cudaError_t launch_grouped_mxfp4_gemm(const Mxfp4Args& a, cudaStream_t stream) {
  if (a.total_rows == 0) return cudaSuccess;
  const bool swiglu = a.epi == E4B_EPI_SWIGLU;
  const int rows_per_tile_w = swiglu ? kTileW / 2 : kTileW;
  const int gy = (swiglu ? a.N / 2 : a.N) / rows_per_tile_w;
  const int64_t gx = (a.total_rows + kTileT - 1) / kTileT + (a.E < a.total_rows ? a.E : a.total_rows);
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  LaunchScope ls(swiglu ? "mxfp4.mma.swiglu" : "mxfp4.mma", stream);
  grouped_mxfp4_mma_kernel<<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace e4b
