// Grouped NF4 GEMM on warp-level tensor cores (mma.sync m16n8k16, bf16 -> fp32).
//
// Computes, for every row p of group e (expert_offsets), y[p, :] = A[row(p)] . W_e^T
// with W_e decoded from NF4 nibbles in registers -- the single-launch grouped
// GEMM of the Solutions page's grouped-nf4-gemm row (gemm_4bit_grouped): one
// launch over all groups, nibbles decoded inside the mainloop, fp32
// accumulation, no bf16 expert tensor in memory.  Epilogues: plain store, or
// the SwiGLU of the expert MLP with the optional per-expert LoRA delta added
// before the activation.
//
// This is the portable warp-MMA implementation; the tcgen05/TMEM kernel is the
// one the large-M forward runs.  It also serves the small-M grouped calls.
//
// Design ("swap AB"): weight rows are the MMA's M dimension (16 per warp) and
// routed tokens the N dimension (8 per MMA), so a group with few tokens wastes
// little.  A CTA tile is 64 weight rows x 64 tokens, one K step is one absmax
// block (64).  Per K step each 16-row MMA block accumulates the unscaled
// codebook values (bf16) into a fresh fp32 tile, which is then folded into the
// main accumulator times the row's absmax -- the scale is applied in fp32 once
// per block instead of once per weight.
//
// K order inside a 32-wide chunk is permuted consistently for both operands:
// lane t of a quad owns physical k in [8t, 8t+8), which is one 32-bit word of
// packed nibbles for A and one 16-byte vector of bf16 activations for B.
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

constexpr int kTileW = 64;     // weight rows per CTA tile
constexpr int kTileT = 64;     // tokens per CTA tile
constexpr int kXStride = 96;   // bf16 elements per smem row of the token tile (192 B: conflict-free)
constexpr int kThreads = 128;  // 4 warps x 16 weight rows

__device__ __forceinline__ void mma_bf16_16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
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

// Weight row (global, within the expert) of row i (0..15) of warp w's MMA block.
__device__ __forceinline__ int weight_row(bool swiglu, int tile_y, int warp, int i, int N) {
  if (swiglu) {
    const int n = tile_y * (kTileW / 2) + warp * 8 + (i & 7);
    return (i < 8) ? n : (N / 2 + n);
  }
  return tile_y * kTileW + warp * 16 + i;
}

__global__ void __launch_bounds__(kThreads) grouped_nf4_mma_kernel(GemmArgs a) {
  __shared__ uint32_t lut[256];                          // byte -> bf16x2 (cb[hi], cb[lo])
  __shared__ __align__(16) uint16_t xs[2][kTileT * kXStride];
  __shared__ int32_t rows_s[kTileT];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const bool swiglu = a.epi == E4B_EPI_SWIGLU;

  int e;
  int64_t row_begin, row_end;
  // Every warp resolves the tile (cheap; avoids a block barrier before the LUT).
  if (!find_group_tile(a.offsets, a.E, a.total_rows, kTileT, blockIdx.x, &e, &row_begin, &row_end)) return;

  // byte b = (code of the even element << 4) | code of the odd element
  for (int b = tid; b < 256; b += kThreads) lut[b] = pack_bf16x2(codebook_entry(a.quant, b >> 4), codebook_entry(a.quant, b & 15));
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
  const int kblocks = K / 64;
  const int64_t expert_row0 = static_cast<int64_t>(e) * N;
  // This thread's two weight rows: MMA rows g and g+8.
  const int wr0 = weight_row(swiglu, blockIdx.y, warp, g, N);
  const int wr1 = weight_row(swiglu, blockIdx.y, warp, g + 8, N);
  const uint8_t* p0 = a.packed + (expert_row0 + wr0) * (K / 2) + 4 * t;
  const uint8_t* p1 = a.packed + (expert_row0 + wr1) * (K / 2) + 4 * t;
  const float* s0p = a.absmax + (expert_row0 + wr0) * kblocks;
  const float* s1p = a.absmax + (expert_row0 + wr1) * kblocks;

  auto load_x = [&](int kb, int buf) {
    // 64 rows x 8 chunks of 16 B; 4 per thread.
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

  uint32_t wq[2][2];  // [row g / g+8][k32 chunk]
  float sc[2];
  wq[0][0] = __ldg(reinterpret_cast<const uint32_t*>(p0));
  wq[0][1] = __ldg(reinterpret_cast<const uint32_t*>(p0 + 16));
  wq[1][0] = __ldg(reinterpret_cast<const uint32_t*>(p1));
  wq[1][1] = __ldg(reinterpret_cast<const uint32_t*>(p1 + 16));
  sc[0] = __ldg(s0p);
  sc[1] = __ldg(s1p);
  load_x(0, 0);

  for (int kb = 0; kb < kblocks; ++kb) {
    const int buf = kb & 1;
    cp_async_wait_all();
    __syncthreads();  // X tile kb visible; buffer buf^1 free
    uint32_t nq[2][2] = {{0, 0}, {0, 0}};
    float nsc[2] = {0.f, 0.f};
    if (kb + 1 < kblocks) {
      load_x(kb + 1, buf ^ 1);
      const int off = (kb + 1) * 32;
      nq[0][0] = __ldg(reinterpret_cast<const uint32_t*>(p0 + off));
      nq[0][1] = __ldg(reinterpret_cast<const uint32_t*>(p0 + off + 16));
      nq[1][0] = __ldg(reinterpret_cast<const uint32_t*>(p1 + off));
      nq[1][1] = __ldg(reinterpret_cast<const uint32_t*>(p1 + off + 16));
      nsc[0] = __ldg(s0p + kb + 1);
      nsc[1] = __ldg(s1p + kb + 1);
    }
    float tmp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) tmp[i][0] = tmp[i][1] = tmp[i][2] = tmp[i][3] = 0.0f;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint32_t w0 = wq[0][c], w1 = wq[1][c];
      // bytes of the word: physical k pairs (8t,8t+1), (8t+2,8t+3), (8t+4,8t+5), (8t+6,8t+7)
      const uint32_t r0b0 = lut[w0 & 0xff], r0b1 = lut[(w0 >> 8) & 0xff];
      const uint32_t r0b2 = lut[(w0 >> 16) & 0xff], r0b3 = lut[w0 >> 24];
      const uint32_t r1b0 = lut[w1 & 0xff], r1b1 = lut[(w1 >> 8) & 0xff];
      const uint32_t r1b2 = lut[(w1 >> 16) & 0xff], r1b3 = lut[w1 >> 24];
      const uint32_t afr0[4] = {r0b0, r1b0, r0b1, r1b1};
      const uint32_t afr1[4] = {r0b2, r1b2, r0b3, r1b3};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const uint4 xv = *reinterpret_cast<const uint4*>(&xs[buf][(nt * 8 + g) * kXStride + c * 32 + 8 * t]);
        mma_bf16_16816(tmp[nt], afr0, xv.x, xv.y);
        mma_bf16_16816(tmp[nt], afr1, xv.z, xv.w);
      }
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      acc[nt][0] = fmaf(tmp[nt][0], sc[0], acc[nt][0]);
      acc[nt][1] = fmaf(tmp[nt][1], sc[0], acc[nt][1]);
      acc[nt][2] = fmaf(tmp[nt][2], sc[1], acc[nt][2]);
      acc[nt][3] = fmaf(tmp[nt][3], sc[1], acc[nt][3]);
    }
    wq[0][0] = nq[0][0];
    wq[0][1] = nq[0][1];
    wq[1][0] = nq[1][0];
    wq[1][1] = nq[1][1];
    sc[0] = nsc[0];
    sc[1] = nsc[1];
  }

  // Epilogue.  acc[nt][0..1]: row g, tokens 8nt+2t, +1; acc[nt][2..3]: row g+8.
  const bool lora = a.lora_B != nullptr && a.r > 0;
  const int outN = swiglu ? N / 2 : N;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int tok = nt * 8 + 2 * t + q;
      if (tok >= nrows) continue;
      const int64_t p = row_begin + tok;
      float v0 = acc[nt][q], v1 = acc[nt][2 + q];
      if (lora) {
        const float* xa = a.xa + p * a.r;
        const uint16_t* b0 = a.lora_B + (expert_row0 + wr0) * a.r;
        const uint16_t* b1 = a.lora_B + (expert_row0 + wr1) * a.r;
        float d0 = 0.f, d1 = 0.f;
        for (int rr = 0; rr < a.r; ++rr) {
          const float xv = xa[rr];
          d0 = fmaf(xv, bf16_bits_to_float(b0[rr]), d0);
          d1 = fmaf(xv, bf16_bits_to_float(b1[rr]), d1);
        }
        v0 = fmaf(a.lora_scale, d0, v0);
        v1 = fmaf(a.lora_scale, d1, v1);
      }
      if (swiglu) {
        const float h = silu_f32(v0) * v1;
        const int col = wr0;  // gate row index == output column
        if (a.out_bf16)
          static_cast<uint16_t*>(a.out)[p * outN + col] = float_to_bf16_bits(h);
        else
          static_cast<float*>(a.out)[p * outN + col] = h;
      } else {
        if (a.out_bf16) {
          static_cast<uint16_t*>(a.out)[p * outN + wr0] = float_to_bf16_bits(v0);
          static_cast<uint16_t*>(a.out)[p * outN + wr1] = float_to_bf16_bits(v1);
        } else {
          static_cast<float*>(a.out)[p * outN + wr0] = v0;
          static_cast<float*>(a.out)[p * outN + wr1] = v1;
        }
      }
    }
  }
}

// LoRA first factor: xa[p, :] = A[row(p)] . lora_A[e]^T (fp32), one warp per row:
// lanes stream 8 consecutive k (16-byte loads of the activation row and of each
// of the r adapter rows), then each of the r sums is reduced across the warp.
__global__ void __launch_bounds__(256) lora_xa_kernel(GemmArgs a) {
  constexpr int kMaxR = 16;
  const int lane = threadIdx.x & 31;
  const int64_t p = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (p >= a.total_rows) return;
  // group of p: last e with offsets[e] <= p (binary search, clamped)
  int lo = 0, hi = a.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.offsets[mid] <= p) lo = mid;
    else hi = mid - 1;
  }
  const int e = lo;
  int64_t src = a.row_index ? a.row_index[p] : p;
  src = clampv<int64_t>(src, 0, a.a_rows - 1);
  const uint16_t* x = a.A + src * a.lda;
  const uint16_t* la = a.lora_A + static_cast<int64_t>(e) * a.r * a.K;
  float acc[kMaxR];
#pragma unroll
  for (int rr = 0; rr < kMaxR; ++rr) acc[rr] = 0.f;
  for (int kk = lane * 8; kk < a.K; kk += 256) {
    const uint4 xv = *reinterpret_cast<const uint4*>(x + kk);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int rr = 0; rr < kMaxR; ++rr) {
      if (rr >= a.r) break;
      const uint4 av = *reinterpret_cast<const uint4*>(la + static_cast<int64_t>(rr) * a.K + kk);
      const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[rr] = fmaf(__uint_as_float(xw[i] << 16), __uint_as_float(aw[i] << 16), acc[rr]);
        acc[rr] = fmaf(__uint_as_float(xw[i] & 0xffff0000u), __uint_as_float(aw[i] & 0xffff0000u), acc[rr]);
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kMaxR; ++rr) {
    if (rr >= a.r) break;
    float v = acc[rr];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) a.xa[p * a.r + rr] = v;
  }
}

}  // namespace

cudaError_t launch_lora_xa(const GemmArgs& a, cudaStream_t stream) {
  if (a.total_rows == 0) return cudaSuccess;
  const int64_t warps = a.total_rows;
  const int grid = static_cast<int>((warps * 32 + 255) / 256);
  LaunchScope ls("gemm.lora_xa", stream);
  lora_xa_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemm_mma(const GemmArgs& a, cudaStream_t stream) {
  if (a.total_rows == 0) return cudaSuccess;
  const bool swiglu = a.epi == E4B_EPI_SWIGLU;
  const int rows_per_tile_w = swiglu ? kTileW / 2 : kTileW;
  const int gy = (swiglu ? a.N / 2 : a.N) / rows_per_tile_w;
  // Upper bound on token tiles: ceil(total/64) + number of non-empty groups.
  const int64_t gx = (a.total_rows + kTileT - 1) / kTileT + (a.E < a.total_rows ? a.E : a.total_rows);
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  LaunchScope ls(a.epi == E4B_EPI_SWIGLU ? "gemm.mma.swiglu" : "gemm.mma", stream);
  grouped_nf4_mma_kernel<<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace e4b

namespace e4b {

size_t gemm_workspace_xa_offset() { return 256; }
size_t gemm_workspace_gather_offset(int64_t total_rows, int r) {
  // 128 bytes per row hold either layout of the LoRA products (r <= 16).
  return 256 + align_up(r > 0 ? static_cast<size_t>(total_rows) * 128 : 0, 256);
}
size_t gemm_workspace_bytes(int64_t total_rows, int64_t K, int r) {
  return gemm_workspace_gather_offset(total_rows, r) + static_cast<size_t>(total_rows) * K * sizeof(uint16_t);
}

namespace {
// Which grouped GEMM kernel runs: the tensor-core (tcgen05) kernel for large
// row counts, the warp-MMA kernel otherwise.  E4B_GEMM=mma|tc forces one (tests,
// benchmarks); a forced kernel that cannot take the call is an error, never a
// silent switch.
int gemm_override() {
  const char* v = getenv("E4B_GEMM");
  if (!v) return 0;
  if (!strcmp(v, "mma")) return 1;
  if (!strcmp(v, "tc")) return 2;
  return 0;
}
constexpr int64_t kTcMinRows = 512;
}  // namespace

cudaError_t launch_grouped_mxfp4(const GemmArgs& a, const Mxfp4Args& m, cudaStream_t stream, const char** path) {
  const int ov = gemm_override();
  GemmArgs c = a;
  if (c.row_index && c.a_gathered) {
    c.A = c.a_gathered;
    c.a_rows = c.total_rows;
    c.lda = c.K;
    c.row_index = nullptr;
  }
  const bool swiglu = a.epi == E4B_EPI_SWIGLU;
  const bool tc_ok = a.quant == kQuantMxfp4 && a.mx_scales != nullptr && !a.lora_B && tc_supported(c);
  const bool use_tc = ov == 2 || (ov == 0 && tc_ok && a.total_rows >= kTcMinRows);
  if (use_tc) {
    if (!tc_ok) return cudaErrorNotSupported;
    if (a.row_index) {
      cudaError_t err = launch_gather_rows(a.A, a.a_rows, a.lda, a.row_index, a.total_rows, a.K, a.a_gathered, stream);
      if (err != cudaSuccess) return err;
    }
    *path = swiglu ? "mxfp4.tc.swiglu" : "mxfp4.tc";
    return launch_grouped_gemm_tc(c, c.err, stream);
  }
  *path = swiglu ? "mxfp4.mma.swiglu" : "mxfp4.mma";
  return launch_grouped_mxfp4_gemm(m, stream);
}

cudaError_t launch_grouped_gemm(const GemmArgs& a, cudaStream_t stream, const char** path) {
  const int ov = gemm_override();
  // The tensor-core kernel reads contiguous operand rows: a row_index call
  // gathers them into the workspace first.
  GemmArgs c = a;
  if (c.row_index && c.a_gathered) {
    c.A = c.a_gathered;
    c.a_rows = c.total_rows;
    c.lda = c.K;
    c.row_index = nullptr;
  }
  const bool tc_ok = tc_supported(c);
  const bool use_tc = ov == 2 || (ov == 0 && tc_ok && a.total_rows >= kTcMinRows);
  if (use_tc) {
    if (!tc_ok) return cudaErrorNotSupported;
    if (a.lora_B && a.r > 0) {
      cudaError_t err = launch_tc_lora_prep(a, stream);  // gathers too
      if (err != cudaSuccess) return err;
    } else if (a.row_index) {
      cudaError_t err = launch_gather_rows(a.A, a.a_rows, a.lda, a.row_index, a.total_rows, a.K, a.a_gathered, stream);
      if (err != cudaSuccess) return err;
    }
    *path = a.epi == E4B_EPI_SWIGLU ? "gemm.tc.swiglu" : "gemm.tc";
    return launch_grouped_gemm_tc(c, c.err, stream);
  }
  if (a.lora_B && a.r > 0) {
    cudaError_t err = launch_lora_xa(a, stream);
    if (err != cudaSuccess) return err;
  }
  *path = a.epi == E4B_EPI_SWIGLU ? "gemm.mma.swiglu" : "gemm.mma";
  return launch_grouped_gemm_mma(a, stream);
}

}  // namespace e4b
