// Input gradient of the grouped NF4 GEMM: one launch over all groups.
//
// Fine-tuning per-expert adapters over a frozen NF4 stack needs, in backward,
// the gradient of each routed row's input through the frozen base:
// dX[p, :] = dY[row(p), :] . W_e, with W_e decoded again from the packed bytes
// (no dequantised expert is kept between passes), plus the adapter's share
// lora_scale * (dY[row(p)] . B_e) . A_e.  The pages route this through a single
// dgrad launch instead of a per-expert decode loop (experts4bit-qlora 0.22.0,
// "Which training path?").
//
// Warp-MMA kernel (mma.sync m16n8k16, bf16 -> fp32).  A CTA tile is 64 columns
// k of dX (the MMA's M dimension, 16 per warp: the rows of W_e^T) by 64 routed
// rows (N, 8 per MMA); the contraction runs over the N dimension of W in steps
// of 64.  The tile's 64 columns are one absmax block of every weight row, so a
// weight row n contributes one scale per step.  Per step the packed tile (64
// rows n x 32 bytes) and the dY tile (64 routed rows x 64 n) are copied into
// shared memory asynchronously (double-buffered), then the packed tile is
// decoded transposed: a thread takes 8 rows n and 4 columns k, interleaves the
// nibbles of row pairs (n, n+1) so that one byte holds the codes of one column
// k of both rows, turns each byte into a bf16 pair through a 256-entry table,
// scales it by (absmax[n], absmax[n+1]) and stores 8 rows n of one column k as
// one 16-byte run of W^T.  The contraction order inside a 32-wide chunk is
// permuted identically on both operands: lane t of a quad owns n in [8t, 8t+8).
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

constexpr int kTileK = 64;     // columns k of dX per CTA tile (= one absmax block)
constexpr int kTileT = 64;     // routed rows per CTA tile
constexpr int kStep = 64;      // contraction (n) per step
constexpr int kRowStride = 72;  // bf16 per shared row of W^T and of dY (144 B: conflict-free)
constexpr int kThreads = 128;   // 4 warps x 16 columns k

__device__ __forceinline__ void mma_16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async(void* smem, const void* gmem, int bytes_valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(bytes_valid));
}
__device__ __forceinline__ void cp_async_4(void* smem, const void* gmem, int bytes_valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(s), "l"(gmem), "r"(bytes_valid));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }

__global__ void __launch_bounds__(kThreads) grouped_nf4_dgrad_kernel(DgradArgs a) {
  __shared__ uint32_t lut[256];  // byte (hi code, lo code) -> bf16x2 (cb[hi] low half, cb[lo] high half)
  __shared__ __align__(16) uint16_t ys[2][kTileT * kRowStride];   // dY tile
  __shared__ __align__(16) uint16_t wt[kTileK * kRowStride];      // W^T tile (rows k, n contiguous)
  __shared__ __align__(16) uint8_t pk[2][kStep * 32];             // packed tile: 64 rows n x 32 bytes
  __shared__ __align__(16) float am[2][kStep];                    // absmax of the 64 rows n
  __shared__ int32_t rows_s[kTileT];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;

  int e;
  int64_t row_begin, row_end;
  if (!find_group_tile(a.offsets, a.E, a.total_rows, kTileT, blockIdx.x, &e, &row_begin, &row_end)) return;

  for (int b = tid; b < 256; b += kThreads) lut[b] = pack_bf16x2(codebook_entry(a.quant, b >> 4), codebook_entry(a.quant, b & 15));
  const int nrows = static_cast<int>(row_end - row_begin);
  for (int i = tid; i < kTileT; i += kThreads) {
    int64_t src = row_begin + i;
    if (i < nrows) {
      if (a.row_index) src = a.row_index[src];
      src = clampv<int64_t>(src, 0, a.dy_rows - 1);
    } else {
      src = -1;
    }
    rows_s[i] = static_cast<int32_t>(src);
  }
  __syncthreads();

  const int N = a.N, K = a.K;
  const int kt = blockIdx.y;                 // column tile: k in [64 kt, 64 kt + 64), absmax block kt
  const int KB = K / 64;
  const int nsteps = N / kStep;
  const int64_t wrow0 = static_cast<int64_t>(e) * N;

  auto load_step = [&](int s, int buf) {
    // dY: 64 rows x 8 chunks of 16 B (4 per thread)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = tid + j * kThreads;
      const int r = c >> 3, ch = c & 7;
      const int src = rows_s[r];
      const uint16_t* gp = a.dY + (src < 0 ? 0 : static_cast<int64_t>(src) * a.lddy) + s * kStep + ch * 8;
      cp_async(&ys[buf][r * kRowStride + ch * 8], gp, src >= 0 ? 16 : 0);
    }
    // packed: 64 rows x 2 chunks of 16 B (one per thread); absmax: one float per row
    {
      const int r = tid >> 1, ch = tid & 1;
      const uint8_t* gp = a.packed + (wrow0 + s * kStep + r) * (K / 2) + kt * 32 + ch * 16;
      cp_async(&pk[buf][r * 32 + ch * 16], gp, 16);
    }
    if (tid < kStep) cp_async_4(&am[buf][tid], a.absmax + (wrow0 + s * kStep + tid) * KB + kt, 4);
    cp_async_commit();
  };

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

  // Decoder role of this thread: rows n in [8 o, 8 o + 8) and columns k in [4 q, 4 q + 4).
  const int o = tid & 7, q = tid >> 3;
  load_step(0, 0);
  for (int s = 0; s < nsteps; ++s) {
    const int buf = s & 1;
    cp_async_wait_all();
    __syncthreads();  // step s landed; every warp is done with W^T of step s - 1
    if (s + 1 < nsteps) load_step(s + 1, buf ^ 1);
    {
      // Transposed decode of step s into W^T.
      uint32_t col[4][4];  // [column c][row pair j] = bf16x2 (row 8o+2j, row 8o+2j+1)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = 8 * o + 2 * j;
        const uint32_t x = *reinterpret_cast<const uint16_t*>(&pk[buf][n * 32 + 2 * q]);
        const uint32_t y = *reinterpret_cast<const uint16_t*>(&pk[buf][(n + 1) * 32 + 2 * q]);
        // byte 0 of x: codes of columns 4q (high nibble) and 4q+1; byte 1: 4q+2, 4q+3
        const uint32_t ev = (x & 0xF0F0u) | ((y >> 4) & 0x0F0Fu);         // columns 4q, 4q+2
        const uint32_t od = ((x << 4) & 0xF0F0u) | (y & 0x0F0Fu);         // columns 4q+1, 4q+3
        const __nv_bfloat162 sc = __floats2bfloat162_rn(am[buf][n], am[buf][n + 1]);
        const uint32_t v[4] = {lut[ev & 0xffu], lut[od & 0xffu], lut[(ev >> 8) & 0xffu], lut[(od >> 8) & 0xffu]};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          __nv_bfloat162 h2 = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&v[c]), sc);
          col[c][j] = *reinterpret_cast<uint32_t*>(&h2);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(&wt[(4 * q + c) * kRowStride + 8 * o]) =
            make_uint4(col[c][0], col[c][1], col[c][2], col[c][3]);
    }
    __syncthreads();  // W^T of step s complete
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      // rows g and g + 8 of this warp's 16 columns k, n in [32 ch + 8t, +8)
      const uint4 w0 = *reinterpret_cast<const uint4*>(&wt[(16 * warp + g) * kRowStride + 32 * ch + 8 * t]);
      const uint4 w1 = *reinterpret_cast<const uint4*>(&wt[(16 * warp + g + 8) * kRowStride + 32 * ch + 8 * t]);
      const uint32_t af0[4] = {w0.x, w1.x, w0.y, w1.y};
      const uint32_t af1[4] = {w0.z, w1.z, w0.w, w1.w};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const uint4 yv = *reinterpret_cast<const uint4*>(&ys[buf][(nt * 8 + g) * kRowStride + 32 * ch + 8 * t]);
        mma_16816(acc[nt], af0, yv.x, yv.y);
        mma_16816(acc[nt], af1, yv.z, yv.w);
      }
    }
  }

  // Epilogue.  acc[nt][0..1]: column k0 + g, routed rows 8nt + 2t, +1; acc[nt][2..3]: column k0 + g + 8.
  const int k0 = kt * kTileK + 16 * warp + g, k1 = k0 + 8;
  const bool lora = a.lora_A != nullptr && a.r > 0;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {
      const int tok = nt * 8 + 2 * t + qq;
      if (tok >= nrows) continue;
      const int64_t p = row_begin + tok;
      float v0 = acc[nt][qq], v1 = acc[nt][2 + qq];
      if (lora) {
        // + scale * sum_rho yb[p, rho] * lora_A[e, rho, k]
        const float* yb = a.yb + p * a.r;
        const uint16_t* la = a.lora_A + static_cast<int64_t>(e) * a.r * K;
        float d0 = 0.f, d1 = 0.f;
        for (int rr = 0; rr < a.r; ++rr) {
          const float yv = yb[rr];
          d0 = fmaf(yv, bf16_bits_to_float(la[static_cast<int64_t>(rr) * K + k0]), d0);
          d1 = fmaf(yv, bf16_bits_to_float(la[static_cast<int64_t>(rr) * K + k1]), d1);
        }
        v0 = fmaf(a.lora_scale, d0, v0);
        v1 = fmaf(a.lora_scale, d1, v1);
      }
      if (a.out_bf16) {
        static_cast<uint16_t*>(a.out)[p * K + k0] = float_to_bf16_bits(v0);
        static_cast<uint16_t*>(a.out)[p * K + k1] = float_to_bf16_bits(v1);
      } else {
        static_cast<float*>(a.out)[p * K + k0] = v0;
        static_cast<float*>(a.out)[p * K + k1] = v1;
      }
    }
  }
}

// LoRA factor of the adapter's share: yb[p, rho] = dY[row(p)] . lora_B[e][:, rho]
// (fp32), one warp per routed row; lane l takes n = l, l + 32, ...
__global__ void __launch_bounds__(256) dgrad_lora_yb_kernel(DgradArgs a) {
  constexpr int kMaxR = 16;
  const int lane = threadIdx.x & 31;
  const int64_t p = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (p >= a.total_rows) return;
  int lo = 0, hi = a.E - 1;  // group of p: last e with offsets[e] <= p
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.offsets[mid] <= p) lo = mid;
    else hi = mid - 1;
  }
  const int e = lo;
  int64_t src = a.row_index ? a.row_index[p] : p;
  src = clampv<int64_t>(src, 0, a.dy_rows - 1);
  const uint16_t* dy = a.dY + src * a.lddy;
  const uint16_t* lb = a.lora_B + static_cast<int64_t>(e) * a.N * a.r;
  float acc[kMaxR];
#pragma unroll
  for (int rr = 0; rr < kMaxR; ++rr) acc[rr] = 0.f;
  for (int n = lane; n < a.N; n += 32) {
    const float d = bf16_bits_to_float(dy[n]);
#pragma unroll
    for (int rr = 0; rr < kMaxR; ++rr) {
      if (rr >= a.r) break;
      acc[rr] = fmaf(d, bf16_bits_to_float(lb[static_cast<int64_t>(n) * a.r + rr]), acc[rr]);
    }
  }
#pragma unroll
  for (int rr = 0; rr < kMaxR; ++rr) {
    if (rr >= a.r) break;
    float v = acc[rr];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) a.yb[p * a.r + rr] = v;
  }
}

// Adapter gradients of one grouped projection, from xa = x . A_e^T and
// yb = da . B_e (both [total_rows, r] fp32), summed over each group's rows in
// row order (deterministic).  One thread per output row n (dB) or column k
// (dA), r accumulators each; experts without rows write zeros.
__global__ void __launch_bounds__(128) lora_grad_b_kernel(LoraGradArgs a) {
  constexpr int kMaxR = 16;
  const int e = blockIdx.x;
  const int n = blockIdx.y * 128 + threadIdx.x;
  const int64_t lo = clampv<int64_t>(a.offsets[e], 0, a.total_rows);
  const int64_t hi = max(lo, clampv<int64_t>(a.offsets[e + 1], 0, a.total_rows));
  float acc[kMaxR];
#pragma unroll
  for (int rr = 0; rr < kMaxR; ++rr) acc[rr] = 0.f;
  if (n < a.N) {
    for (int64_t p = lo; p < hi; ++p) {
      const float d = bf16_bits_to_float(a.da[p * a.ldda + n]);
#pragma unroll
      for (int rr = 0; rr < kMaxR; ++rr) {
        if (rr >= a.r) break;
        acc[rr] = fmaf(d, a.xa[p * a.r + rr], acc[rr]);
      }
    }
    float* out = a.dB + (static_cast<int64_t>(e) * a.N + n) * a.r;
#pragma unroll
    for (int rr = 0; rr < kMaxR; ++rr) {
      if (rr >= a.r) break;
      out[rr] = a.lora_scale * acc[rr];
    }
  }
}

__global__ void __launch_bounds__(128) lora_grad_a_kernel(LoraGradArgs a) {
  constexpr int kMaxR = 16;
  const int e = blockIdx.x;
  const int k = blockIdx.y * 128 + threadIdx.x;
  const int64_t lo = clampv<int64_t>(a.offsets[e], 0, a.total_rows);
  const int64_t hi = max(lo, clampv<int64_t>(a.offsets[e + 1], 0, a.total_rows));
  float acc[kMaxR];
#pragma unroll
  for (int rr = 0; rr < kMaxR; ++rr) acc[rr] = 0.f;
  if (k < a.K) {
    for (int64_t p = lo; p < hi; ++p) {
      int64_t src = a.row_index ? a.row_index[p] : p;
      src = clampv<int64_t>(src, 0, a.x_rows - 1);
      const float xv = bf16_bits_to_float(a.x[src * a.ldx + k]);
#pragma unroll
      for (int rr = 0; rr < kMaxR; ++rr) {
        if (rr >= a.r) break;
        acc[rr] = fmaf(a.yb[p * a.r + rr], xv, acc[rr]);
      }
    }
#pragma unroll
    for (int rr = 0; rr < kMaxR; ++rr) {
      if (rr >= a.r) break;
      a.dA[(static_cast<int64_t>(e) * a.r + rr) * a.K + k] = a.lora_scale * acc[rr];
    }
  }
}

}  // namespace

cudaError_t launch_dgrad_lora_yb(const DgradArgs& a, cudaStream_t stream) {
  if (a.total_rows == 0) return cudaSuccess;
  const int grid = static_cast<int>((a.total_rows * 32 + 255) / 256);
  LaunchScope ls("dgrad.lora_yb", stream);
  dgrad_lora_yb_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_lora_grads(const LoraGradArgs& a, cudaStream_t stream) {
  {
    dim3 grid(static_cast<unsigned>(a.E), static_cast<unsigned>((a.N + 127) / 128));
    LaunchScope ls("lora_grad.b", stream);
    lora_grad_b_kernel<<<grid, 128, 0, stream>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  dim3 grid(static_cast<unsigned>(a.E), static_cast<unsigned>((a.K + 127) / 128));
  LaunchScope ls("lora_grad.a", stream);
  lora_grad_a_kernel<<<grid, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

size_t dgrad_workspace_yb_offset() { return 256; }
size_t dgrad_workspace_bytes(int64_t total_rows, int64_t N, int r) {
  return dgrad_workspace_gather_offset(total_rows, r) + static_cast<size_t>(total_rows) * N * sizeof(uint16_t);
}

size_t lora_grads_workspace_yb_offset(int64_t total_rows, int r) {
  return 256 + align_up(static_cast<size_t>(total_rows) * r * sizeof(float), 256);
}
size_t lora_grads_workspace_bytes(int64_t total_rows, int r) {
  return lora_grads_workspace_yb_offset(total_rows, r) + align_up(static_cast<size_t>(total_rows) * r * sizeof(float), 256);
}

namespace {
int dgrad_override() {
  const char* v = getenv("E4B_DGRAD");
  if (!v) return 0;
  if (!strcmp(v, "mma")) return 1;
  if (!strcmp(v, "tc")) return 2;
  return 0;
}
constexpr int64_t kTcMinRows = 512;

// The adapter's share after the tensor-core product (fp32 output):
// out[p, k] += scale * sum_rho yb[p, rho] * lora_A[e, rho, k].
__global__ void __launch_bounds__(256) dgrad_lora_add_kernel(DgradArgs a) {
  __shared__ float yb_s[16];
  __shared__ int e_s;
  const int64_t p = blockIdx.x;
  if (threadIdx.x == 0) {
    int lo = 0, hi = a.E - 1;  // group of p: last e with offsets[e] <= p
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.offsets[mid] <= p) lo = mid;
      else hi = mid - 1;
    }
    e_s = lo;
  }
  if (threadIdx.x < a.r) yb_s[threadIdx.x] = a.yb[p * a.r + threadIdx.x];
  __syncthreads();
  const int k = blockIdx.y * blockDim.x + threadIdx.x;
  if (k >= a.K) return;
  const uint16_t* la = a.lora_A + static_cast<int64_t>(e_s) * a.r * a.K + k;
  float d = 0.f;
  for (int rr = 0; rr < a.r; ++rr) d = fmaf(yb_s[rr], bf16_bits_to_float(la[static_cast<int64_t>(rr) * a.K]), d);
  float* o = static_cast<float*>(a.out) + p * a.K + k;
  *o = fmaf(a.lora_scale, d, *o);
}
}  // namespace

size_t dgrad_workspace_gather_offset(int64_t total_rows, int r) {
  return 256 + align_up(r > 0 ? static_cast<size_t>(total_rows) * r * sizeof(float) : 0, 256);
}

cudaError_t launch_grouped_dgrad(const DgradArgs& a, cudaStream_t stream, const char** path) {
  if (a.total_rows == 0) return cudaSuccess;
  const bool lora = a.lora_A && a.r > 0;
  if (lora) {
    cudaError_t err = launch_dgrad_lora_yb(a, stream);
    if (err != cudaSuccess) return err;
  }
  const int ov = dgrad_override();
  const bool tc_ok = dgrad_tc_supported(a, a.row_index ? a.N : a.lddy);
  const bool use_tc = ov == 2 || (ov == 0 && tc_ok && a.total_rows >= kTcMinRows);
  if (use_tc) {
    if (!tc_ok) return cudaErrorNotSupported;
    const uint16_t* dy = a.dY;
    int64_t rows = a.dy_rows, ld = a.lddy;
    if (a.row_index) {  // the tensor-core kernel reads dY rows as contiguous tiles
      cudaError_t err = launch_gather_rows(a.dY, a.dy_rows, a.lddy, a.row_index, a.total_rows, a.N, a.gathered, stream);
      if (err != cudaSuccess) return err;
      dy = a.gathered;
      rows = a.total_rows;
      ld = a.N;
    }
    cudaError_t err = launch_grouped_dgrad_tc(a, dy, rows, ld, a.err, stream);
    if (err != cudaSuccess) return err;
    if (lora) {
      dim3 grid(static_cast<unsigned>(a.total_rows), static_cast<unsigned>((a.K + 255) / 256));
      LaunchScope ls("dgrad.lora_add", stream);
      dgrad_lora_add_kernel<<<grid, 256, 0, stream>>>(a);
      err = cudaGetLastError();
      if (err != cudaSuccess) return err;
    }
    *path = "dgrad.tc";
    return cudaSuccess;
  }
  // Upper bound on routed-row tiles: ceil(total/64) + number of non-empty groups.
  const int64_t gx = (a.total_rows + kTileT - 1) / kTileT + (a.E < a.total_rows ? a.E : a.total_rows);
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(a.K / kTileK));
  LaunchScope ls("dgrad.mma", stream);
  grouped_nf4_dgrad_kernel<<<grid, kThreads, 0, stream>>>(a);
  *path = "dgrad.mma";
  return cudaGetLastError();
}

}  // namespace e4b
