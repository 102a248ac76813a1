// Grouped NF4 GEMM on the 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
// The large-M (prefill / training-shaped) path of the grouped NF4 GEMM: the
// single-launch grouped kernel of the Solutions page's grouped-nf4-gemm row
// (gemm_4bit_grouped: nibbles decoded inside the mainloop, fp32 accumulation, no
// bf16 expert tensor in memory), laid out for sm_100a.
//
// Tile: 2 x 128 weight rows (the MMA's M; for SwiGLU the gate rows and the
// matching up rows, so the activation is computed in the epilogue from two
// accumulators of the same TMEM lanes) x 128 routed rows (the MMA's N) x K.
// One K step is one absmax block (64).  Warp roles, one persistent CTA per SM:
//   warp 12      TMA producer: packed nibbles (2-D tiled box 32 B x 128 rows per
//                half) and the 128 B operand rows -- a 2-D tiled box when the rows
//                are contiguous, four-row gathers (tile::gather4) through
//                row_index otherwise -- into a 4-stage ring;
//   warps 4-11   decoders: one weight row per thread; nibbles -> bf16 through a
//                per-lane-replicated byte -> bf16x2 codebook table, times the
//                block's absmax (bf16x2 multiply), stored in the canonical
//                128-byte-swizzled K-major layout the MMA reads (2-stage ring);
//   warp 13      TMEM allocator and MMA issuer (one thread): 4 x 2 MMAs
//                (M=128, N=128, K=16) per K step into a double-buffered pair of
//                accumulators (4 x 128 of the 512 TMEM columns);
//   warps 0-3    epilogue: TMEM -> registers (32 lanes x 32 columns at a time),
//                SwiGLU or plain store, overlapped with the next tile's mainloop.
// Every wait is bounded; TMEM is freed on every exit path.
#include <cuda.h>

#include "async.cuh"
#include "common.cuh"
#include "e4b_internal.h"
#include "tcgen05.cuh"

namespace e4b {
namespace {

constexpr int kBM = 128;           // weight rows per MMA (per half)
constexpr int kBN = 128;           // routed rows per tile
constexpr int kKS = 4;             // TMA ring stages
constexpr int kAS = 2;             // decoded-A ring stages
constexpr int kWarpDec = 4;        // warps 4..11
constexpr int kNumDecWarps = 8;
constexpr int kWarpTma = 12;
constexpr int kWarpMma = 13;
constexpr int kThreadsTc = 14 * 32;

constexpr uint32_t kPackedHalfBytes = kBM * 32;           // 128 rows x 32 B
constexpr uint32_t kPackedBytes = 2 * kPackedHalfBytes;   // 8 KB
constexpr uint32_t kBBytes = kBN * 128;                   // 16 KB
constexpr uint32_t kTmaStageBytes = kPackedBytes + kBBytes;
constexpr uint32_t kAHalfBytes = kBM * 128;               // 16 KB
constexpr uint32_t kAStageBytes = 2 * kAHalfBytes;
constexpr uint32_t kLutBytes = 256 * 32 * 4;

constexpr uint32_t kOffTma = 0;
constexpr uint32_t kOffA = kOffTma + kKS * kTmaStageBytes;
constexpr uint32_t kOffLut = kOffA + kAS * kAStageBytes;
constexpr uint32_t kOffBar = kOffLut + kLutBytes;
constexpr uint32_t kNumBars = 2 * kKS + 2 * kAS + 4;
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffRows = kOffTmemSlot + 16;
constexpr uint32_t kSmemBytes = kOffRows + kBN * 4 + 1024;  // + slack for 1024-B alignment

struct TcParams {
  const int32_t* offsets;
  int E;
  int64_t total_rows;
  const int32_t* row_index;  // gather rows of A (nullable: contiguous rows)
  int64_t a_rows;
  const float* absmax;
  int N, K;
  int swiglu;
  void* out;
  int out_bf16;
  int n_tiles;
  int* err;
};

__device__ __forceinline__ void tile_rows(const TcParams& p, int n_tile, int* r0, int* r1) {
  if (p.swiglu) {
    *r0 = n_tile * kBM;
    *r1 = p.N / 2 + n_tile * kBM;
  } else {
    *r0 = n_tile * 2 * kBM;
    *r1 = n_tile * 2 * kBM + kBM;
  }
}

// Tile t -> (group, routed-row range, n tile); warp-collective.
__device__ __forceinline__ bool locate(const TcParams& p, int64_t t, int* e, int64_t* rb, int64_t* re, int* n_tile) {
  const int64_t tok_tile_span = static_cast<int64_t>(kBN);
  int g;
  int64_t b0, b1;
  // Each group owns ceil(cnt / kBN) * n_tiles tiles: locate by (token tile, n tile).
  const int64_t q = t / p.n_tiles;
  if (!find_group_tile(p.offsets, p.E, p.total_rows, static_cast<int>(tok_tile_span), q, &g, &b0, &b1)) return false;
  *e = g;
  *rb = b0;
  *re = b1;
  *n_tile = static_cast<int>(t % p.n_tiles);
  return true;
}

__global__ void __launch_bounds__(kThreadsTc, 1)
    grouped_nf4_tc_kernel(const __grid_constant__ CUtensorMap tm_packed, const __grid_constant__ CUtensorMap tm_b,
                          TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* tma_full = bars;
  uint64_t* tma_empty = bars + kKS;
  uint64_t* a_full = bars + 2 * kKS;
  uint64_t* a_empty = a_full + kAS;
  uint64_t* acc_full = a_empty + kAS;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmemSlot);
  int32_t* rows_s = reinterpret_cast<int32_t*>(smem + kOffRows);
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + kOffLut);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = p.K / 64;

  if (tid == 0) {
    for (int s = 0; s < kKS; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&tma_empty[s], 1);
    }
    for (int s = 0; s < kAS; ++s) {
      mbar_init(&a_full[s], kNumDecWarps);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 4);
    }
    fence_mbar_init();
  }
  for (int i = tid; i < 256 * 32; i += blockDim.x) {
    const int b = i >> 5;
    lut[i] = pack_bf16x2(kNf4CodebookDev[b >> 4], kNf4CodebookDev[b & 15]);
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Total tiles: every CTA walks the same global list with a stride of gridDim.x.
  // A tile past the last group ends the walk (locate() returns false).
  if (warp == kWarpTma) {
    // ------------------------------------------------------------- producer
    uint32_t kbg = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok; t += gridDim.x) {
      int e, n_tile;
      int64_t rb, re;
      if (!locate(p, t, &e, &rb, &re, &n_tile)) break;
      int r0, r1;
      tile_rows(p, n_tile, &r0, &r1);
      const int32_t y0 = e * p.N + r0, y1 = e * p.N + r1;
      if (p.row_index) {
        // Row indices of this tile (rows past the group repeat a valid row).
        for (int i = lane; i < kBN; i += 32) {
          int64_t q = rb + i;
          if (q >= re) q = rb;
          int64_t src = p.row_index[q];
          src = src < 0 ? 0 : (src >= p.a_rows ? p.a_rows - 1 : src);
          rows_s[i] = static_cast<int32_t>(src);
        }
      }
      __syncwarp();
      int32_t rowv[kBN / 32];
      if (p.row_index) {
#pragma unroll
        for (int i = 0; i < kBN / 32; ++i) rowv[i] = rows_s[lane * (kBN / 32) + i];
      }
      for (int kb = 0; kb < KB; ++kb, ++kbg) {
        const int s = kbg % kKS;
        if (kbg >= kKS && !mbar_wait(&tma_empty[s], ((kbg / kKS) - 1) & 1)) {
          record_error(p.err, kErrWaitEmpty);
          ok = false;
          break;
        }
        unsigned char* st = smem + kOffTma + s * kTmaStageBytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&tma_full[s], kTmaStageBytes);
          tma_load_2d(st, &tm_packed, kb * 32, y0, &tma_full[s]);
          tma_load_2d(st + kPackedHalfBytes, &tm_packed, kb * 32, y1, &tma_full[s]);
          if (!p.row_index) tma_load_2d(st + kPackedBytes, &tm_b, kb * 64, static_cast<int32_t>(rb), &tma_full[s]);
        }
        __syncwarp();
        if (p.row_index) {
          // 32 gathers of 4 rows; lane l issues the gathers of rows 4l .. 4l+3.
          tma_gather4(st + kPackedBytes + lane * 4 * 128, &tm_b, kb * 64, rowv[0], rowv[1], rowv[2], rowv[3],
                      &tma_full[s]);
        }
        __syncwarp();
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
    uint32_t kbg = 0, j = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok; t += gridDim.x, ++j) {
      int e, n_tile;
      int64_t rb, re;
      if (!locate(p, t, &e, &rb, &re, &n_tile)) break;
      const int b = j & 1;
      if (j >= 2 && !mbar_wait(&acc_empty[b], ((j >> 1) - 1) & 1)) {
        record_error(p.err, kErrWaitEmpty);
        break;
      }
      tc_fence_after();
      const uint32_t d0 = tmem_base + (2 * b + 0) * kBN, d1 = tmem_base + (2 * b + 1) * kBN;
      for (int kb = 0; kb < KB; ++kb, ++kbg) {
        const int s = kbg % kKS, a = kbg % kAS;
        if (!mbar_wait(&a_full[a], (kbg / kAS) & 1) || !mbar_wait(&tma_full[s], (kbg / kKS) & 1)) {
          record_error(p.err, kErrWaitFull);
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_addr = smem_u32(smem + kOffA + a * kAStageBytes);
          const uint32_t b_addr = smem_u32(smem + kOffTma + s * kTmaStageBytes + kPackedBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (kb | kk) ? 1u : 0u;
            const uint64_t bd = smem_desc_sw128(b_addr + kk * 32);
            umma_bf16(d0, smem_desc_sw128(a_addr + kk * 32), bd, idesc, acc);
            umma_bf16(d1, smem_desc_sw128(a_addr + kAHalfBytes + kk * 32), bd, idesc, acc);
          }
          umma_commit(&tma_empty[s]);
          umma_commit(&a_empty[a]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&acc_full[b]);
      __syncwarp();
    }
  } else if (warp >= kWarpDec && warp < kWarpDec + kNumDecWarps) {
    // ------------------------------------------------------------- decoders
    const int r = tid - kWarpDec * 32;  // 0..255: weight row of the tile
    const int half = r >> 7, ri = r & 127;
    const uint32_t* lut_lane = lut + lane;
    uint32_t kbg = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok; t += gridDim.x) {
      int e, n_tile;
      int64_t rb, re;
      if (!locate(p, t, &e, &rb, &re, &n_tile)) break;
      int r0, r1;
      tile_rows(p, n_tile, &r0, &r1);
      const int n = (half ? r1 : r0) + ri;
      const bool valid = n < p.N;
      const float* am = p.absmax + (static_cast<int64_t>(e) * p.N + (valid ? n : 0)) * KB;
      float sc_next = valid ? __ldg(am) : 0.0f;
      for (int kb = 0; kb < KB; ++kb, ++kbg) {
        const int s = kbg % kKS, a = kbg % kAS;
        const float sc = sc_next;
        if (kb + 1 < KB) sc_next = valid ? __ldg(am + kb + 1) : 0.0f;
        if (!mbar_wait(&tma_full[s], (kbg / kKS) & 1) ||
            (kbg >= kAS && !mbar_wait(&a_empty[a], ((kbg / kAS) - 1) & 1))) {
          record_error(p.err, kErrWaitFull);
          ok = false;
          break;
        }
        const unsigned char* pk = smem + kOffTma + s * kTmaStageBytes + half * kPackedHalfBytes + ri * 32;
        const uint4 q0 = *reinterpret_cast<const uint4*>(pk);
        const uint4 q1 = *reinterpret_cast<const uint4*>(pk + 16);
        const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        const __nv_bfloat162 s2 = __float2bfloat162_rn(sc);
        unsigned char* arow = smem + kOffA + a * kAStageBytes + half * kAHalfBytes + (ri >> 3) * 1024 + (ri & 7) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // chunk c = k [8c, 8c+8) = one packed word
          const uint32_t w = words[c];
          uint32_t v[4];
#pragma unroll
          for (int by = 0; by < 4; ++by) {
            uint32_t pair = lut_lane[((w >> (8 * by)) & 0xffu) << 5];
            __nv_bfloat162 h2 = *reinterpret_cast<__nv_bfloat162*>(&pair);
            h2 = __hmul2(h2, s2);
            v[by] = *reinterpret_cast<uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(arow + ((c ^ (ri & 7)) << 4)) = make_uint4(v[0], v[1], v[2], v[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[a]);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------- epilogue
    const int q = warp;  // TMEM lane quadrant
    const int ri = q * 32 + lane;
    uint32_t j = 0;
    for (int64_t t = blockIdx.x;; t += gridDim.x, ++j) {
      int e, n_tile;
      int64_t rb, re;
      if (!locate(p, t, &e, &rb, &re, &n_tile)) break;
      const int b = j & 1;
      if (!mbar_wait(&acc_full[b], (j >> 1) & 1)) {
        record_error(p.err, kErrWaitFull);
        break;
      }
      tc_fence_after();
      int r0, r1;
      tile_rows(p, n_tile, &r0, &r1);
      const int nrows = static_cast<int>(re - rb);
      const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
      const uint32_t c0 = tmem_base + lane_off + (2 * b) * kBN, c1 = tmem_base + lane_off + (2 * b + 1) * kBN;
      if (p.swiglu) {
        const int n = r0 + ri;  // output column
        const int outN = p.N / 2;
        const bool valid = n < outN;
        for (int cc = 0; cc < kBN; cc += 32) {
          float g[32], u[32];
          tmem_ld_32x32b_x32(c0 + cc, g);
          tmem_ld_32x32b_x32(c1 + cc, u);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int tok = cc + i;
              if (tok < nrows) {
                const float hv = silu_f32(g[i]) * u[i];
                const int64_t o = (rb + tok) * outN + n;
                if (p.out_bf16)
                  static_cast<uint16_t*>(p.out)[o] = float_to_bf16_bits(hv);
                else
                  static_cast<float*>(p.out)[o] = hv;
              }
            }
          }
        }
      } else {
        for (int h = 0; h < 2; ++h) {
          const int n = (h ? r1 : r0) + ri;
          const bool valid = n < p.N;
          const uint32_t cb = h ? c1 : c0;
          for (int cc = 0; cc < kBN; cc += 32) {
            float v[32];
            tmem_ld_32x32b_x32(cb + cc, v);
            tmem_ld_wait();
            if (valid) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int tok = cc + i;
                if (tok < nrows) {
                  const int64_t o = (rb + tok) * p.N + n;
                  if (p.out_bf16)
                    static_cast<uint16_t*>(p.out)[o] = float_to_bf16_bits(v[i]);
                  else
                    static_cast<float*>(p.out)[o] = v[i];
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }
  // All roles are done (every MMA was waited on through acc_full): free TMEM.
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---- host side: tensor maps ---------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                 uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(const GemmArgs& a) {
  // No LoRA epilogue in the tensor-core kernel yet; K % 64 and N % 64 hold by contract.
  return a.lora_B == nullptr && a.lda % 8 == 0 && encode_fn() != nullptr;
}

cudaError_t launch_grouped_gemm_tc(const GemmArgs& a, int* err_word, cudaStream_t stream) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  static bool configured = false;
  if (!configured) {
    err = cudaFuncSetAttribute(grouped_nf4_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSmemBytes));
    if (err != cudaSuccess) return err;
    configured = true;
  }
  CUtensorMap tm_packed, tm_b;
  const uint64_t total_w_rows = static_cast<uint64_t>(a.E) * a.N;
  if (!make_map_2d(&tm_packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.packed, a.K / 2, total_w_rows, a.K / 2, 32, kBM,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const uint32_t box_rows = a.row_index ? 1u : static_cast<uint32_t>(kBN);
  if (!make_map_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.A, a.K, a.a_rows, a.lda * 2, 64, box_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.offsets = a.offsets;
  p.E = a.E;
  p.total_rows = a.total_rows;
  p.row_index = a.row_index;
  p.a_rows = a.a_rows;
  p.absmax = a.absmax;
  p.N = a.N;
  p.K = a.K;
  p.swiglu = a.epi == E4B_EPI_SWIGLU;
  p.out = a.out;
  p.out_bf16 = a.out_bf16;
  p.n_tiles = p.swiglu ? (a.N / 2 + kBM - 1) / kBM : (a.N + 2 * kBM - 1) / (2 * kBM);
  p.err = err_word;
  // Upper bound of the tile count: (ceil(rows / BN) + groups) * n_tiles.
  const int64_t tiles = ((a.total_rows + kBN - 1) / kBN + (a.E < a.total_rows ? a.E : a.total_rows)) * p.n_tiles;
  const int grid = static_cast<int>(tiles < di.sm_count ? tiles : di.sm_count);
  LaunchScope ls(p.swiglu ? "gemm.tc.swiglu" : "gemm.tc", stream);
  grouped_nf4_tc_kernel<<<grid, kThreadsTc, kSmemBytes, stream>>>(tm_packed, tm_b, p);
  return cudaGetLastError();
}

}  // namespace e4b
