// Grouped NF4 GEMM on the 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
// The large-M (prefill / training-shaped) path of the grouped NF4 GEMM: the
// single-launch grouped kernel of the Solutions page's grouped-nf4-gemm row
// (gemm_4bit_grouped: nibbles decoded inside the mainloop, fp32 accumulation, no
// bf16 expert tensor in memory), laid out for sm_100a.
//
// The routed activation rows of a group are contiguous here (the caller gathers
// them once, in routed order, before the launch): each K step loads them as one
// 2-D tiled TMA box, which the TMA engine moves far faster than per-row
// gathers of the same bytes.
//
// Tile: HALVES x 128 weight rows (the MMA's M, per half; for SwiGLU the gate
// rows and the matching up rows, so the activation is computed in the epilogue
// from two accumulators of the same TMEM lanes) x BN routed rows (the MMA's N,
// cut to the rows present in a group's last tile) x K, with NACC accumulator
// sets so that the epilogue of one tile can overlap the mainloop of the next
// (HALVES x BN x NACC <= the 512 TMEM columns).  One K step is one absmax
// block (64).  Warp roles, one persistent CTA per SM:
//   warp 20      TMA producer: packed nibbles (2-D tiled box 32 B x 128 rows per
//                half) and the 128 B x BN operand rows into a KS-stage ring;
//   warps 4-19   decoders: one weight row and 1/2 or 1/4 of a k block per thread;
//                nibbles -> bf16 in registers (byte permutes over the codebook's
//                low and high bytes, no table in shared memory), times the
//                block's absmax (bf16x2 multiply), stored in the canonical
//                128-byte-swizzled K-major layout the MMA reads (2-stage ring);
//   warp 21      TMEM allocator and MMA issuer (one thread): 4 x HALVES MMAs
//                (M=128, N<=BN, K=16) per K step;
//   warps 0-3    epilogue: TMEM -> registers (32 lanes x 16 columns at a time),
//                SwiGLU or plain, staged 32 routed rows at a time in shared
//                memory (double-buffered) and written by TMA tensor stores; a
//                group's ragged last rows are copied out with plain stores so
//                that no store reaches the next group's rows.
// Every wait is bounded; TMEM is freed on every exit path.
#include <cuda.h>

#include <cstdlib>
#include <cstring>

#include "async.cuh"
#include "common.cuh"
#include "e4b_internal.h"
#include "tcgen05.cuh"

namespace e4b {
namespace {

constexpr int kBM = 128;           // weight rows per MMA (per half)
constexpr int kWarpDec = 4;        // warps 4..19
constexpr int kNumDecWarps = 16;
constexpr int kDecThreads = kNumDecWarps * 32;
constexpr int kWarpTma = 20;
constexpr int kWarpMma = 21;
constexpr int kThreadsTc = 22 * 32;
constexpr uint32_t kPackedHalfBytes = kBM * 32;  // 128 rows x 32 B
constexpr uint32_t kAHalfBytes = kBM * 128;      // 128 rows x 64 bf16
constexpr int kChunk = 32;                         // routed rows per staged output chunk
constexpr uint32_t kOutChunkBytes = kChunk * kBM * 4;  // 32 rows x 128 columns x fp32
constexpr uint32_t kOutBytes = 2 * kOutChunkBytes;     // double-buffered
constexpr uint32_t kSmemLimit = 227 * 1024;
constexpr uint32_t kSmemMisc = 1024 + 512;       // alignment slack, barriers, TMEM slot
constexpr int kLoraCols = 64;                    // width of a row of scale * x . lora_A^T (bf16, zero past r)
constexpr size_t kLoraPrepSmemMax = 192 * 1024;  // lora_A[e] staged by the prep kernel

// ATMEM: the decoders write the decoded weight tile into tensor memory
// (tcgen05.st) and the MMA reads A from there, so the tile never passes
// through shared memory; the A stages take TMEM columns after the accumulators.
template <int BN_, int HALVES_, int NACC_, bool ATMEM_ = false>
struct TcShape {
  static constexpr int BN = BN_, HALVES = HALVES_, NACC = NACC_;
  static constexpr bool ATMEM = ATMEM_;
  static constexpr int kRows = HALVES * kBM;        // weight rows per tile
  static constexpr int kTpr = kDecThreads / kRows;  // decoder threads per weight row
  static constexpr int kChunks = 8 / kTpr;          // 16-byte decoded chunks per thread per k block
  static constexpr uint32_t kPackedBytes = HALVES * kPackedHalfBytes;
  static constexpr uint32_t kBBytes = BN * 128;
  static constexpr uint32_t kTmaStageBytes = kPackedBytes + kBBytes;
  static constexpr int kAS = 2;
  static constexpr uint32_t kAStageBytes = ATMEM ? 0 : HALVES * kAHalfBytes;
  static constexpr int kKSFit =
      static_cast<int>((kSmemLimit - kSmemMisc - kOutBytes - kAS * kAStageBytes) / kTmaStageBytes);
  static constexpr int kKS = kKSFit < 6 ? kKSFit : 6;
  static constexpr uint32_t kCols = HALVES * BN;    // TMEM columns of one accumulator set
  static constexpr uint32_t kACols = HALVES * 32;   // TMEM columns of one A stage (ATMEM): 64 k as bf16 pairs
  static constexpr uint32_t kAColBase = kCols * NACC;
  static constexpr uint32_t kOffTma = 0;
  static constexpr uint32_t kOffA = kOffTma + kKS * kTmaStageBytes;
  static constexpr uint32_t kOffOut = kOffA + kAS * kAStageBytes;
  static constexpr uint32_t kOffBar = kOffOut + kOutBytes;
  static constexpr uint32_t kNumBars = 2 * kKS + 2 * kAS + 2 * NACC + 1;
  static constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr uint32_t kSmemBytes = kOffTmemSlot + 16 + 1024;
  static_assert(kTpr == 2 || kTpr == 4, "decoder split");
  static_assert(kKS >= 2, "ring depth");
  static_assert(kCols * NACC + (ATMEM ? kAS * kACols : 0) <= 512, "TMEM columns");
  static_assert(!ATMEM || HALVES == 2, "the TMEM decoders cover two halves");
  static_assert(kChunks >= 1 && kAColBase <= 512, "decoder chunks, TMEM A base");
  static_assert(BN % 16 == 0 && BN <= 256, "MMA N");
  static_assert(kSmemBytes <= kSmemLimit, "shared memory");
};

struct TcParams {
  const int32_t* offsets;
  int E;
  int64_t total_rows;
  const float* absmax;
  int N, K;
  int swiglu;
  void* out;
  int out_bf16;
  int out_cols;  // columns of out: N, or N / 2 for SwiGLU
  int n_tiles;
  int* err;
  const uint16_t* lora_B;  // [E, N, r] bf16, or null (no LoRA step)
  int r;
  int quant;                 // e4b_quant_type of the packed codes, or kQuantMxfp4
  const uint8_t* mx_scales;  // kQuantMxfp4: [E*N, K/32] e8m0 scale bytes (absmax unused)
};

// The codebook's bf16 patterns split into low and high bytes, four entries per
// word: lo[j / 4] byte (j % 4) = low byte of bf16(codebook[j]).
struct CodebookBytes {
  uint32_t lo[4], hi[4];
};

__device__ __forceinline__ CodebookBytes codebook_bytes(int quant) {
  CodebookBytes t{};
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t b = float_to_bf16_bits(codebook_entry(quant, j));
    t.lo[j >> 2] |= (b & 0xffu) << (8 * (j & 3));
    t.hi[j >> 2] |= (b >> 8) << (8 * (j & 3));
  }
  return t;
}

// Final interleaves of decode4: the packed order of the two elements of a byte.
constexpr uint32_t kSelHiFirst0 = 0x4051u, kSelHiFirst1 = 0x6273u;  // element 2i in the high nibble (NF4, FP4)
constexpr uint32_t kSelLoFirst0 = 0x5140u, kSelLoFirst1 = 0x7362u;  // element 2i in the low nibble (MXFP4)

// Four nibbles (bits 0-15 of g: the low then the high nibble of two packed
// bytes) -> two bf16x2 words in element order.  A byte permute looks up
// entries 0-7 and 8-15 for all four nibbles at once (its selector takes the
// nibbles' low three bits); a second permute keeps, per nibble, the half its
// top bit names; a third interleaves the low and high bytes, in the byte's
// element order (sel0, sel1: kSelHiFirst* or kSelLoFirst*).
__device__ __forceinline__ void decode4(uint32_t g, const CodebookBytes& t, uint32_t* w0, uint32_t* w1,
                                        uint32_t sel0 = kSelHiFirst0, uint32_t sel1 = kSelHiFirst1) {
  const uint32_t s = g & 0x7777u;
  const uint32_t pick = ((g >> 1) & 0x4444u) | 0x3210u;  // field i: i, or i + 4 when nibble i >= 8
  const uint32_t lo = __byte_perm(__byte_perm(t.lo[0], t.lo[1], s), __byte_perm(t.lo[2], t.lo[3], s), pick);
  const uint32_t hi = __byte_perm(__byte_perm(t.hi[0], t.hi[1], s), __byte_perm(t.hi[2], t.hi[3], s), pick);
  *w0 = __byte_perm(lo, hi, sel0);  // (element 2i, element 2i+1)
  *w1 = __byte_perm(lo, hi, sel1);  // (element 2i+2, element 2i+3)
}

// 2^(x - 127) for an e8m0 scale byte, as a float (x = 0: the subnormal 2^-127;
// x = 255: NaN).  Exact, and exact again after rounding to bf16.
__device__ __forceinline__ float e8m0_scale(uint32_t x) {
  if (x == 255u) return __uint_as_float(0x7fc00000u);
  if (x == 0u) return __uint_as_float(0x00400000u);
  return __uint_as_float(x << 23);
}

// Weight rows of the tile's halves.
template <int HALVES>
__device__ __forceinline__ void tile_rows(const TcParams& p, int n_tile, int* r0, int* r1) {
  if (p.swiglu) {
    *r0 = n_tile * kBM;
    *r1 = p.N / 2 + n_tile * kBM;
  } else {
    *r0 = n_tile * HALVES * kBM;
    *r1 = *r0 + kBM;
  }
}

// Tile t -> (group, routed-row range, n tile); warp-collective.  Each group owns
// ceil(rows / BN) * n_tiles tiles, the n tile running fastest.
template <int BN>
__device__ __forceinline__ bool locate(const TcParams& p, int64_t t, int* e, int64_t* rb, int64_t* re,
                                       int* n_tile) {
  int g;
  int64_t b0, b1;
  if (!find_group_tile(p.offsets, p.E, p.total_rows, BN, t / p.n_tiles, &g, &b0, &b1)) return false;
  *e = g;
  *rb = b0;
  *re = b1;
  *n_tile = static_cast<int>(t % p.n_tiles);
  return true;
}

// Decoders of the TMEM-operand shape.  A warp may only reach the 32 TMEM lanes
// of its quadrant (warp % 4), so warp w takes weight rows 32 (w % 4) + lane of
// one half, and the four warps of a quadrant split (half, 32-k part); a thread
// decodes its row's 32 k of the step into 16 bf16 pairs and stores them as 16
// consecutive TMEM columns of its lane.
template <class S>
__device__ __forceinline__ void tmem_decoders(const TcParams& p, unsigned char* smem, uint64_t* tma_full,
                                              uint64_t* a_empty, uint64_t* a_full, uint32_t tmem_base, int warp,
                                              int lane) {
  constexpr int BN = S::BN, KS = S::kKS, AS = S::kAS;
  const int qd = warp & 3, c = (warp - kWarpDec) >> 2;
  const int half = c >> 1, kpart = c & 1;
  const int ri = qd * 32 + lane;
  const int KB = p.K / 64;
  const CodebookBytes cbt = codebook_bytes(p.quant);
  uint32_t kbg = 0;
  bool ok = true;
  for (int64_t t = blockIdx.x; ok; t += gridDim.x) {
    int e, n_tile;
    int64_t rb, re;
    if (!locate<BN>(p, t, &e, &rb, &re, &n_tile)) break;
    int r0, r1;
    tile_rows<S::HALVES>(p, n_tile, &r0, &r1);
    const int n = (half ? r1 : r0) + ri;
    const bool valid = n < p.N;
    const float* am = p.absmax + (static_cast<int64_t>(e) * p.N + (valid ? n : 0)) * KB;
    float sc_ring[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) sc_ring[i] = (valid && i < KB) ? __ldg(am + i) : 0.0f;
    for (int kb0 = 0; kb0 < KB && ok; kb0 += 4) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int kb = kb0 + i;
        if (kb >= KB) break;
        const float sc = sc_ring[i];
        sc_ring[i] = (valid && kb + 4 < KB) ? __ldg(am + kb + 4) : 0.0f;
        const int s = kbg % KS, a = kbg % AS;
        if (!mbar_wait(&tma_full[s], (kbg / KS) & 1) ||
            (kbg >= AS && !mbar_wait(&a_empty[a], ((kbg / AS) - 1) & 1))) {
          record_error(p.err, kErrWaitFull);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint4 q = *reinterpret_cast<const uint4*>(smem + S::kOffTma + s * S::kTmaStageBytes +
                                                        half * kPackedHalfBytes + ri * 32 + kpart * 16);
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
        const __nv_bfloat162 s2 = __float2bfloat162_rn(sc);
        uint32_t v[16];
#pragma unroll
        for (int cw = 0; cw < 4; ++cw) {
          decode4(words[cw], cbt, &v[4 * cw], &v[4 * cw + 1]);
          decode4(words[cw] >> 16, cbt, &v[4 * cw + 2], &v[4 * cw + 3]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          __nv_bfloat162 h2 = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&v[i]), s2);
          v[i] = *reinterpret_cast<uint32_t*>(&h2);
        }
        tmem_st_32x32b_x16(
            tmem_base + (static_cast<uint32_t>(qd * 32) << 16) + S::kAColBase + a * S::kACols + half * 32 + kpart * 16, v);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[a]);
        ++kbg;
      }
    }
  }
}

// Decoders of the dgrad product.  Thread dt takes rows n in [8o, 8o + 8) of the
// K step and columns k in [4q, 4q + 4) of the tile (q = 0..63: the tile's 256
// columns, o = 0..7).  The nibbles of row pairs (n, n+1) are interleaved so
// that one byte holds one column's codes of both rows; four such bytes decode
// (byte permutes) to the bf16 pairs (W[n][k], W[n+1][k]) of four columns,
// scaled by (absmax[n], absmax[n+1]) of their 64-column block.  Row k of the A
// tile (K-major, 128-byte swizzle) takes the 8 rows n as one 16-byte chunk.
template <class S>
__device__ __forceinline__ void dgrad_decoders(const TcParams& p, unsigned char* smem, uint64_t* tma_full,
                                               uint64_t* a_empty, uint64_t* a_full, int dt, int lane) {
  static_assert(S::HALVES == 2, "the dgrad decoders cover 256 columns per tile");
  constexpr int BN = S::BN, KS = S::kKS, AS = S::kAS;
  constexpr int kRowBytes = S::HALVES * 64;  // packed bytes of one row n in the tile
  const int q = (dt & 7) | (((dt >> 5) & 7) << 3);
  const int o = ((dt >> 3) & 3) | ((dt >> 8) << 2);
  const int KB = p.K / 64, kbw = p.N / 64;
  const CodebookBytes cbt = codebook_bytes(p.quant);
  uint32_t kbg = 0;
  bool ok = true;
  for (int64_t t = blockIdx.x; ok; t += gridDim.x) {
    int e, n_tile;
    int64_t rb, re;
    if (!locate<BN>(p, t, &e, &rb, &re, &n_tile)) break;
    int r0, r1;
    tile_rows<S::HALVES>(p, n_tile, &r0, &r1);
    const int kcol = r0 + 4 * q;  // first of this thread's four columns
    const bool valid = kcol < p.N;
    const float* am = p.absmax + (static_cast<int64_t>(e) * p.K + 8 * o) * kbw + (valid ? kcol / 64 : 0);
    float sc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sc[i] = valid ? __ldg(am + static_cast<int64_t>(i) * kbw) : 0.0f;
    for (int kb = 0; kb < KB && ok; ++kb) {
      float nsc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        nsc[i] = (valid && kb + 1 < KB) ? __ldg(am + static_cast<int64_t>((kb + 1) * 64 + i) * kbw) : 0.0f;
      const int s = kbg % KS, a = kbg % AS;
      if (!mbar_wait(&tma_full[s], (kbg / KS) & 1) ||
          (kbg >= AS && !mbar_wait(&a_empty[a], ((kbg / AS) - 1) & 1))) {
        record_error(p.err, kErrWaitFull);
        ok = false;
        break;
      }
      const unsigned char* src = smem + S::kOffTma + s * S::kTmaStageBytes;
      uint32_t col[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = 8 * o + 2 * j;
        const uint32_t x = *reinterpret_cast<const uint16_t*>(src + n * kRowBytes + 2 * q);
        const uint32_t y = *reinterpret_cast<const uint16_t*>(src + (n + 1) * kRowBytes + 2 * q);
        const uint32_t ev = (x & 0xF0F0u) | ((y >> 4) & 0x0F0Fu);  // columns 4q, 4q+2: (row n, row n+1) codes
        const uint32_t od = ((x << 4) & 0xF0F0u) | (y & 0x0F0Fu);  // columns 4q+1, 4q+3
        uint32_t v[4];
        decode4(ev, cbt, &v[0], &v[2]);
        decode4(od, cbt, &v[1], &v[3]);
        const __nv_bfloat162 s2 = __floats2bfloat162_rn(sc[2 * j], sc[2 * j + 1]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          __nv_bfloat162 h2 = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&v[c]), s2);
          col[c][j] = *reinterpret_cast<uint32_t*>(&h2);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int kl = 4 * q + c;  // A row: column k of the tile
        const int half = kl >> 7, ri = kl & 127;
        unsigned char* arow =
            smem + S::kOffA + a * S::kAStageBytes + half * kAHalfBytes + (ri >> 3) * 1024 + (ri & 7) * 128;
        *reinterpret_cast<uint4*>(arow + ((o ^ (ri & 7)) << 4)) = make_uint4(col[c][0], col[c][1], col[c][2], col[c][3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[a]);
      ++kbg;
#pragma unroll
      for (int i = 0; i < 8; ++i) sc[i] = nsc[i];
    }
  }
}

// DG: the input-gradient product (dgrad).  The tile's "weight rows" are then
// columns k of W (p.N = K of W), the K steps run over the rows n of W
// (p.K = N of W), the packed tile is 64 rows n x (HALVES * 64) bytes, and the
// decoders write W^T: row k of the A tile holds W[n][k] for the step's 64 n.
template <class S, bool DG>
__global__ void __launch_bounds__(kThreadsTc, 1)
    grouped_nf4_tc_kernel(const __grid_constant__ CUtensorMap tm_packed, const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_xa,
                          TcParams p) {
  constexpr int BN = S::BN, HALVES = S::HALVES, NACC = S::NACC, KS = S::kKS, AS = S::kAS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kOffBar);
  uint64_t* tma_full = bars;
  uint64_t* tma_empty = bars + KS;
  uint64_t* a_full = bars + 2 * KS;
  uint64_t* a_empty = a_full + AS;
  uint64_t* acc_full = a_empty + AS;
  uint64_t* acc_empty = acc_full + NACC;
  uint64_t* epi_bar = acc_empty + NACC;  // barrier of the four epilogue warps (bounded waits)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kOffTmemSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = p.K / 64;

  if (tid == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&tma_empty[s], 1);
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(&a_full[s], kNumDecWarps);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < NACC; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 4);
    }
    mbar_init(epi_bar, 4);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Every role walks the same tile list (stride gridDim.x); a tile past the
  // last group ends the walk.
  if (warp == kWarpTma) {
    // ------------------------------------------------------------- producer
    uint32_t kbg = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok; t += gridDim.x) {
      int e, n_tile;
      int64_t rb, re;
      if (!locate<BN>(p, t, &e, &rb, &re, &n_tile)) break;
      int r0, r1;
      tile_rows<HALVES>(p, n_tile, &r0, &r1);
      const int32_t y0 = e * p.N + r0, y1 = e * p.N + r1;
      (void)y0;
      (void)y1;
      for (int kb = 0; kb < KB; ++kb, ++kbg) {
        const int s = kbg % KS;
        if (kbg >= KS && !mbar_wait(&tma_empty[s], ((kbg / KS) - 1) & 1)) {
          record_error(p.err, kErrWaitEmpty);
          ok = false;
          break;
        }
        unsigned char* st = smem + S::kOffTma + s * S::kTmaStageBytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&tma_full[s], S::kTmaStageBytes);
          if constexpr (DG) {
            tma_load_2d(st, &tm_packed, r0 / 2, static_cast<int32_t>(static_cast<int64_t>(e) * p.K + kb * 64),
                        &tma_full[s]);
          } else {
            tma_load_2d(st, &tm_packed, kb * 32, y0, &tma_full[s]);
            if (HALVES == 2) tma_load_2d(st + kPackedHalfBytes, &tm_packed, kb * 32, y1, &tma_full[s]);
          }
          tma_load_2d(st + S::kPackedBytes, &tm_b, kb * 64, static_cast<int32_t>(rb), &tma_full[s]);
        }
        __syncwarp();
      }
      if (ok && p.lora_B) {
        // LoRA step: the tile's rows of scale * x . lora_A^T (bf16, 64 wide, zero past r)
        const int s = kbg % KS;
        if (kbg >= KS && !mbar_wait(&tma_empty[s], ((kbg / KS) - 1) & 1)) {
          record_error(p.err, kErrWaitEmpty);
          ok = false;
          break;
        }
        unsigned char* st = smem + S::kOffTma + s * S::kTmaStageBytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&tma_full[s], S::kBBytes);
          tma_load_2d(st + S::kPackedBytes, &tm_xa, 0, static_cast<int32_t>(rb), &tma_full[s]);
        }
        __syncwarp();
        ++kbg;
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------- MMA issuer
    uint32_t kbg = 0, j = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok; t += gridDim.x, ++j) {
      int e, n_tile;
      int64_t rb, re;
      if (!locate<BN>(p, t, &e, &rb, &re, &n_tile)) break;
      // N of this tile: the routed rows present, rounded up to the MMA's step of 16.
      const int nrows = static_cast<int>(re - rb);
      const int n_mma = min(BN, (nrows + 15) & ~15);
      const uint32_t idesc = idesc_bf16_f32(kBM, n_mma);
      const uint32_t slot = j % NACC;
      if (j >= NACC && !mbar_wait(&acc_empty[slot], ((j / NACC) - 1) & 1)) {
        record_error(p.err, kErrWaitEmpty);
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + slot * S::kCols;
      for (int kb = 0; kb < KB; ++kb, ++kbg) {
        const int s = kbg % KS, a = kbg % AS;
        if (!mbar_wait(&a_full[a], (kbg / AS) & 1) || !mbar_wait(&tma_full[s], (kbg / KS) & 1)) {
          record_error(p.err, kErrWaitFull);
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_addr = smem_u32(smem + S::kOffA + a * S::kAStageBytes);
          const uint32_t b_addr = smem_u32(smem + S::kOffTma + s * S::kTmaStageBytes + S::kPackedBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (kb | kk) ? 1u : 0u;
            const uint64_t bd = smem_desc_sw128(b_addr + kk * 32);
#pragma unroll
            for (int h = 0; h < HALVES; ++h) {
              if constexpr (S::ATMEM)
                umma_bf16_ts(d + h * BN, tmem_base + S::kAColBase + a * S::kACols + h * 32 + kk * 8, bd, idesc, acc);
              else
                umma_bf16(d + h * BN, smem_desc_sw128(a_addr + h * kAHalfBytes + kk * 32), bd, idesc, acc);
            }
          }
          umma_commit(&tma_empty[s]);
          umma_commit(&a_empty[a]);
        }
        __syncwarp();
      }
      if (ok && p.lora_B) {
        // LoRA step: D += lora_B[rows, 0:16] . (scale x . lora_A^T)[tokens, 0:16]^T, one K=16 MMA per half
        const int s = kbg % KS, a = kbg % AS;
        if (!mbar_wait(&a_full[a], (kbg / AS) & 1) || !mbar_wait(&tma_full[s], (kbg / KS) & 1)) {
          record_error(p.err, kErrWaitFull);
          ok = false;
        } else {
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a_addr = smem_u32(smem + S::kOffA + a * S::kAStageBytes);
            const uint64_t bd = smem_desc_sw128(smem_u32(smem + S::kOffTma + s * S::kTmaStageBytes + S::kPackedBytes));
#pragma unroll
            for (int h = 0; h < HALVES; ++h)
              umma_bf16(d + h * BN, smem_desc_sw128(a_addr + h * kAHalfBytes), bd, idesc, 1u);
            umma_commit(&tma_empty[s]);
            umma_commit(&a_empty[a]);
          }
          __syncwarp();
          ++kbg;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&acc_full[slot]);
      __syncwarp();
    }
  } else if (warp >= kWarpDec && warp < kWarpDec + kNumDecWarps) {
    // ------------------------------------------------------------- decoders
    if constexpr (S::ATMEM) {
      tmem_decoders<S>(p, smem, tma_full, a_empty, a_full, tmem_base, warp, lane);
    } else {
    const int dt = tid - kWarpDec * 32;            // 0..511
    if constexpr (DG) {
      dgrad_decoders<S>(p, smem, tma_full, a_empty, a_full, dt, lane);
    } else {
    const int r = dt / S::kTpr, kq = dt % S::kTpr;  // weight row of the tile, part of the k block
    const int half = r >> 7, ri = r & 127;
    const CodebookBytes cbt = codebook_bytes(p.quant);
    // MXFP4: low nibble first, and one e8m0 scale per 32 k -- this thread's
    // 64 / kTpr k of a block lie inside scale (2 kb + 2 kq / kTpr) of the row.
    const bool mx = p.quant == kQuantMxfp4;
    const uint32_t sel0 = mx ? kSelLoFirst0 : kSelHiFirst0, sel1 = mx ? kSelLoFirst1 : kSelHiFirst1;
    const int mx_sub = (2 * kq) / S::kTpr;
    uint32_t kbg = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok; t += gridDim.x) {
      int e, n_tile;
      int64_t rb, re;
      if (!locate<BN>(p, t, &e, &rb, &re, &n_tile)) break;
      int r0, r1;
      tile_rows<HALVES>(p, n_tile, &r0, &r1);
      const int n = (half ? r1 : r0) + ri;
      const bool valid = n < p.N;
      const int64_t wrow = static_cast<int64_t>(e) * p.N + (valid ? n : 0);
      const float* am = mx ? nullptr : p.absmax + wrow * KB;
      const uint8_t* ms = mx ? p.mx_scales + wrow * (2 * KB) + mx_sub : nullptr;
      auto scale_of = [&](int kb) { return mx ? e8m0_scale(__ldg(ms + 2 * kb)) : __ldg(am + kb); };
      // scales of the next 4 k blocks in flight (an L2 round trip outlasts one k block)
      float sc_ring[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) sc_ring[i] = (valid && i < KB) ? scale_of(i) : 0.0f;
      for (int kb0 = 0; kb0 < KB && ok; kb0 += 4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int kb = kb0 + i;
          if (kb >= KB) break;
          const float sc = sc_ring[i];
          sc_ring[i] = (valid && kb + 4 < KB) ? scale_of(kb + 4) : 0.0f;
          const int s = kbg % KS, a = kbg % AS;
          if (!mbar_wait(&tma_full[s], (kbg / KS) & 1) ||
              (kbg >= AS && !mbar_wait(&a_empty[a], ((kbg / AS) - 1) & 1))) {
            record_error(p.err, kErrWaitFull);
            ok = false;
            break;
          }
          // packed words of k [64 kq / kTpr, +64 / kTpr): one word = 8 elements = one chunk
          const unsigned char* src =
              smem + S::kOffTma + s * S::kTmaStageBytes + half * kPackedHalfBytes + ri * 32 + kq * (32 / S::kTpr);
          uint32_t words[S::kChunks];
          if constexpr (S::kChunks == 4) {
            const uint4 q = *reinterpret_cast<const uint4*>(src);
            words[0] = q.x;
            words[1] = q.y;
            words[2] = q.z;
            words[3] = q.w;
          } else {
            const uint2 q = *reinterpret_cast<const uint2*>(src);
            words[0] = q.x;
            words[1] = q.y;
          }
          const __nv_bfloat162 s2 = __float2bfloat162_rn(sc);
          unsigned char* arow =
              smem + S::kOffA + a * S::kAStageBytes + half * kAHalfBytes + (ri >> 3) * 1024 + (ri & 7) * 128;
#pragma unroll
          for (int c = 0; c < S::kChunks; ++c) {
            const uint32_t w = words[c];
            uint32_t v[4];
            decode4(w, cbt, &v[0], &v[1], sel0, sel1);
            decode4(w >> 16, cbt, &v[2], &v[3], sel0, sel1);
#pragma unroll
            for (int by = 0; by < 4; ++by) {
              __nv_bfloat162 h2 = *reinterpret_cast<__nv_bfloat162*>(&v[by]);
              h2 = __hmul2(h2, s2);
              v[by] = *reinterpret_cast<uint32_t*>(&h2);
            }
            const int chunk = kq * S::kChunks + c;
            *reinterpret_cast<uint4*>(arow + ((chunk ^ (ri & 7)) << 4)) = make_uint4(v[0], v[1], v[2], v[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[a]);
          ++kbg;
        }
      }
      if (ok && p.lora_B) {
        // LoRA step: row n's lora_B[e, n, 0:r] as the first 16 k of an A row (chunks 0 and 1).
        const int s = kbg % KS, a = kbg % AS;
        if (!mbar_wait(&tma_full[s], (kbg / KS) & 1) ||
            (kbg >= AS && !mbar_wait(&a_empty[a], ((kbg / AS) - 1) & 1))) {
          record_error(p.err, kErrWaitFull);
          ok = false;
          break;
        }
        if (kq < 2) {
          uint32_t v[4] = {0u, 0u, 0u, 0u};
          if (valid) {
            const uint16_t* lb = p.lora_B + (static_cast<int64_t>(e) * p.N + n) * p.r;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int j = kq * 8 + i;
              const uint32_t b = j < p.r ? lb[j] : 0u;
              v[i >> 1] |= b << (16 * (i & 1));
            }
          }
          unsigned char* arow =
              smem + S::kOffA + a * S::kAStageBytes + half * kAHalfBytes + (ri >> 3) * 1024 + (ri & 7) * 128;
          *reinterpret_cast<uint4*>(arow + ((kq ^ (ri & 7)) << 4)) = make_uint4(v[0], v[1], v[2], v[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[a]);
        ++kbg;
      }
    }
    }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------- epilogue
    const int q = warp;  // TMEM lane quadrant = output columns 32q .. 32q + 31 of a part
    const int ri = q * 32 + lane;
    const int esize = p.out_bf16 ? 2 : 4;
    const uint32_t row_bytes = kBM * esize;
    unsigned char* stage0 = smem + S::kOffOut;
    uint32_t j = 0, chunk_no = 0, epi_phase = 0;
    bool ok = true;
    // All four warps meet here; false (error recorded) if one never arrives.
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_bar);
      const bool w = mbar_wait(epi_bar, epi_phase & 1);
      ++epi_phase;
      if (!w) record_error(p.err, kErrWaitFull);
      return w;
    };
    for (int64_t t = blockIdx.x; ok; t += gridDim.x, ++j) {
      int e, n_tile;
      int64_t rb, re;
      if (!locate<BN>(p, t, &e, &rb, &re, &n_tile)) break;
      const uint32_t slot = j % NACC;
      if (!mbar_wait(&acc_full[slot], (j / NACC) & 1)) {
        record_error(p.err, kErrWaitFull);
        break;
      }
      tc_fence_after();
      int r0, r1;
      tile_rows<HALVES>(p, n_tile, &r0, &r1);
      const int nrows = static_cast<int>(re - rb);
      const uint32_t c0 = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + slot * S::kCols;
      const int parts = p.swiglu ? 1 : HALVES;
      for (int part = 0; part < parts && ok; ++part) {
        const int col0 = (part ? r1 : r0);  // first output column of this part
        if (col0 >= p.out_cols) continue;   // a half past the last weight row
        for (int cr = 0; cr < nrows; cr += kChunk, ++chunk_no) {
          unsigned char* stage = stage0 + (chunk_no & 1) * kOutChunkBytes;
          // The store that last read this buffer (two chunks ago) must be done reading.
          if (tid == 0) bulk_wait_group_read<1>();
          if (!(ok = epi_sync())) break;
#pragma unroll
          for (int hs = 0; hs < kChunk; hs += 16) {
            float v[16];
            if (p.swiglu) {
              float u[16];
              tmem_ld_32x32b_x16(c0 + cr + hs, v);
              tmem_ld_32x32b_x16(c0 + BN + cr + hs, u);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = __fdividef(v[i], 1.0f + __expf(-v[i])) * u[i];
            } else {
              tmem_ld_32x32b_x16(c0 + part * BN + cr + hs, v);
              tmem_ld_wait();
            }
            if (p.out_bf16) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                *reinterpret_cast<uint16_t*>(stage + (hs + i) * row_bytes + ri * 2) = float_to_bf16_bits(v[i]);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) *reinterpret_cast<float*>(stage + (hs + i) * row_bytes + ri * 4) = v[i];
            }
          }
          fence_proxy_async_smem();
          if (!(ok = epi_sync())) break;
          const int rows_here = min(kChunk, nrows - cr);
          if (rows_here == kChunk) {
            if (tid == 0) tma_store_2d(&tm_out, stage, col0, static_cast<int32_t>(rb + cr));
          } else {
            // Ragged end of the group: plain 16-byte (fp32) or 8-byte (bf16) stores, row by row.
            const int ncol = min(kBM, p.out_cols - col0);
            for (int rr = q; rr < rows_here; rr += 4) {
              const int c = lane * 4;  // four columns per lane
              if (c < ncol) {
                const unsigned char* src = stage + rr * row_bytes + c * esize;
                unsigned char* dst = static_cast<unsigned char*>(p.out) +
                                     ((rb + cr + rr) * p.out_cols + col0 + c) * static_cast<int64_t>(esize);
                if (p.out_bf16)
                  *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(src);
                else
                  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
              }
            }
          }
          // One bulk group per chunk (empty for a ragged chunk) keeps the
          // read-wait above tied to the buffer two chunks back.
          if (tid == 0) bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[slot]);
    }
    if (tid == 0) bulk_wait_group_all();
  }
  // All roles are done (every MMA was waited on through acc_full): free TMEM.
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                 uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  const uint64_t dims[2] = {inner, rows};
  const uint64_t strides[1] = {row_stride_bytes};
  const uint32_t box[2] = {box_inner, box_rows};
  return encode_tensor_map(m, dt, 2, base, dims, strides, box, sw);
}

template <class S>
cudaError_t launch_shape(const GemmArgs& a, int* err_word, cudaStream_t stream) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  err = ensure_smem_limit(reinterpret_cast<const void*>(grouped_nf4_tc_kernel<S, false>), S::kSmemBytes);
  if (err != cudaSuccess) return err;
  CUtensorMap tm_packed, tm_b;
  const uint64_t total_w_rows = static_cast<uint64_t>(a.E) * a.N;
  if (!make_map_2d(&tm_packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.packed, a.K / 2, total_w_rows, a.K / 2, 32, kBM,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (!make_map_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.A, a.K, a.a_rows, a.lda * 2, 64, S::BN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int out_cols = a.epi == E4B_EPI_SWIGLU ? a.N / 2 : a.N;
  const int esize = a.out_bf16 ? 2 : 4;
  CUtensorMap tm_out;
  if (!make_map_2d(&tm_out, a.out_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.out,
                   out_cols, a.total_rows, static_cast<uint64_t>(out_cols) * esize, kBM, kChunk,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const bool lora = a.lora_B != nullptr && a.r > 0;
  // The TMEM decoders have no LoRA step: their barrier phases would drift from the MMA issuer's.
  if (S::ATMEM && lora) return cudaErrorInvalidValue;
  CUtensorMap tm_xa = tm_b;  // unused without LoRA
  if (lora && !make_map_2d(&tm_xa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.xa, kLoraCols, a.total_rows, kLoraCols * 2, 64,
                           S::BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.offsets = a.offsets;
  p.E = a.E;
  p.total_rows = a.total_rows;
  p.absmax = a.absmax;
  p.quant = a.quant;
  p.mx_scales = a.mx_scales;
  p.N = a.N;
  p.K = a.K;
  p.swiglu = a.epi == E4B_EPI_SWIGLU;
  p.out = a.out;
  p.out_bf16 = a.out_bf16;
  p.out_cols = out_cols;
  p.lora_B = lora ? a.lora_B : nullptr;
  p.r = lora ? a.r : 0;
  const int wrows = p.swiglu ? kBM : S::HALVES * kBM;  // output columns (weight rows) per tile
  p.n_tiles = ((p.swiglu ? a.N / 2 : a.N) + wrows - 1) / wrows;
  p.err = err_word;
  // Upper bound of the tile count: (ceil(rows / BN) + groups) * n_tiles.
  const int64_t tiles =
      ((a.total_rows + S::BN - 1) / S::BN + (a.E < a.total_rows ? a.E : a.total_rows)) * p.n_tiles;
  const int grid = static_cast<int>(tiles < di.sm_count ? tiles : di.sm_count);
  const bool mx = a.quant == kQuantMxfp4;
  if (mx && (S::ATMEM || lora || a.mx_scales == nullptr)) return cudaErrorInvalidValue;
  LaunchScope ls(mx ? (p.swiglu ? "mxfp4.tc.swiglu" : "mxfp4.tc") : (p.swiglu ? "gemm.tc.swiglu" : "gemm.tc"), stream);
  grouped_nf4_tc_kernel<S, false><<<grid, kThreadsTc, S::kSmemBytes, stream>>>(tm_packed, tm_b, tm_out, tm_xa, p);
  return cudaGetLastError();
}

// The dgrad product on the tensor cores: A tile = W^T (256 columns k per
// tile), B = the dY rows (contiguous, in group order), K steps over the rows n.
template <class S>
cudaError_t launch_dgrad_shape(const DgradArgs& a, const uint16_t* dy, int64_t dy_rows, int64_t lddy, int* err_word,
                               cudaStream_t stream) {
  static_assert(S::HALVES == 2, "dgrad tiles cover 256 columns");
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  err = ensure_smem_limit(reinterpret_cast<const void*>(grouped_nf4_tc_kernel<S, true>), S::kSmemBytes);
  if (err != cudaSuccess) return err;
  CUtensorMap tm_packed, tm_b, tm_out;
  const uint64_t total_w_rows = static_cast<uint64_t>(a.E) * a.N;  // rows n of every expert
  if (!make_map_2d(&tm_packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.packed, a.K / 2, total_w_rows, a.K / 2,
                   S::HALVES * 64, 64, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (!make_map_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dy, a.N, dy_rows, lddy * 2, 64, S::BN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int esize = a.out_bf16 ? 2 : 4;
  if (!make_map_2d(&tm_out, a.out_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.out,
                   a.K, a.total_rows, static_cast<uint64_t>(a.K) * esize, kBM, kChunk, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.offsets = a.offsets;
  p.E = a.E;
  p.total_rows = a.total_rows;
  p.absmax = a.absmax;
  p.quant = a.quant;
  p.N = a.K;  // tile rows: columns k of W
  p.K = a.N;  // K steps: rows n of W
  p.swiglu = 0;
  p.out = a.out;
  p.out_bf16 = a.out_bf16;
  p.out_cols = a.K;
  p.lora_B = nullptr;
  p.r = 0;
  p.n_tiles = (a.K + S::HALVES * kBM - 1) / (S::HALVES * kBM);
  p.err = err_word;
  const int64_t tiles =
      ((a.total_rows + S::BN - 1) / S::BN + (a.E < a.total_rows ? a.E : a.total_rows)) * p.n_tiles;
  const int grid = static_cast<int>(tiles < di.sm_count ? tiles : di.sm_count);
  LaunchScope ls("dgrad.tc", stream);
  grouped_nf4_tc_kernel<S, true><<<grid, kThreadsTc, S::kSmemBytes, stream>>>(tm_packed, tm_b, tm_out, tm_b, p);
  return cudaGetLastError();
}

// LoRA prep for the tensor-core kernel: one CTA per (group, 64-row tile),
// lora_A[e] staged in shared memory.  It copies the tile's routed rows into
// `gathered` (when a row index is given) and writes xa[p, 0:64] =
// bf16(scale * A_row . lora_A[e, j]) for j < r, zeros after -- the B operand
// of the GEMM kernel's extra K=16 MMA step.
struct PrepParams {
  const uint16_t* A;
  int64_t a_rows, lda;
  const int32_t* row_index;  // nullable
  const int32_t* offsets;
  int E;
  int64_t total_rows;
  int K;
  uint16_t* gathered;  // [total_rows, K] or null
  const uint16_t* lora_A;
  int r;
  float scale;
  uint16_t* xa;  // [total_rows, 64]
};

constexpr int kPrepRows = 64;
constexpr int kPrepUnroll = 4;  // 32-k chunks of the two rows' loads in flight per lane

__device__ __forceinline__ void mma_bf16_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Warp w takes routed rows 16w .. 16w + 15 of the tile as the rows of an
// m16n8k16 MMA and the adapter rows (16, zero past r) as its columns; lane
// (g, t) loads physical k [8t, 8t + 8) of each 32-k chunk of rows g and g + 8
// as one 16-byte vector -- the A fragments of two MMAs, with K permuted the
// same way for lora_A (rows g and g + 8 of its staged copy) -- and stores the
// same vectors into `gathered`.  The loads are HBM-bound; the products cost a
// few MMAs per 1 KB read.
__global__ void __launch_bounds__(128) lora_prep_kernel(PrepParams q) {
  extern __shared__ __align__(16) uint16_t la_s[];  // [16, K + 8]: lora_A[e], rows past r zero
  __shared__ int64_t tile_s[3];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  if (warp == 0) {
    int ge;
    int64_t b0, b1;
    const bool found = find_group_tile(q.offsets, q.E, q.total_rows, kPrepRows, blockIdx.x, &ge, &b0, &b1);
    if (lane == 0) {
      tile_s[0] = found ? ge : -1;
      tile_s[1] = b0;
      tile_s[2] = b1;
    }
  }
  __syncthreads();
  const int e = static_cast<int>(tile_s[0]);
  if (e < 0) return;
  const int64_t rb = tile_s[1], re = tile_s[2];
  const int K = q.K, kv = K / 8, ls = K + 8;  // shared row stride (bf16): 16 bytes of padding per row
  const uint4* src_a = reinterpret_cast<const uint4*>(q.lora_A + static_cast<int64_t>(e) * q.r * K);
  for (int i = threadIdx.x; i < 16 * kv; i += blockDim.x) {
    const int row = i / kv, c = i % kv;
    reinterpret_cast<uint4*>(la_s + row * ls)[c] = row < q.r ? src_a[row * kv + c] : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  const int64_t p0 = rb + 16 * warp + g, p1 = p0 + 8;
  const bool v0 = p0 < re, v1 = p1 < re;
  int64_t s0 = v0 ? (q.row_index ? q.row_index[p0] : p0) : 0;
  int64_t s1 = v1 ? (q.row_index ? q.row_index[p1] : p1) : 0;
  s0 = clampv<int64_t>(s0, 0, q.a_rows - 1);
  s1 = clampv<int64_t>(s1, 0, q.a_rows - 1);
  const uint4* x0 = reinterpret_cast<const uint4*>(q.A + s0 * q.lda);
  const uint4* x1 = reinterpret_cast<const uint4*>(q.A + s1 * q.lda);
  uint4* g0 = (q.gathered && v0) ? reinterpret_cast<uint4*>(q.gathered + p0 * K) : nullptr;
  uint4* g1 = (q.gathered && v1) ? reinterpret_cast<uint4*>(q.gathered + p1 * K) : nullptr;
  const bool two = q.r > 8;  // adapter rows 8..15 need the second n tile
  float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
  const int nchunks = K / 32;
  for (int ch0 = 0; ch0 < nchunks; ch0 += kPrepUnroll) {
    uint4 xa0[kPrepUnroll], xa1[kPrepUnroll];
#pragma unroll
    for (int u = 0; u < kPrepUnroll; ++u) {
      const int c = (ch0 + u) * 4 + t;  // 16-byte vector index within the row
      const bool in = ch0 + u < nchunks;
      xa0[u] = (in && v0) ? __ldg(x0 + c) : make_uint4(0, 0, 0, 0);
      xa1[u] = (in && v1) ? __ldg(x1 + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kPrepUnroll; ++u) {
      if (ch0 + u >= nchunks) break;
      const int c = (ch0 + u) * 4 + t;
      if (g0) g0[c] = xa0[u];
      if (g1) g1[c] = xa1[u];
      const uint4 b = reinterpret_cast<const uint4*>(la_s + g * ls)[c];
      mma_bf16_16816(c0, xa0[u].x, xa1[u].x, xa0[u].y, xa1[u].y, b.x, b.y);
      mma_bf16_16816(c0, xa0[u].z, xa1[u].z, xa0[u].w, xa1[u].w, b.z, b.w);
      if (two) {
        const uint4 b2 = reinterpret_cast<const uint4*>(la_s + (g + 8) * ls)[c];
        mma_bf16_16816(c1, xa0[u].x, xa1[u].x, xa0[u].y, xa1[u].y, b2.x, b2.y);
        mma_bf16_16816(c1, xa0[u].z, xa1[u].z, xa0[u].w, xa1[u].w, b2.z, b2.w);
      }
    }
  }
  // c0[0..1]: row g, adapter columns 2t, 2t + 1; c0[2..3]: row g + 8; c1: columns 8 + 2t, 8 + 2t + 1.
  // Columns 16..63 of an xa row are zero: lane t writes words 8 + 6t .. 8 + 6t + 5.
  if (v0) {
    uint32_t* row = reinterpret_cast<uint32_t*>(q.xa + p0 * kLoraCols);
    row[t] = pack_bf16x2(q.scale * c0[0], q.scale * c0[1]);
    row[4 + t] = pack_bf16x2(q.scale * c1[0], q.scale * c1[1]);
#pragma unroll
    for (int i = 0; i < 6; ++i) row[8 + 6 * t + i] = 0u;
  }
  if (v1) {
    uint32_t* row = reinterpret_cast<uint32_t*>(q.xa + p1 * kLoraCols);
    row[t] = pack_bf16x2(q.scale * c0[2], q.scale * c0[3]);
    row[4 + t] = pack_bf16x2(q.scale * c1[2], q.scale * c1[3]);
#pragma unroll
    for (int i = 0; i < 6; ++i) row[8 + 6 * t + i] = 0u;
  }
}

using ShapeWide = TcShape<256, 2, 1>;    // 2 x 128 weight rows x 256 routed rows, one accumulator set
using ShapeDouble = TcShape<128, 2, 2>;  // 2 x 128 x 128, two accumulator sets
using ShapeNarrow = TcShape<256, 1, 2>;  // 128 x 256, two accumulator sets (no SwiGLU)
using ShapeTmem = TcShape<192, 2, 1, true>;  // 2 x 128 x 192, A in TMEM (no LoRA step)

int shape_override() {
  const char* v = getenv("E4B_TC_SHAPE");
  if (!v) return 0;
  if (!strcmp(v, "wide")) return 1;
  if (!strcmp(v, "double")) return 2;
  if (!strcmp(v, "narrow")) return 3;
  if (!strcmp(v, "tmem")) return 4;
  return 0;
}

}  // namespace

// ---- host side: tensor maps ---------------------------------------------------------
namespace {
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
}  // namespace

bool tensor_maps_available() { return encode_fn() != nullptr; }

bool encode_tensor_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  return fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, st, b, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_supported(const GemmArgs& a) {
  // The operand rows must be contiguous (row_index already applied); K % 64
  // and N % 64 hold by contract.  With LoRA, lora_A[e] must fit the prep
  // kernel's shared memory and the products need their workspace rows.
  if (a.row_index != nullptr || a.lda % 8 != 0 || !tensor_maps_available()) return false;
  if (a.lora_B && a.r > 0)
    return a.r <= 16 && a.xa != nullptr && static_cast<size_t>(16) * (a.K + 8) * 2 <= kLoraPrepSmemMax &&
           (reinterpret_cast<uintptr_t>(a.lora_A) & 15u) == 0;
  return true;
}

cudaError_t launch_grouped_gemm_tc(const GemmArgs& a, int* err_word, cudaStream_t stream) {
  const bool swiglu = a.epi == E4B_EPI_SWIGLU;
  int s = shape_override();
  if (s == 3 && swiglu) s = 0;
  if (s == 0) {
    // Measured on B200 (OLMoE-, Qwen3- and gpt-oss-shaped prefill): SwiGLU
    // runs best on the 2 x 128 x 256 tile; the plain GEMM on 128 x 256 with two
    // accumulator sets unless the groups are large.
    const int64_t rows_per_group = a.total_rows / (a.E > 0 ? a.E : 1);
    s = swiglu ? 1 : (rows_per_group >= 512 ? 1 : 3);
  }
  if (s == 4 && !(a.lora_B && a.r > 0) && a.quant != kQuantMxfp4) return launch_shape<ShapeTmem>(a, err_word, stream);
  if (s == 4) s = swiglu ? 1 : 3;
  if (s == 1) return launch_shape<ShapeWide>(a, err_word, stream);
  if (s == 2) return launch_shape<ShapeDouble>(a, err_word, stream);
  return launch_shape<ShapeNarrow>(a, err_word, stream);
}

bool dgrad_tc_supported(const DgradArgs& a, int64_t lddy) {
  return tensor_maps_available() && lddy % 8 == 0 && (a.lora_A == nullptr || !a.out_bf16);
}

cudaError_t launch_grouped_dgrad_tc(const DgradArgs& a, const uint16_t* dy, int64_t dy_rows, int64_t lddy,
                                    int* err_word, cudaStream_t stream) {
  // Groups of 512 rows and more fill the 256-row tile; smaller ones waste less
  // with 128 routed rows and two accumulator sets.
  const int64_t rows_per_group = a.total_rows / (a.E > 0 ? a.E : 1);
  int s = shape_override();
  if (s != 1 && s != 2) s = rows_per_group >= 512 ? 1 : 2;
  if (s == 1) return launch_dgrad_shape<ShapeWide>(a, dy, dy_rows, lddy, err_word, stream);
  return launch_dgrad_shape<ShapeDouble>(a, dy, dy_rows, lddy, err_word, stream);
}

cudaError_t launch_tc_lora_prep(const GemmArgs& a, cudaStream_t stream) {
  if (a.total_rows == 0) return cudaSuccess;
  PrepParams q{};
  q.A = a.A;
  q.a_rows = a.a_rows;
  q.lda = a.lda;
  q.row_index = a.row_index;
  q.offsets = a.offsets;
  q.E = a.E;
  q.total_rows = a.total_rows;
  q.K = a.K;
  q.gathered = a.row_index ? a.a_gathered : nullptr;
  q.lora_A = a.lora_A;
  q.r = a.r;
  q.scale = a.lora_scale;
  q.xa = reinterpret_cast<uint16_t*>(a.xa);
  const size_t smem = static_cast<size_t>(16) * (a.K + 8) * 2;
  cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(lora_prep_kernel), smem);
  if (err != cudaSuccess) return err;
  const int64_t tiles = (a.total_rows + kPrepRows - 1) / kPrepRows + (a.E < a.total_rows ? a.E : a.total_rows);
  LaunchScope ls("gemm.tc.lora_prep", stream);
  lora_prep_kernel<<<static_cast<unsigned>(tiles), 128, smem, stream>>>(q);
  return cudaGetLastError();
}

}  // namespace e4b
