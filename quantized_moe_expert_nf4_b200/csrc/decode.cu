// Fused small-M (decode) forward of the NF4 expert layer: two kernels, no host sync.
//
// The pages' inference fast path for single-token decode is a fused 4-bit GEMV
// over the routed experts (experts4bit-qlora 0.22.0, "Inference: serve the
// fine-tune you just made"), and decode is launch-bound at ~89 launches per
// layer step ("CUDA-graph decode capture").  Here the whole layer is two
// kernels chained with programmatic dependent launch:
//
//   kernel A  routing (every CTA, redundantly: M <= 8 tokens), then the gate
//             and up rows of every touched expert in items of 8 gate + 8 up
//             rows over all of K = H -> SiLU(gate) * up (+ LoRA delta) -> h
//             (bf16, [M*k, I], slot order).  It also prefetches the touched
//             experts' down rows into L2, so that HBM keeps streaming while the
//             second kernel starts.
//   kernel B  the routing kernel A published, then for every block
//             of 16 output rows of H the down rows of every touched expert, with
//             the routing weights folded into the per-block scale, so the
//             combine happens inside the CTA in a fixed order (deterministic).
//
// Only experts that some token selected are read.  Both kernels are split-K
// GEMVs on warp tensor cores: each CTA owns a contiguous run of items, its 16
// warps split K in spans of two absmax blocks (128 k), and each lane loads its
// 16-byte slice of a span of the packed rows straight from HBM into the
// registers of an mma.sync m16n8k16 fragment (weight rows = MMA rows, the <= 8
// tokens = the 8 MMA columns), several items ahead.  Nibbles become bf16
// through a per-lane replicated byte -> bf16x2 codebook table in shared memory
// (lane l reads only bank l), scaled by the block's bf16 absmax before the
// MMA.  One block barrier per batch gathers the 16 warps' partials.
#include <algorithm>

#include "async.cuh"
#include "common.cuh"
#include "e4b_internal.h"
#include "topk.cuh"

namespace e4b {
namespace {

constexpr int kMaxM = 8;
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxSlots = 8;               // (item, span) load slots per warp per batch in kernel A
constexpr int kPairSlots = 2;              // (expert, span) load slots per warp per batch in kernel B
constexpr int kMaxKBW = 2;                 // spans (2 k-blocks) per warp per item: H <= 128 * 16 * 2 = 4096
constexpr unsigned long long kPrefetchLimit = 64ull << 20;
constexpr uint32_t kPrefetchChunk = 32 * 1024;

struct DecodeParams {
  const uint16_t* x;
  const float* logits;
  int M, k, E, H, I;
  int renorm;
  const uint8_t* gu_packed;
  const float* gu_absmax;
  const uint8_t* dn_packed;
  const float* dn_absmax;
  const uint16_t* lora_A;
  const uint16_t* lora_B;
  int r;
  float lora_scale;
  uint16_t* h;    // [S, I] bf16 (slot order)
  uint16_t* out;  // [M, H] bf16
  // Routing result of the gate_up kernel for the down kernel: [nU, pad x3],
  // touched [S], slotmap [S * kMaxM], weights [S] (as float bits).
  int* meta;
};

struct Layout {
  uint32_t lut, xs, red, ids, w, uidx, touched, slotmap, xa, total;
};

__host__ __device__ inline uint32_t al(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Spans of 128 k (2 absmax blocks, 64 packed bytes of a row) per warp per item.
__host__ __device__ inline int kbw_of(int H) { return ((H / 64 + 1) / 2 + kWarps - 1) / kWarps; }

// (item, span) load slots per warp per batch of kernel A: eight for one token
// with one span per warp (a CTA's whole share in one batch; measured faster at
// M = 1), four otherwise (more tokens need the registers for x; measured
// faster at M = 4 and 8).
__host__ __device__ inline int slots_for(int M, int H) { return (M == 1 && kbw_of(H) == 1) ? 8 : 4; }

// Shared-memory carve of kernel A (gate_up) or B (down).
__host__ __device__ inline Layout make_layout(bool is_a, int M, int k, int E, int H, int r) {
  Layout L;
  uint32_t o = 0;
  L.lut = o;
  o = al(o + 256 * 32 * 4, 16);
  L.xs = o;
  if (is_a) o = al(o + M * (2 * H + 16), 16);
  L.red = o;
  const int items = is_a ? slots_for(M, H) : 1;  // partial sums of the items of a batch (A), 1 row block (B)
  o = al(o + items * kWarps * 32 * 16, 16);
  const int S = M * k;
  L.ids = o;
  o = al(o + S * 4, 16);
  L.w = o;
  o = al(o + S * 4, 16);
  L.uidx = o;
  o = al(o + E * 4, 16);
  L.touched = o;
  o = al(o + S * 4, 16);
  L.slotmap = o;
  o = al(o + S * kMaxM * 4, 16);
  L.xa = o;
  if (is_a && r > 0) o = al(o + S * r * 4, 16);
  L.total = o;
  return L;
}

__device__ __forceinline__ void mma_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_stream_u4(const uint8_t* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}

// One span (128 k = 2 absmax blocks) of a 16-row tile, accumulated into c.
// Thread (g, t) owns physical k [32t, 32t+32) of the span -- 16 packed bytes of
// row g (r0) and of row g+8 (r1), all inside k-block t/2 -- and the matching 32
// bf16 of its token column g (x).  Each byte's codebook pair is scaled by its
// row's bf16(absmax) before the MMA (the block scale differs between threads of
// one MMA, so it cannot be applied to the product).  MMA j takes bytes 2j and
// 2j+1 of each row; K is permuted identically on both operands.
__device__ __forceinline__ void span_mma(const uint32_t* __restrict__ lut_lane, uint4 r0, uint4 r1, float a0,
                                         float a1, const uint4 x[4], float c[4]) {
  const __nv_bfloat162 s0 = __float2bfloat162_rn(a0), s1 = __float2bfloat162_rn(a1);
  const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w}, w1[4] = {r1.x, r1.y, r1.z, r1.w};
  const uint32_t xw[16] = {x[0].x, x[0].y, x[0].z, x[0].w, x[1].x, x[1].y, x[1].z, x[1].w,
                           x[2].x, x[2].y, x[2].z, x[2].w, x[3].x, x[3].y, x[3].z, x[3].w};
  auto pair = [&](uint32_t word, int byte, __nv_bfloat162 sc) {
    uint32_t v = lut_lane[((word >> (8 * byte)) & 0xffu) << 5];
    __nv_bfloat162 h2 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&v), sc);
    return *reinterpret_cast<uint32_t*>(&h2);
  };
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int b = 2 * (j & 1);
    const uint32_t wa = w0[j >> 1], wb = w1[j >> 1];
    mma_16816(c, pair(wa, b, s0), pair(wb, b, s1), pair(wa, b + 1, s0), pair(wb, b + 1, s1), xw[2 * j],
              xw[2 * j + 1]);
  }
}

// Top-k of token `t` by the calling warp, with the key array sized for E.
__device__ __forceinline__ void route_one(const DecodeParams& p, int t, int* ids_s, float* w_s) {
  const int maxj = (p.E + 31) / 32;
  if (maxj <= 1) route_token<1>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
  else if (maxj <= 2) route_token<2>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
  else if (maxj <= 4) route_token<4>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
  else if (maxj <= 8) route_token<8>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
  else route_token<16>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
}

// Byte -> bf16x2 codebook pairs, replicated per lane (entry b of lane l at
// b * 32 + l), written by the warps [w0, kWarps) of the block.
__device__ __forceinline__ void fill_lut_warps(uint32_t* lut, int w0) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp < w0) return;
  const float cbl = kNf4CodebookDev[lane & 15];
  for (int b = warp - w0; b < 256; b += kWarps - w0) {
    const float hi = __shfl_sync(0xffffffffu, cbl, b >> 4);
    const float lo = __shfl_sync(0xffffffffu, cbl, b & 15);
    lut[b * 32 + lane] = pack_bf16x2(hi, lo);
  }
}

// Prologue shared by both kernels: warps < M route one token each while the
// other warps build the codebook table (and, in kernel A, stage x).  Then the
// touched experts (ascending id) and slotmap[u][t] = slot of token t in expert
// touched[u] (or -1) are built.
__device__ void decode_prologue(const DecodeParams& p, uint32_t* lut, uint16_t* xs, int xstride, int* ids_s,
                                float* w_s, int* uidx, int* touched, int* slotmap, int* nU_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.M * p.k;
  for (int e = tid; e < p.E; e += blockDim.x) uidx[e] = -1;
  if (warp < p.M) {
    route_one(p, warp, ids_s, w_s);
  } else {
    fill_lut_warps(lut, p.M);
    if (xs) {
      const int nthr = (kWarps - p.M) * 32, me = tid - p.M * 32;
      for (int i = me; i < p.M * (p.H / 8); i += nthr) {
        const int t = i / (p.H / 8), c = i % (p.H / 8);
        reinterpret_cast<uint4*>(xs + t * xstride)[c] =
            reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(t) * p.H)[c];
      }
    }
  }
  __syncthreads();
  for (int s = tid; s < S; s += blockDim.x) uidx[ids_s[s]] = 0;  // flag
  __syncthreads();
  if (warp == 0) {
    int count = 0;
    for (int base = 0; base < p.E; base += 32) {
      const int e = base + lane;
      const bool f = (e < p.E) && uidx[e] == 0;
      const uint32_t bal = __ballot_sync(0xffffffffu, f);
      if (f) {
        const int u = count + __popc(bal & lanemask_lt());
        touched[u] = e;
        uidx[e] = u;
      }
      count += __popc(bal);
    }
    if (lane == 0) *nU_out = count;
  }
  __syncthreads();
  const int nU = *nU_out;
  for (int i = tid; i < nU * kMaxM; i += blockDim.x) slotmap[i] = -1;
  __syncthreads();
  for (int s = tid; s < S; s += blockDim.x) slotmap[uidx[ids_s[s]] * kMaxM + s / p.k] = s;
  __syncthreads();
}

// L2 prefetch of the gate and up rows (and their absmax) of items [a, b),
// one thread per item.
__device__ __forceinline__ void prefetch_items(const DecodeParams& p, const int* touched, int a, int b) {
  const int i = a + static_cast<int>(threadIdx.x);
  if (i >= b) return;
  const int ipe = p.I / 8;
  const int u = i / ipe, rb = i % ipe;
  const int64_t grow = static_cast<int64_t>(touched[u]) * 2 * p.I + rb * 8;
  const int64_t row_bytes = p.H / 2, kb = p.H / 64;
  prefetch_l2(p.gu_packed + grow * row_bytes, static_cast<uint32_t>(8 * row_bytes));
  prefetch_l2(p.gu_packed + (grow + p.I) * row_bytes, static_cast<uint32_t>(8 * row_bytes));
  prefetch_l2(p.gu_absmax + grow * kb, static_cast<uint32_t>(8 * kb * 4));
  prefetch_l2(p.gu_absmax + (grow + p.I) * kb, static_cast<uint32_t>(8 * kb * 4));
}

// ---------------------------------------------------------------------------
// Kernel A: gate_up + SwiGLU (+ LoRA delta) -> h.  KBW = k-blocks per warp per item.
template <int KBW, int SLOTS>
__global__ void __launch_bounds__(kThreads, 1) decode_gate_up_kernel(DecodeParams p) {
  static_assert(SLOTS <= kMaxSlots, "load slots");
  constexpr int IB = SLOTS / KBW;  // items per batch
  extern __shared__ __align__(16) unsigned char smem[];
  const Layout L = make_layout(true, p.M, p.k, p.E, p.H, p.r);
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs);
  float4* red = reinterpret_cast<float4*>(smem + L.red);
  int* ids_s = reinterpret_cast<int*>(smem + L.ids);
  float* w_s = reinterpret_cast<float*>(smem + L.w);
  int* uidx = reinterpret_cast<int*>(smem + L.uidx);
  int* touched = reinterpret_cast<int*>(smem + L.touched);
  int* slotmap = reinterpret_cast<int*>(smem + L.slotmap);
  float* xa = reinterpret_cast<float*>(smem + L.xa);
  __shared__ int nU_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, I = p.I, KB = H / 64;
  const int xstride = H + 8;  // bf16 elements (2H + 16 bytes: conflict-free 16-byte reads)

  pdl_wait();               // the inputs of this call are final
  pdl_launch_dependents();  // the down kernel may launch and run its prologue
  decode_prologue(p, lut, xs, xstride, ids_s, w_s, uidx, touched, slotmap, &nU_s);
  const int nU = nU_s;
  if (blockIdx.x == 0) {
    // Every CTA routed identically; one publishes the result for the down kernel.
    const int S = p.M * p.k;
    int* m_touched = p.meta + 4;
    int* m_slotmap = m_touched + S;
    float* m_w = reinterpret_cast<float*>(m_slotmap + S * kMaxM);
    if (tid == 0) p.meta[0] = nU;
    for (int i = tid; i < nU; i += blockDim.x) m_touched[i] = touched[i];
    for (int i = tid; i < nU * kMaxM; i += blockDim.x) m_slotmap[i] = slotmap[i];
    for (int i = tid; i < S; i += blockDim.x) m_w[i] = w_s[i];
  }
  const int ipe = I / 8;  // items per expert
  const int nitems = nU * ipe;
  // A contiguous run of items per CTA: consecutive items are consecutive rows.
  const int q = nitems / gridDim.x, rem = nitems % gridDim.x;
  const int i0 = blockIdx.x * q + min(static_cast<int>(blockIdx.x), rem);
  const int i1 = i0 + q + (static_cast<int>(blockIdx.x) < rem ? 1 : 0);

  if (warp == kWarps - 1) {
    // Prefetch this CTA's share of the touched experts' down rows into L2.
    const uint64_t per_expert = static_cast<uint64_t>(H) * I / 2;
    const uint64_t per_expert_am = static_cast<uint64_t>(H) * (I / 64) * 4;
    const uint64_t chunks_pk = (per_expert + kPrefetchChunk - 1) / kPrefetchChunk;
    const uint64_t chunks_am = (per_expert_am + kPrefetchChunk - 1) / kPrefetchChunk;
    const uint64_t per_u = chunks_pk + chunks_am;
    uint64_t total = static_cast<uint64_t>(nU) * per_u;
    const uint64_t cap = kPrefetchLimit / kPrefetchChunk;
    if (total > cap) total = cap;
    for (uint64_t c = static_cast<uint64_t>(blockIdx.x) * 32 + lane; c < total; c += static_cast<uint64_t>(gridDim.x) * 32) {
      const uint64_t u = c / per_u, qq = c % per_u;
      const int64_t e = touched[u];
      if (qq < chunks_pk) {
        const uint64_t off = qq * kPrefetchChunk;
        const uint64_t n = min(static_cast<uint64_t>(kPrefetchChunk), per_expert - off);
        prefetch_l2(p.dn_packed + e * per_expert + off, static_cast<uint32_t>(n));
      } else {
        const uint64_t off = (qq - chunks_pk) * kPrefetchChunk;
        const uint64_t n = min(static_cast<uint64_t>(kPrefetchChunk), per_expert_am - off);
        prefetch_l2(reinterpret_cast<const unsigned char*>(p.dn_absmax) + e * per_expert_am + off,
                    static_cast<uint32_t>(n));
      }
    }
  }

  const int g = lane >> 2, t = lane & 3;
  const int S = p.M * p.k;
  if (p.r > 0) {
    // LoRA first factor per slot: xa[s, rho] = x[token(s)] . lora_A[e(s), rho]
    for (int qd = warp; qd < S * p.r; qd += kWarps) {
      const int s = qd / p.r, rho = qd % p.r;
      const int tok = s / p.k;
      const uint16_t* la = p.lora_A + (static_cast<int64_t>(ids_s[s]) * p.r + rho) * H;
      float acc = 0.f;
      for (int kk = lane * 8; kk < H; kk += 256) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xs + tok * xstride + kk);
        const uint4 av = *reinterpret_cast<const uint4*>(la + kk);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc = fmaf(__uint_as_float(xw[i] << 16), __uint_as_float(aw[i] << 16), acc);
          acc = fmaf(__uint_as_float(xw[i] & 0xffff0000u), __uint_as_float(aw[i] & 0xffff0000u), acc);
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) xa[qd] = acc;
    }
    __syncthreads();
  }
  const uint32_t* lut_lane = lut + lane;
  const int64_t row_bytes = H / 2;
  // Batches after the first read L2: keep the bulk prefetch two batches ahead.
  if (tid < 2 * IB) prefetch_items(p, touched, min(i0 + IB, i1), min(i0 + 3 * IB, i1));
  for (int b0 = i0; b0 < i1; b0 += IB) {
    const int nb = min(IB, i1 - b0);
    if (b0 > i0 && tid < IB) prefetch_items(p, touched, min(b0 + 2 * IB, i1), min(b0 + 3 * IB, i1));
    // Issue every load of the batch first (HBM latency is hidden by the batch).
    // 16-byte loads: a lane's 32 k of a span lie in k-block 2 * span + t / 2.
    uint4 pk[IB][KBW][2];
    float am[IB][KBW][2];
#pragma unroll
    for (int ii = 0; ii < IB; ++ii) {
      const int it = b0 + (ii < nb ? ii : 0);
      const int u = it / ipe, rb = it % ipe;
      const int64_t grow = static_cast<int64_t>(touched[u]) * 2 * I + rb * 8 + g;  // gate row of lane's MMA row g
      const uint8_t* gp = p.gu_packed + grow * row_bytes + 16 * t;
      const uint8_t* up = gp + static_cast<int64_t>(I) * row_bytes;
      const float* ga = p.gu_absmax + grow * KB;
      const float* ua = ga + static_cast<int64_t>(I) * KB;
#pragma unroll
      for (int q2 = 0; q2 < KBW; ++q2) {
        const int sp = warp + kWarps * q2;
        const int kb = 2 * sp + (t >> 1);
        if (ii < nb && kb < KB) {
          pk[ii][q2][0] = ld_stream_u4(gp + sp * 64);
          pk[ii][q2][1] = ld_stream_u4(up + sp * 64);
          am[ii][q2][0] = __ldg(ga + kb);
          am[ii][q2][1] = __ldg(ua + kb);
        } else {
          pk[ii][q2][0] = pk[ii][q2][1] = make_uint4(0, 0, 0, 0);
          am[ii][q2][0] = am[ii][q2][1] = 0.f;
        }
      }
    }
#pragma unroll
    for (int ii = 0; ii < IB; ++ii) {
      if (ii >= nb) break;
      const int u = (b0 + ii) / ipe;
      const bool has_g = (g < p.M) && slotmap[u * kMaxM + g] >= 0;  // token g routes to this expert
      const uint16_t* xrow = xs + g * xstride + 32 * t;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q2 = 0; q2 < KBW; ++q2) {
        const int sp = warp + kWarps * q2;
        if (2 * sp >= KB) break;
        uint4 xv[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        if (has_g && 2 * sp + (t >> 1) < KB) {
#pragma unroll
          for (int i = 0; i < 4; ++i) xv[i] = *reinterpret_cast<const uint4*>(xrow + sp * 128 + 8 * i);
        }
        span_mma(lut_lane, pk[ii][q2][0], pk[ii][q2][1], am[ii][q2][0], am[ii][q2][1], xv, acc);
      }
      red[(ii * kWarps + warp) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
    __syncthreads();
    if (warp < nb) {
      // Warp `warp` finishes item b0 + warp: sum the 16 partials in warp order.
      float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < kWarps; ++w) {
        const float4 v = red[(warp * kWarps + w) * 32 + lane];
        c.x += v.x;
        c.y += v.y;
        c.z += v.z;
        c.w += v.w;
      }
      const int it = b0 + warp;
      const int u = it / ipe, rb = it % ipe;
      const int e = touched[u];
      const int col = rb * 8 + g;  // h column == gate row index
      const float gate_v[2] = {c.x, c.y}, up_v[2] = {c.z, c.w};
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int tok = 2 * t + qq;
        if (tok >= p.M) continue;
        const int slot = slotmap[u * kMaxM + tok];
        if (slot < 0) continue;
        float gv = gate_v[qq], uv = up_v[qq];
        if (p.r > 0) {
          const uint16_t* bg = p.lora_B + (static_cast<int64_t>(e) * 2 * I + col) * p.r;
          const uint16_t* bu = p.lora_B + (static_cast<int64_t>(e) * 2 * I + I + col) * p.r;
          float dg = 0.f, du = 0.f;
          for (int rho = 0; rho < p.r; ++rho) {
            const float xv = xa[slot * p.r + rho];
            dg = fmaf(xv, bf16_bits_to_float(bg[rho]), dg);
            du = fmaf(xv, bf16_bits_to_float(bu[rho]), du);
          }
          gv = fmaf(p.lora_scale, dg, gv);
          uv = fmaf(p.lora_scale, du, uv);
        }
        p.h[static_cast<int64_t>(slot) * I + col] = float_to_bf16_bits(silu_f32(gv) * uv);
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Kernel B: down rows of every touched expert, weighted combine -> out.
__global__ void __launch_bounds__(kThreads, 1) decode_down_kernel(DecodeParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const Layout L = make_layout(false, p.M, p.k, p.E, p.H, 0);
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
  float4* red = reinterpret_cast<float4*>(smem + L.red);
  float* w_s = reinterpret_cast<float*>(smem + L.w);
  int* touched = reinterpret_cast<int*>(smem + L.touched);
  int* slotmap = reinterpret_cast<int*>(smem + L.slotmap);
  __shared__ int nU_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, I = p.I, KB = I / 64;
  // The down kernel starts once the gate_up kernel's CTAs leave the SMs; it
  // builds its codebook table, waits for that kernel's results (h and the
  // routing it published) and reads the routing instead of recomputing it.
  fill_lut_warps(lut, 0);
  pdl_wait();  // h and the routing written by the gate_up kernel are visible from here on
  {
    const int S = p.M * p.k;
    const int* m_touched = p.meta + 4;
    const int* m_slotmap = m_touched + S;
    const float* m_w = reinterpret_cast<const float*>(m_slotmap + S * kMaxM);
    const int n = __ldcg(p.meta);
    if (tid == 0) nU_s = n;
    for (int i = tid; i < n; i += blockDim.x) touched[i] = __ldcg(m_touched + i);
    for (int i = tid; i < n * kMaxM; i += blockDim.x) slotmap[i] = __ldcg(m_slotmap + i);
    for (int i = tid; i < S; i += blockDim.x) w_s[i] = __ldcg(m_w + i);
  }
  __syncthreads();
  const int nU = nU_s;
  const int NSP = (KB + 1) / 2;  // spans of 128 k (two absmax blocks) in a down row
  const int npairs = nU * NSP;   // (expert, span) pairs of one row block
  const int g = lane >> 2, t = lane & 3;
  const uint32_t* lut_lane = lut + lane;
  const int64_t row_bytes = I / 2;
  for (int rb = blockIdx.x; rb < H / 16; rb += gridDim.x) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int pb = warp; pb < npairs; pb += kWarps * kPairSlots) {
      uint4 pk[kPairSlots][2];
      float am[kPairSlots][2];
      uint4 hx[kPairSlots][4];
      float wc[kPairSlots][2];
#pragma unroll
      for (int sl = 0; sl < kPairSlots; ++sl) {
        const int pi = pb + kWarps * sl;
        pk[sl][0] = pk[sl][1] = make_uint4(0, 0, 0, 0);
        am[sl][0] = am[sl][1] = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) hx[sl][i] = make_uint4(0, 0, 0, 0);
        wc[sl][0] = wc[sl][1] = 0.f;
        if (pi < npairs) {
          const int u = pi / NSP, sp = pi % NSP;
          const int kb = 2 * sp + (t >> 1);  // this lane's 32 k of the span lie in k-block kb
          const int64_t row = static_cast<int64_t>(touched[u]) * H + rb * 16 + g;
          if (kb < KB) {
            const uint8_t* rp = p.dn_packed + row * row_bytes + sp * 64 + 16 * t;
            pk[sl][0] = ld_stream_u4(rp);
            pk[sl][1] = ld_stream_u4(rp + 8 * row_bytes);
            am[sl][0] = __ldg(p.dn_absmax + row * KB + kb);
            am[sl][1] = __ldg(p.dn_absmax + (row + 8) * KB + kb);
            const int slot_g = (g < p.M) ? slotmap[u * kMaxM + g] : -1;
            if (slot_g >= 0) {
              const uint16_t* hr = p.h + static_cast<int64_t>(slot_g) * I + sp * 128 + 32 * t;
#pragma unroll
              for (int i = 0; i < 4; ++i) hx[sl][i] = *reinterpret_cast<const uint4*>(hr + 8 * i);
            }
          }
          const int s0 = (2 * t < p.M) ? slotmap[u * kMaxM + 2 * t] : -1;
          const int s1 = (2 * t + 1 < p.M) ? slotmap[u * kMaxM + 2 * t + 1] : -1;
          wc[sl][0] = s0 >= 0 ? w_s[s0] : 0.f;
          wc[sl][1] = s1 >= 0 ? w_s[s1] : 0.f;
        }
      }
#pragma unroll
      for (int sl = 0; sl < kPairSlots; ++sl) {
        if (pb + kWarps * sl >= npairs) break;
        float tmp[4] = {0.f, 0.f, 0.f, 0.f};
        span_mma(lut_lane, pk[sl][0], pk[sl][1], am[sl][0], am[sl][1], hx[sl], tmp);
        acc[0] = fmaf(tmp[0], wc[sl][0], acc[0]);
        acc[1] = fmaf(tmp[1], wc[sl][1], acc[1]);
        acc[2] = fmaf(tmp[2], wc[sl][0], acc[2]);
        acc[3] = fmaf(tmp[3], wc[sl][1], acc[3]);
      }
    }
    red[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    if (warp == 0) {
      float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < kWarps; ++w) {
        const float4 v = red[w * 32 + lane];
        c.x += v.x;
        c.y += v.y;
        c.z += v.z;
        c.w += v.w;
      }
      const int row0 = rb * 16 + g;
      const float v[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int q2 = 0; q2 < 4; ++q2) {
        const int tok = 2 * t + (q2 & 1);
        const int row = row0 + ((q2 >> 1) ? 8 : 0);
        if (tok < p.M) p.out[static_cast<int64_t>(tok) * H + row] = float_to_bf16_bits(v[q2]);
      }
    }
    __syncthreads();
  }
}

template <int KBW, int SLOTS>
cudaError_t raise_smem_limits(size_t smem_a, size_t smem_b) {
  cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(decode_gate_up_kernel<KBW, SLOTS>), smem_a);
  if (err != cudaSuccess) return err;
  return ensure_smem_limit(reinterpret_cast<const void*>(decode_down_kernel), smem_b);
}

template <int KBW, int SLOTS>
cudaError_t launch_pair(const DecodeParams& p, int sm_count, size_t smem_a, size_t smem_b, cudaStream_t stream) {
  cudaError_t aerr = raise_smem_limits<KBW, SLOTS>(smem_a, smem_b);
  if (aerr != cudaSuccess) return aerr;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int nitems_upper = std::min(p.M * p.k, p.E) * (p.I / 8);
  cfg.gridDim = dim3(std::max(1, std::min(sm_count, nitems_upper)));
  cfg.dynamicSmemBytes = smem_a;
  {
    LaunchScope ls("decode.gate_up", stream);
    cudaError_t err = cudaLaunchKernelEx(&cfg, decode_gate_up_kernel<KBW, SLOTS>, p);
    if (err != cudaSuccess) return err;
  }
  cfg.gridDim = dim3(std::max(1, std::min(sm_count, p.H / 16)));
  cfg.dynamicSmemBytes = smem_b;
  LaunchScope ls("decode.down", stream);
  return cudaLaunchKernelEx(&cfg, decode_down_kernel, p);
}

struct DecodeWs {
  size_t h, meta, total;
};

// Workspace: the error word every workspace begins with (no decode kernel
// waits, so it stays untouched), h [M*k, I] bf16, then the published routing
// (4 + S * (2 + kMaxM) ints).
DecodeWs decode_ws(int64_t M, int k, int64_t I) {
  DecodeWs w;
  const int64_t S = M * k;
  w.h = 256;
  w.meta = w.h + align_up(static_cast<size_t>(S * I * 2), 256);
  w.total = w.meta + align_up(static_cast<size_t>(4 + S * (2 + kMaxM)) * 4, 256);
  return w;
}

}  // namespace

bool decode_supported(int64_t M, int64_t E, int k, int64_t H, int64_t I) {
  if (M < 1 || M > kMaxM || k > 32 || E > 512 || H > 128 * kWarps * kMaxKBW) return false;
  (void)I;
  DeviceInfo di;
  if (device_info(&di) != cudaSuccess) return false;
  const Layout a = make_layout(true, static_cast<int>(M), k, static_cast<int>(E), static_cast<int>(H), 16);
  const Layout b = make_layout(false, static_cast<int>(M), k, static_cast<int>(E), static_cast<int>(H), 0);
  const size_t lim = di.smem_optin - 1024;  // leave room for the kernels' static shared memory
  return a.total <= lim && b.total <= lim;
}

size_t decode_workspace_bytes(int64_t M, int64_t E, int k, int64_t H, int64_t I, int r) {
  (void)E;
  (void)H;
  (void)r;
  if (M < 1 || M > kMaxM) return 0;
  return decode_ws(M, k, I).total;
}

cudaError_t launch_decode_forward(const DecodeArgs& a, cudaStream_t stream) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const e4b_expert_stack* w = a.w;
  const int r = w->lora_A ? w->lora_r : 0;
  const DecodeWs ws = decode_ws(a.M, a.k, w->I);
  DecodeParams p{};
  p.x = a.x;
  p.logits = a.logits;
  p.M = static_cast<int>(a.M);
  p.k = a.k;
  p.E = static_cast<int>(w->E);
  p.H = static_cast<int>(w->H);
  p.I = static_cast<int>(w->I);
  p.renorm = a.renormalize ? 1 : 0;
  p.gu_packed = w->gu_packed;
  p.gu_absmax = w->gu_absmax;
  p.dn_packed = w->dn_packed;
  p.dn_absmax = w->dn_absmax;
  p.lora_A = r ? w->lora_A : nullptr;
  p.lora_B = r ? w->lora_B : nullptr;
  p.r = r;
  p.lora_scale = r ? w->lora_alpha / static_cast<float>(r) : 0.f;
  p.h = reinterpret_cast<uint16_t*>(static_cast<char*>(a.workspace) + ws.h);
  p.meta = reinterpret_cast<int*>(static_cast<char*>(a.workspace) + ws.meta);
  p.out = a.out;
  const size_t smem_a = make_layout(true, p.M, p.k, p.E, p.H, r).total;
  const size_t smem_b = make_layout(false, p.M, p.k, p.E, p.H, 0).total;
  if (kbw_of(p.H) == 1) {
    if (slots_for(p.M, p.H) == 8) return launch_pair<1, 8>(p, di.sm_count, smem_a, smem_b, stream);
    return launch_pair<1, 4>(p, di.sm_count, smem_a, smem_b, stream);
  }
  return launch_pair<2, 4>(p, di.sm_count, smem_a, smem_b, stream);
}

}  // namespace e4b
