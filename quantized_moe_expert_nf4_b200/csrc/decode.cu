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
//             (bf16, [M*k, I], slot order).  Once its ring is full, its
//             producer prefetches the touched experts' down rows into L2.
//   kernel B  the same routing, then for every block of 16 output rows of H
//             the down rows of every touched expert, with the routing weights
//             folded in, so the combine happens inside the CTA in a fixed
//             order (deterministic).  Its weight stream starts before kernel A
//             has finished; only the h rows wait for it.
//
// Only experts that some token selected are read.  Each CTA streams its share
// of the packed rows and their absmax through a ring of shared-memory stages
// filled by bulk asynchronous copies (one producer warp, one copy per row,
// mbarrier transaction counts), so HBM keeps streaming while the math warps
// decode.  The 16 math warps split K in spans of two absmax blocks (128 k) and
// run mma.sync m16n8k16 with the weight rows as MMA rows and the <= 8 tokens as
// the 8 MMA columns.  Nibbles become bf16 through a per-lane replicated byte ->
// bf16x2 codebook table in shared memory (lane l reads only bank l); every MMA
// stays inside one absmax block, so the fp32 absmax scales its products.  Rows
// are staged 16 bytes apart from the next row's bank so that the fragment loads
// are conflict-free.
#include <algorithm>
#include <string>

#include "async.cuh"
#include "common.cuh"
#include "e4b_internal.h"
#include "topk.cuh"

namespace e4b {
namespace {

constexpr int kMaxM = 8;
constexpr int kMath = 16;                  // math warps of the down kernel (and at most of gate_up)
constexpr int kProducer = kMath;           // down kernel: warp issuing the bulk copies
constexpr int kEpilogue = kMath + 1;       // down kernel: warp summing the math warps' partials
constexpr int kWarps = kMath + 2;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxKBW = 2;                 // spans per math warp per row: K <= 128 * 16 * 2 = 4096
constexpr int kMaxStages = 12;
constexpr int kMinStages = 2;
constexpr uint32_t kRedLaneBytes = 32 * 16;  // one float4 per lane of a math warp
constexpr unsigned long long kPrefetchLimit = 64ull << 20;  // L2 prefetch of the down rows, bytes
constexpr uint32_t kPrefetchChunk = 32 * 1024;
constexpr uint32_t kRedBytes = kMath * kRedLaneBytes;

struct DecodeParams {
  const uint16_t* x;
  const float* logits;
  int M, k, E, H, I;
  int renorm;
  const uint8_t* gu_packed;
  const float* gu_absmax;
  const uint8_t* dn_packed;
  const float* dn_absmax;
  int quant;  // e4b_quant_type of both stacks
  const uint16_t* lora_A;
  const uint16_t* lora_B;
  int r;
  float lora_scale;
  uint16_t* h;    // [S, I] bf16 (slot order)
  uint16_t* out;  // [M, H] bf16
  int* err;       // error word (a bounded wait gave up)
  int stages_a, stages_b;
};

__host__ __device__ inline uint32_t al(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// One ring stage: 16 rows of K/2 packed bytes, their absmax, optionally the h
// rows of the stage's tokens (kernel B) and the math warps' partials (kernel A).
struct RingGeom {
  uint32_t ps;       // shared-memory stride of a packed row, bytes (K/2 + 16)
  uint32_t sa;       // stride of an absmax row, floats
  bool am_rows;      // absmax copied row by row (strided) or as two 8-row chunks
  uint32_t am_off;   // offsets inside the stage, bytes
  uint32_t h_off;
  uint32_t hs;       // stride of an h row, bytes (2 K + 16)
  uint32_t red_off;
  uint32_t bytes;    // stage size (128-byte multiple)
};

// K = row length of the streamed matrix; h_rows = token rows of h per stage;
// red_warps = math warps whose partials the stage holds (0: none).
__host__ __device__ inline RingGeom ring_geom(int K, int h_rows, int red_warps) {
  RingGeom g;
  const int KB = K / 64;
  g.ps = static_cast<uint32_t>(K / 2 + 16);
  // A row's absmax can be copied on its own only if it is a 16-byte multiple;
  // then the stride is KB rounded up to 4 (mod 8), which puts the 8 rows of a
  // fragment on 8 distinct groups of 4 banks.  Otherwise the rows of a chunk
  // stay contiguous (KB is not a multiple of 4: at most 2-way conflicts).
  g.am_rows = (KB % 4) == 0;
  g.sa = static_cast<uint32_t>(g.am_rows ? (KB % 8 == 4 ? KB : KB + 4) : KB);
  g.am_off = 16 * g.ps;
  g.h_off = g.am_off + al(16 * g.sa * 4, 16);
  g.hs = static_cast<uint32_t>(2 * K + 16);
  g.red_off = g.h_off + static_cast<uint32_t>(h_rows) * g.hs;
  g.bytes = al(g.red_off + static_cast<uint32_t>(red_warps) * kRedLaneBytes, 128);
  return g;
}

struct Layout {
  uint32_t lut, ids, w, uidx, touched, slotmap, xa, bars, seq, red, ring, total;
};

// Shared-memory carve of kernel A (gate_up) or B (down) with `stages` ring stages.
__host__ __device__ inline Layout make_layout(bool is_a, int M, int k, int E, int r, const RingGeom& g,
                                              int stages) {
  Layout L;
  uint32_t o = 0;
  const int S = M * k;
  L.lut = o;
  o += 256 * 32 * 4;
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
  L.bars = o;
  o = al(o + (is_a ? 3 * stages : 2 * stages + 4) * 8, 16);
  L.seq = o;
  if (!is_a) o = al(o + stages * 4, 16);  // stage held by each ring slot
  L.red = o;
  if (!is_a) o += 2 * kRedBytes;  // partials of two row blocks
  L.ring = al(o, 128);
  L.total = L.ring + static_cast<uint32_t>(stages) * g.bytes;
  return L;
}

// Deepest ring that fits `limit` bytes, or 0.
inline int pick_stages(bool is_a, int M, int k, int E, int r, const RingGeom& g, size_t limit) {
  for (int s = kMaxStages; s >= kMinStages; --s)
    if (make_layout(is_a, M, k, E, r, g, s).total <= limit) return s;
  return 0;
}

__device__ __forceinline__ void mma_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bulk asynchronous copy global -> this CTA's shared memory, completing on `bar`
// (both addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// One span (128 k = 2 absmax blocks) of a 16-row tile, accumulated into c.
// In each k-block h of the span, thread (g, t) owns physical k [16t, 16t+16):
// 8 packed bytes of row g (w0[2h], w0[2h+1]) and of row g+8 (w1[2h], w1[2h+1])
// and the matching 16 bf16 of its token column g (x[2h], x[2h+1]).  MMAs 0-3
// cover the first k-block and 4-7 the second, so every MMA sees one absmax per
// row: the products of a k-block are scaled in fp32 afterwards (a0 = row g,
// a1 = row g+8), with no rounding of the scale.  MMA j of a k-block takes bytes
// 2j and 2j+1 of the thread's 8 bytes; K is permuted identically on both
// operands.  A k-block past the end of the row must come with zero x and scale.
__device__ __forceinline__ void span_mma(const uint32_t* __restrict__ lut_lane, const uint32_t w0[4],
                                         const uint32_t w1[4], const float a0[2], const float a1[2],
                                         const uint4 x[4], float c[4]) {
  auto pair = [&](uint32_t word, int byte) { return lut_lane[((word >> (8 * byte)) & 0xffu) << 5]; };
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t xw[8] = {x[2 * h].x,     x[2 * h].y,     x[2 * h].z,     x[2 * h].w,
                            x[2 * h + 1].x, x[2 * h + 1].y, x[2 * h + 1].z, x[2 * h + 1].w};
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int b = 2 * (j & 1);
      const uint32_t wa = w0[2 * h + (j >> 1)], wb = w1[2 * h + (j >> 1)];
      mma_16816(d, pair(wa, b), pair(wb, b), pair(wa, b + 1), pair(wb, b + 1), xw[2 * j], xw[2 * j + 1]);
    }
    c[0] = fmaf(a0[h], d[0], c[0]);
    c[1] = fmaf(a0[h], d[1], c[1]);
    c[2] = fmaf(a1[h], d[2], c[2]);
    c[3] = fmaf(a1[h], d[3], c[3]);
  }
}

// Loads the span's fragment of rows g and g+8 of a stage (two 8-byte pieces
// per row, one per k-block) and their absmax; zeros past the row's end.
__device__ __forceinline__ void load_span(const RingGeom& G, const unsigned char* st, int g, int t, int sp, int KB,
                                          uint32_t w0[4], uint32_t w1[4], float a0[2], float a1[2]) {
  const float* am = reinterpret_cast<const float*>(st + G.am_off);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int kb = 2 * sp + h;
    uint2 v0 = make_uint2(0u, 0u), v1 = make_uint2(0u, 0u);
    a0[h] = a1[h] = 0.f;
    if (kb < KB) {
      v0 = *reinterpret_cast<const uint2*>(st + g * G.ps + sp * 64 + 32 * h + 8 * t);
      v1 = *reinterpret_cast<const uint2*>(st + (g + 8) * G.ps + sp * 64 + 32 * h + 8 * t);
      a0[h] = am[g * G.sa + kb];
      a1[h] = am[(g + 8) * G.sa + kb];
    }
    w0[2 * h] = v0.x;
    w0[2 * h + 1] = v0.y;
    w1[2 * h] = v1.x;
    w1[2 * h + 1] = v1.y;
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
// b * 32 + l), entries first, first + step, ... written by the calling warp.
__device__ __forceinline__ void fill_lut(uint32_t* lut, int quant, int first, int step) {
  const int lane = threadIdx.x & 31;
  const float cbl = codebook_entry(quant, lane & 15);
  for (int b = first; b < 256; b += step) {
    const float hi = __shfl_sync(0xffffffffu, cbl, b >> 4);
    const float lo = __shfl_sync(0xffffffffu, cbl, b & 15);
    lut[b * 32 + lane] = pack_bf16x2(hi, lo);
  }
}

// Prologue of both kernels: warps < M route one token each while the other
// warps build the codebook table.  Then the touched experts (ascending id) and
// slotmap[u][t] = slot of token t in expert touched[u] (or -1) are built.  Ends
// with a block barrier (which also publishes the mbarrier initialisation).
__device__ void route_prologue(const DecodeParams& p, uint32_t* lut, int* ids_s, float* w_s, int* uidx,
                               int* touched, int* slotmap, int* nU_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.M * p.k;
  for (int e = tid; e < p.E; e += blockDim.x) uidx[e] = -1;
  const int nwarps = static_cast<int>(blockDim.x >> 5);
  if (warp < p.M) route_one(p, warp, ids_s, w_s);
  else fill_lut(lut, p.quant, warp - p.M, nwarps - p.M);
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

// Issues the copies of one stage: 16 packed rows (rows [0, 8) from `row_a`,
// [8, 16) from `row_b`) and their absmax, announcing `extra` more bytes that
// the caller copies itself.  Called by the whole producer warp.
__device__ __forceinline__ void issue_rows(const RingGeom& G, unsigned char* st, uint64_t* full,
                                           const uint8_t* packed, const float* absmax, int K, int64_t row_a,
                                           int64_t row_b, uint32_t extra) {
  const int lane = threadIdx.x & 31;
  const int KB = K / 64;
  const uint32_t rowb = static_cast<uint32_t>(K / 2);
  if (lane == 0) mbar_arrive_expect_tx(full, 16 * rowb + 16 * KB * 4 + extra);
  __syncwarp();
  if (lane < 16) {
    const int64_t row = (lane < 8 ? row_a : row_b) + (lane & 7);
    bulk_g2s(st + lane * G.ps, packed + row * rowb, rowb, full);
  } else if (G.am_rows) {
    const int i = lane - 16;
    const int64_t row = (i < 8 ? row_a : row_b) + (i & 7);
    bulk_g2s(st + G.am_off + i * G.sa * 4, absmax + row * KB, KB * 4, full);
  } else if (lane < 18) {
    const int i = lane - 16;
    bulk_g2s(st + G.am_off + i * 8 * G.sa * 4, absmax + (i == 0 ? row_a : row_b) * KB, 8 * KB * 4, full);
  }
}

// Waits (bounded) until ring slot s holds stage j and its copies have landed.
// A warp that takes only some stages of the ring can reach stage j before the
// slot's previous stage j - stages has even landed; the parity of the full
// barrier alone would then look complete.  The producer publishes j in seq[s]
// (release) after the slot's previous stage was consumed, so once seq[s] == j
// is seen (acquire) the barrier is at the phase of j or just past it, where
// the parity wait is exact.
__device__ __forceinline__ bool wait_stage(uint64_t* full, const int* seq, int s, int j, int stages) {
  auto ready = [&]() { return ld_acquire_shared(seq + s) == j && mbar_try_wait(&full[s], (j / stages) & 1); };
  if (ready()) return true;
  const unsigned long long t0 = global_ns();
  while (!ready())
    if (global_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// Drains the producer's copies in flight (bounded) before the CTA exits.
__device__ __forceinline__ void drain_ring(uint64_t* full, int issued, int stages) {
  for (int j = max(0, issued - stages); j < issued; ++j) mbar_wait(&full[j % stages], (j / stages) & 1);
}

// L2 prefetch of this CTA's share (by 32 KB chunks across the grid and the
// calling warp's lanes) of the touched experts' down rows and absmax, at most
// kPrefetchLimit bytes in all.
__device__ __forceinline__ void prefetch_down_rows(const DecodeParams& p, const int* touched, int nU) {
  const int lane = threadIdx.x & 31;
  const uint64_t per_expert = static_cast<uint64_t>(p.H) * p.I / 2;
  const uint64_t per_expert_am = static_cast<uint64_t>(p.H) * (p.I / 64) * 4;
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
      const uint64_t nb = min(static_cast<uint64_t>(kPrefetchChunk), per_expert - off);
      prefetch_l2(p.dn_packed + e * per_expert + off, static_cast<uint32_t>(nb));
    } else {
      const uint64_t off = (qq - chunks_pk) * kPrefetchChunk;
      const uint64_t nb = min(static_cast<uint64_t>(kPrefetchChunk), per_expert_am - off);
      prefetch_l2(reinterpret_cast<const unsigned char*>(p.dn_absmax) + e * per_expert_am + off,
                  static_cast<uint32_t>(nb));
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel A: gate_up + SwiGLU (+ LoRA delta) -> h.  MATH math warps with KBW
// spans each (MATH * KBW >= the spans of a row), then the producer and the
// epilogue warp.
template <int KBW, int MATH>
__global__ void __launch_bounds__((MATH + 2) * 32, 1) decode_gate_up_kernel(DecodeParams p) {
  constexpr int kProducerA = MATH, kEpilogueA = MATH + 1;
  extern __shared__ __align__(128) unsigned char smem[];
  const int RS = p.stages_a;
  const RingGeom G = ring_geom(p.H, 0, MATH);
  const Layout L = make_layout(true, p.M, p.k, p.E, p.r, G, RS);
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
  int* ids_s = reinterpret_cast<int*>(smem + L.ids);
  float* w_s = reinterpret_cast<float*>(smem + L.w);
  int* uidx = reinterpret_cast<int*>(smem + L.uidx);
  int* touched = reinterpret_cast<int*>(smem + L.touched);
  int* slotmap = reinterpret_cast<int*>(smem + L.slotmap);
  float* xa = reinterpret_cast<float*>(smem + L.xa);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);  // stage landed
  uint64_t* done = full + RS;                                    // math warps' partials written
  uint64_t* empty = done + RS;                                   // stage free again
  unsigned char* ring = smem + L.ring;
  __shared__ int nU_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, I = p.I, KB = H / 64, NSP = (KB + 1) / 2;
  const int nact = min(MATH, NSP);  // math warps with a span
  if (tid == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], nact);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  pdl_wait();               // the inputs of this call are final
  pdl_launch_dependents();  // the down kernel may launch and start its weight stream
  route_prologue(p, lut, ids_s, w_s, uidx, touched, slotmap, &nU_s);
  const int nU = nU_s;
  const int ipe = I / 8;  // items per expert
  const int nitems = nU * ipe;
  // A contiguous run of items per CTA: consecutive items are consecutive rows.
  const int q = nitems / gridDim.x, rem = nitems % gridDim.x;
  const int i0 = blockIdx.x * q + min(static_cast<int>(blockIdx.x), rem);
  const int n = q + (static_cast<int>(blockIdx.x) < rem ? 1 : 0);

  const int g = lane >> 2, t = lane & 3;
  const int S = p.M * p.k;
  if (p.r > 0) {
    // LoRA first factor per slot: xa[s, rho] = x[token(s)] . lora_A[e(s), rho]
    if (warp < MATH) {
      for (int qd = warp; qd < S * p.r; qd += MATH) {
        const int s = qd / p.r, rho = qd % p.r;
        const uint16_t* xr = p.x + static_cast<int64_t>(s / p.k) * H;
        const uint16_t* la = p.lora_A + (static_cast<int64_t>(ids_s[s]) * p.r + rho) * H;
        float acc = 0.f;
        for (int kk = lane * 8; kk < H; kk += 256) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xr + kk);
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
    }
    __syncthreads();
  }

  if (warp == kProducerA) {
    int issued = 0;
    for (int j = 0; j < n; ++j) {
      const int s = j % RS;
      if (j >= RS && !mbar_wait(&empty[s], ((j / RS) - 1) & 1)) {
        record_error(p.err, kErrWaitEmpty);
        break;
      }
      const int it = i0 + j, u = it / ipe, rb = it % ipe;
      const int64_t grow = static_cast<int64_t>(touched[u]) * 2 * I + rb * 8;
      issue_rows(G, ring + s * G.bytes, &full[s], p.gu_packed, p.gu_absmax, H, grow, grow + I, 0);
      ++issued;
      // Once the ring is full: this CTA's share of the touched experts' down
      // rows into L2.  The down kernel cannot share an SM with this one, so
      // without it that kernel's stream would start only after this one ends.
      if (issued == min(n, RS)) prefetch_down_rows(p, touched, nU);
    }
    if (n == 0) prefetch_down_rows(p, touched, nU);
    drain_ring(full, issued, RS);
  } else if (warp == kEpilogueA) {
    for (int j = 0; j < n; ++j) {
      const int s = j % RS;
      if (!mbar_wait(&done[s], (j / RS) & 1)) {
        record_error(p.err, kErrWaitFull);
        break;
      }
      // Sum the partials in warp order, then hand the stage back.
      const float4* red = reinterpret_cast<const float4*>(ring + s * G.bytes + G.red_off);
      float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < nact; ++w) {
        const float4 v = red[w * 32 + lane];
        c.x += v.x;
        c.y += v.y;
        c.z += v.z;
        c.w += v.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      const int it = i0 + j;
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
  } else if (warp < nact) {
    // The warp's spans are the same in every item: its slice of x (token g of
    // the MMA column) stays in registers.  Columns of tokens that do not route
    // to an item's expert compute values that the epilogue never stores.
    uint4 xv[KBW][4];
#pragma unroll
    for (int q2 = 0; q2 < KBW; ++q2) {
      const int sp = warp + MATH * q2;
      const uint16_t* xr = p.x + static_cast<int64_t>(g) * H + sp * 128 + 16 * t;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool live = g < p.M && sp < NSP && 2 * sp + (i >> 1) < KB;  // k-block i / 2 of the span
        xv[q2][i] = live ? *reinterpret_cast<const uint4*>(xr + 64 * (i >> 1) + 8 * (i & 1)) : make_uint4(0, 0, 0, 0);
      }
    }
    const uint32_t* lut_lane = lut + lane;
    for (int j = 0; j < n; ++j) {
      const int s = j % RS;
      if (!mbar_wait(&full[s], (j / RS) & 1)) {
        record_error(p.err, kErrWaitFull);
        break;
      }
      const unsigned char* st = ring + s * G.bytes;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q2 = 0; q2 < KBW; ++q2) {
        const int sp = warp + MATH * q2;
        if (sp >= NSP) break;
        uint32_t w0[4], w1[4];
        float a0[2], a1[2];
        load_span(G, st, g, t, sp, KB, w0, w1, a0, a1);
        span_mma(lut_lane, w0, w1, a0, a1, xv[q2], acc);
      }
      float4* red = reinterpret_cast<float4*>(ring + s * G.bytes + G.red_off);
      red[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&done[s]);
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel B: down rows of every touched expert, weighted combine -> out.
// Stage j of a CTA = (row block blockIdx.x + (j / nU) * gridDim.x, expert
// touched[j % nU]): 16 down rows over all of K = I plus the h rows of the
// tokens routed to that expert.  The math warps take the (stage, span) pairs
// of a row block in turn; each keeps one running sum per row block.
__global__ void __launch_bounds__(kThreads, 1) decode_down_kernel(DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int RS = p.stages_b;
  const RingGeom G = ring_geom(p.I, p.M, 0);
  const Layout L = make_layout(false, p.M, p.k, p.E, 0, G, RS);
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
  int* ids_s = reinterpret_cast<int*>(smem + L.ids);
  float* w_s = reinterpret_cast<float*>(smem + L.w);
  int* uidx = reinterpret_cast<int*>(smem + L.uidx);
  int* touched = reinterpret_cast<int*>(smem + L.touched);
  int* slotmap = reinterpret_cast<int*>(smem + L.slotmap);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);  // stage landed
  uint64_t* empty = full + RS;                                   // every span of the stage consumed
  uint64_t* rdone = empty + RS;                                  // [2] partials of a row block written
  uint64_t* rfree = rdone + 2;                                   // [2] partials of a row block summed
  int* seq = reinterpret_cast<int*>(smem + L.seq);              // stage held by each slot
  float4* red = reinterpret_cast<float4*>(smem + L.red);         // [2][kMath][32]
  unsigned char* ring = smem + L.ring;
  __shared__ int nU_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, I = p.I, KB = I / 64, NSP = (KB + 1) / 2;
  if (tid == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NSP);
      seq[s] = -1;
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&rdone[b], kMath);
      mbar_init(&rfree[b], 1);
    }
    fence_mbar_init();
  }
  // Routing again (it reads only this call's logits, final before the gate_up
  // kernel let this one launch); h is waited for by the producer alone.
  route_prologue(p, lut, ids_s, w_s, uidx, touched, slotmap, &nU_s);
  const int nU = nU_s;
  const int nrb_all = H / 16;
  const int nrb = (nrb_all - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                  static_cast<int>(gridDim.x);  // row blocks of this CTA
  const int T = nrb * nU;                       // stages of this CTA
  const int g = lane >> 2, t = lane & 3;

  if (warp == kProducer) {
    const uint32_t hrow = static_cast<uint32_t>(I) * 2;
    auto issue_w = [&](int j) {
      const int s = j % RS, u = j % nU;
      if (lane == 0) st_release_shared(&seq[s], j);  // the slot's previous stage is consumed
      __syncwarp();
      const int rb = static_cast<int>(blockIdx.x) + (j / nU) * static_cast<int>(gridDim.x);
      const bool has = lane < p.M && slotmap[u * kMaxM + lane] >= 0;
      const int nh = __popc(__ballot_sync(0xffffffffu, has));
      const int64_t row0 = static_cast<int64_t>(touched[u]) * H + rb * 16;
      issue_rows(G, ring + s * G.bytes, &full[s], p.dn_packed, p.dn_absmax, I, row0, row0 + 8, nh * hrow);
    };
    auto issue_h = [&](int j) {
      const int s = j % RS, u = j % nU;
      if (lane < p.M) {
        const int slot = slotmap[u * kMaxM + lane];
        if (slot >= 0)
          bulk_g2s(ring + s * G.bytes + G.h_off + lane * G.hs, p.h + static_cast<int64_t>(slot) * I, hrow, &full[s]);
      }
    };
    // The first stages' weights stream while the gate_up kernel finishes.
    const int pre = min(RS, T);
    for (int j = 0; j < pre; ++j) issue_w(j);
    pdl_wait();  // h written by the gate_up kernel is visible from here on
    for (int j = 0; j < pre; ++j) issue_h(j);
    int issued = pre;
    for (int j = pre; j < T; ++j) {
      const int s = j % RS;
      if (!mbar_wait(&empty[s], ((j / RS) - 1) & 1)) {
        record_error(p.err, kErrWaitEmpty);
        break;
      }
      issue_w(j);
      issue_h(j);
      ++issued;
    }
    drain_ring(full, issued, RS);
  } else if (warp == kEpilogue) {
    for (int rbi = 0; rbi < nrb; ++rbi) {
      const int par = rbi & 1;
      if (!mbar_wait(&rdone[par], (rbi >> 1) & 1)) {
        record_error(p.err, kErrWaitFull);
        break;
      }
      float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < kMath; ++w) {
        const float4 v = red[(par * kMath + w) * 32 + lane];
        c.x += v.x;
        c.y += v.y;
        c.z += v.z;
        c.w += v.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfree[par]);
      const int rb = static_cast<int>(blockIdx.x) + rbi * static_cast<int>(gridDim.x);
      const int row0 = rb * 16 + g;
      const float v[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int q2 = 0; q2 < 4; ++q2) {
        const int tok = 2 * t + (q2 & 1);
        const int row = row0 + ((q2 >> 1) ? 8 : 0);
        if (tok < p.M) p.out[static_cast<int64_t>(tok) * H + row] = float_to_bf16_bits(v[q2]);
      }
    }
  } else {
    const uint32_t* lut_lane = lut + lane;
    const int npr = nU * NSP;  // (expert, span) pairs of one row block
    bool ok = true;
    for (int rbi = 0; rbi < nrb && ok; ++rbi) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int qp = warp; qp < npr; qp += kMath) {
        const int u = qp / NSP, sp = qp % NSP;
        const int j = rbi * nU + u, s = j % RS;
        if (!wait_stage(full, seq, s, j, RS)) {
          record_error(p.err, kErrWaitFull);
          ok = false;
          break;
        }
        const unsigned char* st = ring + s * G.bytes;
        uint32_t w0[4], w1[4];
        float a0[2], a1[2];
        load_span(G, st, g, t, sp, KB, w0, w1, a0, a1);
        uint4 hx[4];
        const int slot_g = (g < p.M) ? slotmap[u * kMaxM + g] : -1;  // h row of token g landed
        const unsigned char* hr = st + G.h_off + g * G.hs + sp * 256 + 32 * t;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const bool live = slot_g >= 0 && 2 * sp + (i >> 1) < KB;  // k-block i / 2 of the span
          hx[i] = live ? *reinterpret_cast<const uint4*>(hr + 128 * (i >> 1) + 16 * (i & 1)) : make_uint4(0, 0, 0, 0);
        }
        const int s0 = (2 * t < p.M) ? slotmap[u * kMaxM + 2 * t] : -1;
        const int s1 = (2 * t + 1 < p.M) ? slotmap[u * kMaxM + 2 * t + 1] : -1;
        const float wc0 = s0 >= 0 ? w_s[s0] : 0.f, wc1 = s1 >= 0 ? w_s[s1] : 0.f;
        float tmp[4] = {0.f, 0.f, 0.f, 0.f};
        span_mma(lut_lane, w0, w1, a0, a1, hx, tmp);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        acc[0] = fmaf(tmp[0], wc0, acc[0]);
        acc[1] = fmaf(tmp[1], wc1, acc[1]);
        acc[2] = fmaf(tmp[2], wc0, acc[2]);
        acc[3] = fmaf(tmp[3], wc1, acc[3]);
      }
      if (!ok) break;
      // Publish this warp's sum for the row block (every warp, work or not).
      const int par = rbi & 1;
      if (rbi >= 2 && !mbar_wait(&rfree[par], ((rbi >> 1) - 1) & 1)) {
        record_error(p.err, kErrWaitEmpty);
        break;
      }
      red[(par * kMath + warp) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&rdone[par]);
    }
  }
}

template <int KBW, int MATH>
cudaError_t launch_pair(const DecodeParams& p, int sm_count, size_t smem_a, size_t smem_b, cudaStream_t stream) {
  cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(decode_gate_up_kernel<KBW, MATH>), smem_a);
  if (err != cudaSuccess) return err;
  err = ensure_smem_limit(reinterpret_cast<const void*>(decode_down_kernel), smem_b);
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3((MATH + 2) * 32);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int nitems_upper = std::min(p.M * p.k, p.E) * (p.I / 8);
  cfg.gridDim = dim3(std::max(1, std::min(sm_count, nitems_upper)));
  cfg.dynamicSmemBytes = smem_a;
  {
    LaunchScope ls("decode.gate_up", stream);
    err = cudaLaunchKernelEx(&cfg, decode_gate_up_kernel<KBW, MATH>, p);
    if (err != cudaSuccess) return err;
  }
  cfg.blockDim = dim3(kThreads);
  cfg.gridDim = dim3(std::max(1, std::min(sm_count, p.H / 16)));
  cfg.dynamicSmemBytes = smem_b;
  LaunchScope ls("decode.down", stream);
  return cudaLaunchKernelEx(&cfg, decode_down_kernel, p);
}

struct DecodeWs {
  size_t h, meta, total;
};

// Workspace: the error word every workspace begins with (256-byte slot),
// h [M*k, I] bf16, then 4 + S * (2 + kMaxM) ints (kept for the layout's size).
DecodeWs decode_ws(int64_t M, int k, int64_t I) {
  DecodeWs w;
  const int64_t S = M * k;
  w.h = 256;
  w.meta = w.h + align_up(static_cast<size_t>(S * I * 2), 256);
  w.total = w.meta + align_up(static_cast<size_t>(4 + S * (2 + kMaxM)) * 4, 256);
  return w;
}

// Math warps of the gate_up kernel and spans per warp for rows of H: the
// fewest span slots (MATH * KBW) that cover the row's spans, so that no warp
// of an item waits for another with more spans.
struct MathSplit {
  int kbw, math;
};
inline MathSplit math_split(int H) {
  const int nsp = (H / 64 + 1) / 2;
  if (nsp <= kMath) return {1, kMath};
  if (nsp <= 24) return {2, 12};
  return {2, kMath};
}

struct Stages {
  int a, b;
  size_t smem_a, smem_b;
};

Stages plan_stages(int M, int k, int E, int H, int I, int r, size_t limit) {
  Stages st{};
  const RingGeom ga = ring_geom(H, 0, math_split(H).math), gb = ring_geom(I, M, 0);
  st.a = pick_stages(true, M, k, E, r, ga, limit);
  st.b = pick_stages(false, M, k, E, 0, gb, limit);
  if (st.a) st.smem_a = make_layout(true, M, k, E, r, ga, st.a).total;
  if (st.b) st.smem_b = make_layout(false, M, k, E, 0, gb, st.b).total;
  return st;
}

}  // namespace

std::string decode_unsupported_reason(int64_t M, int64_t E, int k, int64_t H, int64_t I) {
  if (M < 1 || M > kMaxM) return "the decode path takes 1 to " + std::to_string(kMaxM) + " tokens (M=" + std::to_string(M) + ")";
  if (k > 32) return "the decode path takes k <= 32 (k=" + std::to_string(k) + ")";
  if (E > 512) return "the decode path takes at most 512 experts (E=" + std::to_string(E) + ")";
  if (H > 128 * kMath * kMaxKBW)
    return "the decode path takes H <= " + std::to_string(128 * kMath * kMaxKBW) + " (H=" + std::to_string(H) + ")";
  DeviceInfo di;
  if (device_info(&di) != cudaSuccess) return "device query failed";
  const size_t lim = di.smem_optin - 1024;  // leave room for the kernels' static shared memory
  const Stages st = plan_stages(static_cast<int>(M), k, static_cast<int>(E), static_cast<int>(H),
                                static_cast<int>(I), 16, lim);
  if (st.a < kMinStages || st.b < kMinStages)
    return "the decode kernels' shared-memory rings do not fit this shape";
  return "";
}

bool decode_supported(int64_t M, int64_t E, int k, int64_t H, int64_t I) {
  return decode_unsupported_reason(M, E, k, H, I).empty();
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
  p.quant = w->quant_type;
  p.lora_A = r ? w->lora_A : nullptr;
  p.lora_B = r ? w->lora_B : nullptr;
  p.r = r;
  p.lora_scale = r ? w->lora_alpha / static_cast<float>(r) : 0.f;
  p.h = reinterpret_cast<uint16_t*>(static_cast<char*>(a.workspace) + ws.h);
  p.err = static_cast<int*>(a.workspace);
  p.out = a.out;
  const Stages st = plan_stages(p.M, p.k, p.E, p.H, p.I, r, di.smem_optin - 1024);
  if (st.a < kMinStages || st.b < kMinStages) return cudaErrorInvalidConfiguration;
  p.stages_a = st.a;
  p.stages_b = st.b;
  const MathSplit ms = math_split(p.H);
  if (ms.kbw == 1) return launch_pair<1, kMath>(p, di.sm_count, st.smem_a, st.smem_b, stream);
  if (ms.math == 12) return launch_pair<2, 12>(p, di.sm_count, st.smem_a, st.smem_b, stream);
  return launch_pair<2, kMath>(p, di.sm_count, st.smem_a, st.smem_b, stream);
}

}  // namespace e4b
