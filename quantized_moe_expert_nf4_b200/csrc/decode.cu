// Fused small-M (decode) forward of the NF4 expert layer: two kernels, no host sync.
//
// The pages' inference fast path for single-token decode is a fused 4-bit GEMV
// over the routed experts (experts4bit-qlora 0.22.0, "Inference: serve the
// fine-tune you just made"), and decode is launch-bound at ~89 launches per
// layer step ("CUDA-graph decode capture").  Here the whole layer is two
// kernels chained with programmatic dependent launch:
//
//   kernel A  routing (every CTA, redundantly: M <= 8 tokens), then for every
//             touched expert and block of 8 output columns, the gate and up
//             rows (8 + 8 weight rows, all of K = H) -> SiLU(gate) * up -> h
//             (bf16, [M*k, I], slot order); also prefetches the down rows of
//             the touched experts into L2 so HBM never idles between kernels.
//   kernel B  routing again, then for every block of 16 output rows of H, the
//             down rows of every touched expert in ascending expert order,
//             accumulated with the routing weights folded in -> out (bf16).
//             The sum over a token's experts happens inside one CTA in a fixed
//             order, so the result is deterministic.
//
// Only the experts that some token selected are read.  Weight rows stream
// through a shared-memory ring filled by 1-D bulk copies (TMA engine) from one
// producer thread; 16 consumer warps split K, decode nibbles through a
// per-lane-replicated byte -> bf16x2 codebook table (conflict-free) into
// mma.sync m16n8k16 fragments (weight rows = M dimension, tokens = the 8
// columns), and fold each 64-block's absmax into the fp32 accumulator once.
#include <algorithm>

#include "async.cuh"
#include "common.cuh"
#include "e4b_internal.h"
#include "topk.cuh"

namespace e4b {
namespace {

constexpr int kMaxM = 8;
constexpr int kCW = 16;                   // consumer warps
constexpr int kThreads = (kCW + 1) * 32;  // + one producer warp
constexpr uint32_t kRingBytes = 96 * 1024;
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
  int* err;
};

// Stage geometry for 16 weight rows of length K (bytes, with bank padding).
struct StageGeom {
  uint32_t row_stride;    // packed row stride in smem (bytes)
  uint32_t am_stride;     // absmax row stride in smem (floats)
  bool per_row_absmax;    // absmax copied row by row (padded) or 8 rows at a time
  uint32_t packed_bytes;  // 16 * row_stride
  uint32_t bytes;         // whole stage (packed + absmax), multiple of 128
  uint32_t tx_bytes;      // bytes the bulk copies deliver
};

__host__ __device__ inline StageGeom stage_geom(int K) {
  StageGeom g;
  const uint32_t rb = static_cast<uint32_t>(K / 2);
  // row stride = 32 (mod 128): the 8 rows a warp reads at once fall in distinct banks
  g.row_stride = rb + ((32u - (rb % 128u)) + 128u) % 128u;
  const uint32_t kb = static_cast<uint32_t>(K / 64);
  if (kb % 4 == 0) {
    g.per_row_absmax = true;
    g.am_stride = kb + (((kb / 4) % 2 == 0) ? 4u : 8u);  // 4 * odd words: distinct banks
  } else {
    g.per_row_absmax = false;  // kb odd or 2 mod 4: unpadded rows are conflict-free
    g.am_stride = kb;
  }
  g.packed_bytes = 16 * g.row_stride;
  const uint32_t am_bytes = 16 * g.am_stride * 4;
  g.bytes = (g.packed_bytes + am_bytes + 127u) / 128u * 128u;
  g.tx_bytes = 16 * rb + 16 * kb * 4;
  return g;
}

struct Layout {
  uint32_t ring, bars, lut, xs, red, ids, w, uidx, touched, slotmap, xa, total;
  int stages;
  StageGeom geom;
};

__host__ __device__ inline uint32_t al(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Shared-memory carve of kernel A (gate_up) or B (down).
__host__ __device__ inline Layout make_layout(bool is_a, int M, int k, int E, int H, int I, int r) {
  Layout L;
  L.geom = stage_geom(is_a ? H : I);
  int st = static_cast<int>(kRingBytes / L.geom.bytes);
  L.stages = st < 2 ? 2 : (st > 12 ? 12 : st);
  uint32_t o = 0;
  L.ring = o;
  o = al(o + L.stages * L.geom.bytes, 128);
  L.bars = o;
  o = al(o + 2 * L.stages * 8, 16);
  L.lut = o;
  o = al(o + 256 * 32 * 4, 16);
  L.xs = o;
  if (is_a) o = al(o + M * (2 * H + 16), 16);
  L.red = o;
  o = al(o + 2 * kCW * 32 * 16, 16);
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

// One 64-block of a 16-row stage: rows g (A rows 0..7) and g+8, thread t owns
// physical k in [16t, 16t+16) = 8 byte pairs; MMA j takes pairs 2j and 2j+1.
__device__ __forceinline__ void block_mma(const uint32_t* __restrict__ lut_lane, uint2 r0, uint2 r1, uint4 x0, uint4 x1,
                                          float tmp[4]) {
  auto L = [&](uint32_t word, int byte) { return lut_lane[((word >> (8 * byte)) & 0xffu) << 5]; };
  tmp[0] = tmp[1] = tmp[2] = tmp[3] = 0.0f;
  mma_16816(tmp, L(r0.x, 0), L(r1.x, 0), L(r0.x, 1), L(r1.x, 1), x0.x, x0.y);
  mma_16816(tmp, L(r0.x, 2), L(r1.x, 2), L(r0.x, 3), L(r1.x, 3), x0.z, x0.w);
  mma_16816(tmp, L(r0.y, 0), L(r1.y, 0), L(r0.y, 1), L(r1.y, 1), x1.x, x1.y);
  mma_16816(tmp, L(r0.y, 2), L(r1.y, 2), L(r0.y, 3), L(r1.y, 3), x1.z, x1.w);
}

// Routing of all M tokens into shared memory (every CTA does it; M <= 8).
// Builds: ids/w per slot, the touched experts in ascending id order, and
// slotmap[u][t] = slot of token t in expert touched[u] (or -1).
template <int MAXJ>
__device__ void decode_route(const DecodeParams& p, int* ids_s, float* w_s, int* uidx, int* touched, int* slotmap,
                             int* nU_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.M * p.k;
  for (int e = tid; e < p.E; e += blockDim.x) uidx[e] = -1;
  if (warp < p.M) route_token<MAXJ>(p.logits, warp, p.E, p.k, p.renorm != 0, ids_s, w_s);
  __syncthreads();
  for (int s = tid; s < S; s += blockDim.x) uidx[ids_s[s]] = 0;  // flag
  __syncthreads();
  if (warp == 0) {
    int count = 0;
    for (int base = 0; base < p.E; base += 32) {
      const int e = base + lane;
      const bool f = (e < p.E) && uidx[e] == 0;
      const uint32_t b = __ballot_sync(0xffffffffu, f);
      if (f) {
        const int u = count + __popc(b & lanemask_lt());
        touched[u] = e;
        uidx[e] = u;
      }
      count += __popc(b);
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

__device__ __forceinline__ void fill_lut(uint32_t* lut) {
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
    const int b = i >> 5;
    lut[i] = pack_bf16x2(kNf4CodebookDev[b >> 4], kNf4CodebookDev[b & 15]);
  }
}

// Producer: issue the bulk copies of one 16-row stage (rows row0[0..7], row1[0..7]
// as two runs of 8 consecutive rows) into `dst`.
__device__ __forceinline__ void issue_stage(const StageGeom& g, unsigned char* dst, uint64_t* full, const uint8_t* packed,
                                            const float* absmax, int K, int64_t run0, int64_t run1) {
  const uint32_t rb = K / 2, kb = K / 64;
  mbar_arrive_expect_tx(full, g.tx_bytes);
  const int64_t runs[2] = {run0, run1};
  float* am = reinterpret_cast<float*>(dst + g.packed_bytes);
  for (int h = 0; h < 2; ++h) {
    const int64_t r0 = runs[h];
    if (g.row_stride == rb) {
      bulk_g2s(dst + h * 8 * g.row_stride, packed + r0 * rb, 8 * rb, full);
    } else {
      for (int i = 0; i < 8; ++i) bulk_g2s(dst + (h * 8 + i) * g.row_stride, packed + (r0 + i) * rb, rb, full);
    }
    if (g.per_row_absmax) {
      for (int i = 0; i < 8; ++i) bulk_g2s(am + (h * 8 + i) * g.am_stride, absmax + (r0 + i) * kb, kb * 4, full);
    } else {
      bulk_g2s(am + h * 8 * g.am_stride, absmax + r0 * kb, 8 * kb * 4, full);
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel A: gate_up + SwiGLU (+ LoRA delta) -> h
template <int MAXJ>
__global__ void __launch_bounds__(kThreads, 1) decode_gate_up_kernel(DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const Layout L = make_layout(true, p.M, p.k, p.E, p.H, p.I, p.r);
  const StageGeom& G = L.geom;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + L.stages;
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
  const int H = p.H, I = p.I;
  const int xstride = H + 8;  // bf16 elements (2H + 16 bytes)

  if (tid == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_mbar_init();
  }
  pdl_wait();               // inputs of this call are final
  if (blockIdx.x == 0 && tid == 0) *p.err = kErrNone;
  pdl_launch_dependents();  // the down kernel may launch and run its prologue
  fill_lut(lut);
  for (int i = tid; i < p.M * (H / 8); i += blockDim.x) {
    const int t = i / (H / 8), c = i % (H / 8);
    reinterpret_cast<uint4*>(xs + t * xstride)[c] = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(t) * H)[c];
  }
  decode_route<MAXJ>(p, ids_s, w_s, uidx, touched, slotmap, &nU_s);
  const int nU = nU_s;
  const int items_per_expert = I / 8;
  const int nitems = nU * items_per_expert;

  if (warp == kCW) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      int j = 0;
      for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++j) {
        const int s = j % L.stages;
        if (j >= L.stages && !mbar_wait(&empty[s], ((j / L.stages) - 1) & 1)) {
          record_error(p.err, kErrWaitEmpty);
          break;
        }
        const int u = it / items_per_expert, rb = it % items_per_expert;
        const int64_t e = touched[u];
        const int64_t gate0 = e * 2 * I + rb * 8, up0 = gate0 + I;
        issue_stage(G, smem + L.ring + s * G.bytes, &full[s], p.gu_packed, p.gu_absmax, H, gate0, up0);
      }
    } else {
      // Lanes 1..31: prefetch this CTA's share of the touched experts' down rows into L2.
      const uint64_t per_expert = static_cast<uint64_t>(H) * I / 2;
      const uint64_t per_expert_am = static_cast<uint64_t>(H) * (I / 64) * 4;
      const uint64_t chunks_pk = (per_expert + kPrefetchChunk - 1) / kPrefetchChunk;
      const uint64_t chunks_am = (per_expert_am + kPrefetchChunk - 1) / kPrefetchChunk;
      const uint64_t per_u = chunks_pk + chunks_am;
      uint64_t total = static_cast<uint64_t>(nU) * per_u;
      const uint64_t cap = kPrefetchLimit / kPrefetchChunk;
      if (total > cap) total = cap;
      for (uint64_t c = static_cast<uint64_t>(blockIdx.x) * 31 + (lane - 1); c < total;
           c += static_cast<uint64_t>(gridDim.x) * 31) {
        const uint64_t u = c / per_u, q = c % per_u;
        const int64_t e = touched[u];
        if (q < chunks_pk) {
          const uint64_t off = q * kPrefetchChunk;
          const uint64_t n = min(static_cast<uint64_t>(kPrefetchChunk), per_expert - off);
          prefetch_l2(p.dn_packed + e * per_expert + off, static_cast<uint32_t>(n));
        } else {
          const uint64_t off = (q - chunks_pk) * kPrefetchChunk;
          const uint64_t n = min(static_cast<uint64_t>(kPrefetchChunk), per_expert_am - off);
          prefetch_l2(reinterpret_cast<const unsigned char*>(p.dn_absmax) + e * per_expert_am + off,
                      static_cast<uint32_t>(n));
        }
      }
    }
    return;
  }

  // ---------------- consumer warps ----------------
  const int g = lane >> 2, t = lane & 3;
  const int S = p.M * p.k;
  if (p.r > 0) {
    // LoRA first factor per slot: xa[s, rho] = x[token(s)] . lora_A[e(s), rho]
    for (int q = warp; q < S * p.r; q += kCW) {
      const int s = q / p.r, rho = q % p.r;
      const int tok = s / p.k;
      const uint16_t* la = p.lora_A + (static_cast<int64_t>(ids_s[s]) * p.r + rho) * H;
      float acc = 0.f;
      for (int kk = lane; kk < H; kk += 32)
        acc = fmaf(bf16_bits_to_float(xs[tok * xstride + kk]), bf16_bits_to_float(la[kk]), acc);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) xa[q] = acc;
    }
    named_barrier(1, kCW * 32);
  }
  const uint32_t* lut_lane = lut + lane;
  const int KB = H / 64;
  int j = 0;
  for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++j) {
    const int s = j % L.stages;
    const int u = it / items_per_expert, rb = it % items_per_expert;
    const int slot_g = (g < p.M) ? slotmap[u * kMaxM + g] : -1;
    const uint16_t* xrow = xs + g * xstride + 16 * t;
    if (!mbar_wait(&full[s], (j / L.stages) & 1)) {
      record_error(p.err, kErrWaitFull);
      break;
    }
    const unsigned char* st = smem + L.ring + s * G.bytes;
    const float* am = reinterpret_cast<const float*>(st + G.packed_bytes);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int kb = warp; kb < KB; kb += kCW) {
      const uint2 r0 = *reinterpret_cast<const uint2*>(st + g * G.row_stride + kb * 32 + 8 * t);
      const uint2 r1 = *reinterpret_cast<const uint2*>(st + (g + 8) * G.row_stride + kb * 32 + 8 * t);
      const float a0 = am[g * G.am_stride + kb], a1 = am[(g + 8) * G.am_stride + kb];
      uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
      if (slot_g >= 0) {
        x0 = *reinterpret_cast<const uint4*>(xrow + kb * 64);
        x1 = *reinterpret_cast<const uint4*>(xrow + kb * 64 + 8);
      }
      float tmp[4];
      block_mma(lut_lane, r0, r1, x0, x1, tmp);
      acc[0] = fmaf(tmp[0], a0, acc[0]);
      acc[1] = fmaf(tmp[1], a0, acc[1]);
      acc[2] = fmaf(tmp[2], a1, acc[2]);
      acc[3] = fmaf(tmp[3], a1, acc[3]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    red[((j & 1) * kCW + warp) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    named_barrier(1, kCW * 32);
    if (warp == 0) {
      float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < kCW; ++w) {
        const float4 v = red[((j & 1) * kCW + w) * 32 + lane];
        c.x += v.x;
        c.y += v.y;
        c.z += v.z;
        c.w += v.w;
      }
      const int e = touched[u];
      const int col = rb * 8 + g;  // h column == gate row index
      const float gate_v[2] = {c.x, c.y}, up_v[2] = {c.z, c.w};
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int tok = 2 * t + q;
        if (tok >= p.M) continue;
        const int slot = slotmap[u * kMaxM + tok];
        if (slot < 0) continue;
        float gv = gate_v[q], uv = up_v[q];
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
  }
}

// ---------------------------------------------------------------------------
// Kernel B: down rows of every touched expert, weighted combine -> out
template <int MAXJ>
__global__ void __launch_bounds__(kThreads, 1) decode_down_kernel(DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const Layout L = make_layout(false, p.M, p.k, p.E, p.H, p.I, 0);
  const StageGeom& G = L.geom;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + L.stages;
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
  float4* red = reinterpret_cast<float4*>(smem + L.red);
  int* ids_s = reinterpret_cast<int*>(smem + L.ids);
  float* w_s = reinterpret_cast<float*>(smem + L.w);
  int* uidx = reinterpret_cast<int*>(smem + L.uidx);
  int* touched = reinterpret_cast<int*>(smem + L.touched);
  int* slotmap = reinterpret_cast<int*>(smem + L.slotmap);
  __shared__ int nU_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, I = p.I;
  if (tid == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_mbar_init();
  }
  // The prologue only reads inputs the gate_up kernel does not write.
  fill_lut(lut);
  decode_route<MAXJ>(p, ids_s, w_s, uidx, touched, slotmap, &nU_s);
  const int nU = nU_s;
  const int nrb = H / 16;

  if (warp == kCW) {
    if (lane == 0) {
      // Weights do not depend on the gate_up kernel: start streaming at once.
      int j = 0;
      for (int rb = blockIdx.x; rb < nrb; rb += gridDim.x) {
        bool ok = true;
        for (int u = 0; u < nU; ++u, ++j) {
          const int s = j % L.stages;
          if (j >= L.stages && !mbar_wait(&empty[s], ((j / L.stages) - 1) & 1)) {
            record_error(p.err, kErrWaitEmpty);
            ok = false;
            break;
          }
          const int64_t row0 = static_cast<int64_t>(touched[u]) * H + rb * 16;
          issue_stage(G, smem + L.ring + s * G.bytes, &full[s], p.dn_packed, p.dn_absmax, I, row0, row0 + 8);
        }
        if (!ok) break;
      }
    }
    return;
  }

  pdl_wait();  // h written by the gate_up kernel is visible from here on
  const int g = lane >> 2, t = lane & 3;
  const uint32_t* lut_lane = lut + lane;
  const int KB = I / 64;
  int j = 0, item = 0;
  bool ok = true;
  for (int rb = blockIdx.x; rb < nrb && ok; rb += gridDim.x, ++item) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int u = 0; u < nU; ++u, ++j) {
      const int s = j % L.stages;
      // token columns g (B operand) and 2t, 2t+1 (accumulator columns)
      const int slot_g = (g < p.M) ? slotmap[u * kMaxM + g] : -1;
      const int sc0 = (2 * t < p.M) ? slotmap[u * kMaxM + 2 * t] : -1;
      const int sc1 = (2 * t + 1 < p.M) ? slotmap[u * kMaxM + 2 * t + 1] : -1;
      const float wc0 = sc0 >= 0 ? w_s[sc0] : 0.f, wc1 = sc1 >= 0 ? w_s[sc1] : 0.f;
      const uint16_t* hrow = p.h + static_cast<int64_t>(slot_g < 0 ? 0 : slot_g) * I + 16 * t;
      // Issue the h loads of this stage before waiting for its weights.
      uint4 hx[2][2];
      int nkb = 0;
      for (int kb = warp; kb < KB && nkb < 2; kb += kCW, ++nkb) {
        hx[nkb][0] = hx[nkb][1] = make_uint4(0, 0, 0, 0);
        if (slot_g >= 0) {
          hx[nkb][0] = *reinterpret_cast<const uint4*>(hrow + kb * 64);
          hx[nkb][1] = *reinterpret_cast<const uint4*>(hrow + kb * 64 + 8);
        }
      }
      if (!mbar_wait(&full[s], (j / L.stages) & 1)) {
        record_error(p.err, kErrWaitFull);
        ok = false;
        break;
      }
      const unsigned char* st = smem + L.ring + s * G.bytes;
      const float* am = reinterpret_cast<const float*>(st + G.packed_bytes);
      int q = 0;
      for (int kb = warp; kb < KB; kb += kCW, ++q) {
        uint4 x0, x1;
        if (q < 2) {
          x0 = hx[q][0];
          x1 = hx[q][1];
        } else {
          x0 = x1 = make_uint4(0, 0, 0, 0);
          if (slot_g >= 0) {
            x0 = *reinterpret_cast<const uint4*>(hrow + kb * 64);
            x1 = *reinterpret_cast<const uint4*>(hrow + kb * 64 + 8);
          }
        }
        const uint2 r0 = *reinterpret_cast<const uint2*>(st + g * G.row_stride + kb * 32 + 8 * t);
        const uint2 r1 = *reinterpret_cast<const uint2*>(st + (g + 8) * G.row_stride + kb * 32 + 8 * t);
        const float a0 = am[g * G.am_stride + kb], a1 = am[(g + 8) * G.am_stride + kb];
        float tmp[4];
        block_mma(lut_lane, r0, r1, x0, x1, tmp);
        acc[0] = fmaf(tmp[0], a0 * wc0, acc[0]);
        acc[1] = fmaf(tmp[1], a0 * wc1, acc[1]);
        acc[2] = fmaf(tmp[2], a1 * wc0, acc[2]);
        acc[3] = fmaf(tmp[3], a1 * wc1, acc[3]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (!ok) break;
    red[((item & 1) * kCW + warp) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    named_barrier(1, kCW * 32);
    if (warp == 0) {
      float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < kCW; ++w) {
        const float4 v = red[((item & 1) * kCW + w) * 32 + lane];
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
  }
}

template <int MAXJ>
cudaError_t launch_pair(const DecodeParams& p, int sm_count, size_t smem_a, size_t smem_b, cudaStream_t stream) {
  // The dynamic shared-memory limit is a per-function attribute: raise it to
  // what this call needs (kept per instantiation; raising is idempotent).
  static size_t configured_a = 0, configured_b = 0;
  if (smem_a > configured_a) {
    cudaError_t e1 = cudaFuncSetAttribute(decode_gate_up_kernel<MAXJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(smem_a));
    if (e1 != cudaSuccess) return e1;
    configured_a = smem_a;
  }
  if (smem_b > configured_b) {
    cudaError_t e1 = cudaFuncSetAttribute(decode_down_kernel<MAXJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(smem_b));
    if (e1 != cudaSuccess) return e1;
    configured_b = smem_b;
  }
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
    cudaError_t err = cudaLaunchKernelEx(&cfg, decode_gate_up_kernel<MAXJ>, p);
    if (err != cudaSuccess) return err;
  }
  cfg.gridDim = dim3(std::max(1, std::min(sm_count, p.H / 16)));
  cfg.dynamicSmemBytes = smem_b;
  LaunchScope ls("decode.down", stream);
  return cudaLaunchKernelEx(&cfg, decode_down_kernel<MAXJ>, p);
}

struct DecodeWs {
  size_t h, err, total;
};

DecodeWs decode_ws(int64_t M, int k, int64_t I) {
  DecodeWs w;
  w.h = 0;
  w.err = align_up(static_cast<size_t>(M * k * I * 2), 256);
  w.total = w.err + 256;
  return w;
}

}  // namespace

bool decode_supported(int64_t M, int64_t E, int k, int64_t H, int64_t I) {
  if (M < 1 || M > kMaxM || k > 32 || E > 512) return false;
  DeviceInfo di;
  if (device_info(&di) != cudaSuccess) return false;
  const Layout a = make_layout(true, static_cast<int>(M), k, static_cast<int>(E), static_cast<int>(H),
                               static_cast<int>(I), 16);
  const Layout b = make_layout(false, static_cast<int>(M), k, static_cast<int>(E), static_cast<int>(H),
                               static_cast<int>(I), 0);
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
  p.out = a.out;
  p.err = reinterpret_cast<int*>(static_cast<char*>(a.workspace) + ws.err);
  const size_t smem_a = make_layout(true, p.M, p.k, p.E, p.H, p.I, r).total;
  const size_t smem_b = make_layout(false, p.M, p.k, p.E, p.H, p.I, 0).total;
  if (p.E <= 32) return launch_pair<1>(p, di.sm_count, smem_a, smem_b, stream);
  if (p.E <= 64) return launch_pair<2>(p, di.sm_count, smem_a, smem_b, stream);
  if (p.E <= 128) return launch_pair<4>(p, di.sm_count, smem_a, smem_b, stream);
  if (p.E <= 256) return launch_pair<8>(p, di.sm_count, smem_a, smem_b, stream);
  return launch_pair<16>(p, di.sm_count, smem_a, smem_b, stream);  // E <= 512 (decode_supported)
}

}  // namespace e4b
