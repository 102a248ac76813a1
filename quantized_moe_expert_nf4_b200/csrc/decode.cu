// Fused small-M (decode) forward of the NF4 expert layer: one kernel, no host sync.
//
// The pages' inference fast path for single-token decode is a fused 4-bit GEMV
// over the routed experts (experts4bit-qlora 0.22.0, "Inference: serve the
// fine-tune you just made"), and decode is launch-bound at ~89 launches per
// layer step ("CUDA-graph decode capture").  Here the whole layer is ONE
// cooperative launch of one CTA per SM:
//
//   prologue  every CTA routes the M <= 8 tokens (top-k + weights) and lists
//             the touched experts (ascending id); only those are read.
//   phase 1   gate_up: the CTA's contiguous run of items (16 gate + 16 up rows
//             of one touched expert over all of K = H) -> SiLU(gate) * up
//             (+ LoRA delta) -> h (bf16, [M*k, I], slot order) in the workspace.
//   barrier   grid-wide: every CTA's h is written.
//   phase 2   down: for each block of 16 output rows the CTA owns, the down
//             rows of every touched expert times h, the routing weights
//             folded in per token column -> out (bf16).  The combine over the
//             experts of a token happens inside the CTA in a fixed order, so
//             the result is deterministic and needs no extra kernel.
//
// One producer warp streams the packed rows and their fp32 absmax with bulk
// asynchronous copies (mbarrier transaction counts) through a ring of
// shared-memory stages: first phase 1's items, then -- without waiting for the
// barrier, since weights do not depend on h -- phase 2's stages, so HBM keeps
// streaming the down rows while phase 1 computes and the barrier resolves.
// A copy engine pays a fixed cost per copy (measured on B200: 1 KB copies
// stream at about half the rate of 4 KB ones), so rows travel four at a time:
// a block of 16 rows is four copies of 4 consecutive rows, each copy 32 bytes
// (mod 128) past the previous one.  MMA row g (and g + 8) reads row
// 4 (g % 4) + g / 4 (+ 2) of its block, so the four rows a half-warp's
// fragment loads touch lie in four different copies, on four different bank
// groups.  Sixteen math warps decode and multiply: nibbles become bf16 pairs
// through a per-lane replicated byte -> bf16x2 codebook table (lane l reads
// only bank l; one byte permute forms a lookup's address) and feed mma.sync
// m16n8k16 with the weight rows as MMA rows and the <= 8 tokens as the 8 MMA
// columns.  Each MMA stays inside one 64-element absmax block, so the block's
// fp32 absmax scales the products (no rounding of the scale).
//
// The grid barrier needs no initialised workspace: a 64-bit epoch word sits
// beside one slot per CTA.  Every CTA reads the epoch e at its start, publishes
// e + 1 in its own slot once its h is written, and waits until every slot
// holds e + 1; CTA 0 then stores e + 1 as the new epoch (every CTA read e
// before it published, so none reads the new value in this launch).  Stale
// slots of earlier calls hold smaller tags and garbage matches a 64-bit tag
// only by chance, so a fresh workspace works, as does one the grouped path
// wrote in between, and graph replays (which repeat the grid launch's own
// identifiers) still get a new tag each time.  Every wait is bounded; a wait that
// gives up records an error code in the workspace's error word, marks the CTA
// aborted (later waits return at once, the results are unspecified) and the
// kernel still runs to its end.
#include <algorithm>
#include <string>

#include "async.cuh"
#include "common.cuh"
#include "e4b_internal.h"
#include "topk.cuh"

namespace e4b {
namespace {

constexpr int kMaxM = 8;
constexpr int kMath = 16;               // math warps
constexpr int kProducer = kMath;        // warp issuing the bulk copies
constexpr int kWarps = kMath + 1;
constexpr int kThreads = kWarps * 32;
constexpr int kGroups = 2;              // phase 1: items alternate between two groups of math warps
constexpr int kGW = kMath / kGroups;    // warps per group
constexpr int kMaxSPW = 4;              // spans (128 k) per warp of an item: H <= 8 * 4 * 128 = 4096
constexpr int kMaxPPW = 3;              // (expert, k-block) pairs per warp of a down stage
constexpr int kMaxDPE = 4;              // down experts per stage (8 copies each: one producer lane per copy)
constexpr int kMaxKBI = kMath * kMaxPPW;  // k-blocks of a down row: I <= 3072
constexpr int kMaxGrid = 1024;          // barrier slots in the workspace
constexpr int kMaxStages = 32;
// Byte -> bf16x2 table: entry b for lane l at byte 256 b + 4 l, so one byte
// permute of the packed word and 4 l forms the address.  The upper 128 bytes of
// every entry hold the partial sums of both phases (red_offset).
constexpr uint32_t kLutBytes = 256 * 256;
constexpr uint32_t kRedBytes = kGroups * 2 * kGW * 2 * 32 * 16;  // phase 1: [group][parity][warp][tile][lane] float4
static_assert(kRedBytes <= 256 * 128, "the partial sums fit the table's upper halves");
constexpr int kBarMath = 3;             // named barrier of the 16 math warps

struct FusedParams {
  const uint16_t* x;
  const float* logits;
  int M, k, E, H, I;
  int renorm;
  const uint8_t* gu_packed;
  const float* gu_absmax;
  const uint8_t* dn_packed;
  const float* dn_absmax;
  int quant;                   // e4b_quant_type of both stacks (the table the decoders build)
  const uint16_t* lora_A;
  const uint16_t* lora_B;
  int r;
  float lora_scale;
  uint16_t* h;                 // [S, I] bf16 (slot order)
  uint16_t* out;               // [M, H] bf16
  int* err;                    // error word
  unsigned long long* flags;   // [kMaxGrid] barrier slots, then the epoch word
  int stages;                  // ring depth (even)
  int dpe;                     // down experts per phase-2 stage
};

__host__ __device__ inline uint32_t al(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// A staged block of 16 rows of K elements: packed copy c (rows 4c .. 4c+3,
// dense, K/2 bytes apart) at c * copy_stride(K) = c * (2K + 32) bytes, which is
// 32 mod 128, then the absmax copies (4 rows x KB floats each) at
// am_stride(KB) = 16 KB + pad bytes, 16 mod 128.  A gate_up stage holds two
// such blocks side by side (gate copies 0-3, up copies 4-7, then their
// absmax copies 0-7); a down stage holds one block per expert.
__host__ __device__ inline uint32_t copy_stride(int K) { return static_cast<uint32_t>(2 * K + 32); }
__host__ __device__ inline uint32_t am_stride(int KB) {
  const uint32_t b = static_cast<uint32_t>(16 * KB);
  return b + (144u - b % 128u) % 128u;
}
__host__ __device__ inline uint32_t gu_stage_bytes(int H) { return 8 * copy_stride(H) + 8 * am_stride(H / 64); }
__host__ __device__ inline uint32_t dn_block_bytes(int I) { return 4 * copy_stride(I) + 4 * am_stride(I / 64); }

// Float4 slot i of the partial sums (phase 1: [group][parity][warp][tile][lane];
// phase 2: [warp][lane]) in the upper half of table entry i / 8: a quarter
// warp's float4 accesses fill one 128-byte row.
__host__ __device__ inline uint32_t red_offset(int i) {
  return (static_cast<uint32_t>(i >> 3) << 8) + 128u + (static_cast<uint32_t>(i & 7) << 4);
}

struct Smem {
  uint32_t lut, ids, w, uidx, touched, slotmap, xa, bars, ring, total;
};

__host__ __device__ inline Smem make_smem(int M, int k, int E, int r, int I, int stages, uint32_t slot) {
  Smem L;
  const int S = M * k;
  uint32_t o = 0;
  L.lut = o;
  o += kLutBytes;
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
  if (r > 0) o = al(o + S * r * 4, 16);
  L.bars = o;
  o = al(o + (2 * stages + 2 * kGroups) * 8, 16);
  L.ring = al(o, 128);
  L.total = L.ring + static_cast<uint32_t>(stages) * slot;
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

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}


// L2 policy for data read exactly once per call (the packed weights): evict it
// first, so the stream does not push out what the kernel reads again (its h,
// barrier slots, x, and its own instructions).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Bulk asynchronous copy global -> this CTA's shared memory, completing on `bar`
// (both addresses 16-byte aligned, bytes a multiple of 16), with an L2 policy.
__device__ __forceinline__ void bulk_g2s_stream(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar,
                                                uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ uint2 lds64(const unsigned char* p) { return *reinterpret_cast<const uint2*>(p); }

__device__ __forceinline__ void st_release_gpu(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_gpu(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}


// Bounded wait on a ring barrier.  Once any wait of the CTA has given up
// (*abort set), every later wait returns false at once.
__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* err, int code) {
  if (mbar_try_wait(bar, parity)) return true;
  unsigned long long t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (*abort) return false;
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if ((it & 63u) == 0) {  // the clock only now and then: see mbar_wait
      const unsigned long long now = global_ns();
      if (it == 0) {
        t0 = now;
      } else if (now - t0 > kWaitLimitNs) {
        *abort = 1;
        record_error(err, code);
        return false;
      }
    }
  }
}

// The four MMAs of one 64-element k-block of a 16-row tile, into d (zeroed by
// the caller).  Thread (g, t) holds packed bytes [8t, 8t+8) of the block for
// row g (w0) and row g+8 (w1) -- elements 16t .. 16t+15 -- and the matching 16
// bf16 of its token column g (xw, 8 words).  MMA j takes bytes 2j, 2j+1: their
// bf16 pairs are the A fragment (row g / g+8, k slots 2t..2t+1 and 2t+8..2t+9)
// and x words 2j, 2j+1 the B fragment, so both operands see the same physical
// k for every slot.  The table entry of byte b for lane l is at byte
// 256 b + 4 l of the table: one byte permute puts byte b of the packed word
// above lane4 = 4 l (byte 0), so a lookup costs one ALU op and one load.
__device__ __forceinline__ void block_mma(const unsigned char* __restrict__ lut, uint32_t lane4, uint2 w0, uint2 w1,
                                          const uint32_t* xw, float d[4]) {
  auto pair = [&](uint32_t word, int byte) {
    const uint32_t ad = __byte_perm(word, lane4, 0x5504u | (static_cast<uint32_t>(byte) << 4));
    return *reinterpret_cast<const uint32_t*>(lut + ad);
  };
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t wa = (j < 2) ? w0.x : w0.y, wb = (j < 2) ? w1.x : w1.y;
    const int b = 2 * (j & 1);
    mma_16816(d, pair(wa, b), pair(wb, b), pair(wa, b + 1), pair(wb, b + 1), xw[2 * j], xw[2 * j + 1]);
  }
}

// Two independent blocks (a and b) at once, their MMAs interleaved: each
// MMA of a chain waits for the previous one of the same chain, so two chains
// keep the tensor pipe busy where one would leave it idle.
__device__ __forceinline__ void block_mma2(const unsigned char* __restrict__ lut, uint32_t lane4, uint2 w0a,
                                           uint2 w1a, const uint32_t* xa, uint2 w0b, uint2 w1b, const uint32_t* xb,
                                           float da[4], float db[4]) {
  auto pair = [&](uint32_t word, int byte) {
    const uint32_t ad = __byte_perm(word, lane4, 0x5504u | (static_cast<uint32_t>(byte) << 4));
    return *reinterpret_cast<const uint32_t*>(lut + ad);
  };
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int b = 2 * (j & 1);
    const uint32_t wa0 = (j < 2) ? w0a.x : w0a.y, wa1 = (j < 2) ? w1a.x : w1a.y;
    const uint32_t wb0 = (j < 2) ? w0b.x : w0b.y, wb1 = (j < 2) ? w1b.x : w1b.y;
    const uint32_t a0 = pair(wa0, b), a1 = pair(wa1, b), a2 = pair(wa0, b + 1), a3 = pair(wa1, b + 1);
    const uint32_t b0 = pair(wb0, b), b1 = pair(wb1, b), b2 = pair(wb0, b + 1), b3 = pair(wb1, b + 1);
    mma_16816(da, a0, a1, a2, a3, xa[2 * j], xa[2 * j + 1]);
    mma_16816(db, b0, b1, b2, b3, xb[2 * j], xb[2 * j + 1]);
  }
}

// Top-k of token `t` by the calling warp, with the key array sized for E.
__device__ __forceinline__ void route_one(const FusedParams& p, int t, int* ids_s, float* w_s) {
  const int maxj = (p.E + 31) / 32;
  if (maxj <= 1) route_token<1>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
  else if (maxj <= 2) route_token<2>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
  else if (maxj <= 4) route_token<4>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
  else if (maxj <= 8) route_token<8>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
  else route_token<16>(p.logits, t, p.E, p.k, p.renorm != 0, ids_s, w_s);
}

// Prologue: warps < M route one token each while the other warps build the
// byte -> bf16x2 table of the stacks' codebook (NF4 or FP4) (entry b of lane l
// at word 64 b + l: low half the high nibble's value, i.e. element 2i, high
// half element 2i+1).  Then the
// touched experts (ascending id) and slotmap[u][t] = slot of token t in expert
// touched[u] (or -1).
__device__ void prologue(const FusedParams& p, uint32_t* lut, int* ids_s, float* w_s, int* uidx, int* touched,
                         int* slotmap, int* nU_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.M * p.k;
  for (int e = tid; e < p.E; e += blockDim.x) uidx[e] = -1;
  if (warp < p.M) {
    route_one(p, warp, ids_s, w_s);
  } else {
    const float cbl = codebook_entry(p.quant, lane & 15);
    for (int b = warp - p.M; b < 256; b += kWarps - p.M) {
      const float hi = __shfl_sync(0xffffffffu, cbl, b >> 4);
      const float lo = __shfl_sync(0xffffffffu, cbl, b & 15);
      lut[b * 64 + lane] = pack_bf16x2(hi, lo);
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

// Copy `lane_c` (0-3 packed, 4-7 absmax) of a block of 16 rows starting at
// global row `row0` of a packed matrix with K columns into the block at `dst`
// (packed copies at dst + c * copy_stride, absmax copies at am_dst + c * am_stride).
__device__ __forceinline__ void copy_block_part(int lane_c, unsigned char* dst, unsigned char* am_dst,
                                                uint64_t* full, const uint8_t* packed, const float* absmax, int K,
                                                int64_t row0, uint64_t pol) {
  const int KB = K / 64;
  const int c = lane_c & 3;
  const int64_t row = row0 + 4 * c;
  if (lane_c < 4)
    bulk_g2s_stream(dst + c * copy_stride(K), packed + row * (K / 2), static_cast<uint32_t>(2 * K), full, pol);
  else
    bulk_g2s_stream(am_dst + c * am_stride(KB), absmax + row * KB, static_cast<uint32_t>(16 * KB), full, pol);
}

// ---------------------------------------------------------------------------
// SPW: spans (two k-blocks) per math warp of a phase-1 item; PPW: (expert,
// k-block) pairs per math warp of a phase-2 stage.
template <int SPW, int PPW>
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(FusedParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int H = p.H, I = p.I, KB = H / 64, KBI = I / 64;
  const int RS = p.stages, DPE = p.dpe;
  const uint32_t cs_gu = copy_stride(H), as_gu = am_stride(KB) / 4, am_gu = 8 * cs_gu;
  const uint32_t cs_dn = copy_stride(I), as_dn = am_stride(KBI) / 4, am_dn = 4 * cs_dn;
  const uint32_t exp_dn = dn_block_bytes(I);
  const uint32_t slot = al(max(gu_stage_bytes(H), static_cast<uint32_t>(DPE) * exp_dn), 128);
  const Smem L = make_smem(p.M, p.k, p.E, p.r, p.I, RS, slot);
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
  unsigned char* lutb = smem + L.lut;
  auto red_at = [&](int i) { return reinterpret_cast<float4*>(lutb + red_offset(i)); };
  int* ids_s = reinterpret_cast<int*>(smem + L.ids);
  float* w_s = reinterpret_cast<float*>(smem + L.w);
  int* uidx = reinterpret_cast<int*>(smem + L.uidx);
  int* touched = reinterpret_cast<int*>(smem + L.touched);
  int* slotmap = reinterpret_cast<int*>(smem + L.slotmap);
  float* xa = reinterpret_cast<float*>(smem + L.xa);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);  // stage landed
  uint64_t* empty = full + RS;                                   // stage consumed (16 arrivals)
  uint64_t* rfree = empty + RS;                                  // [group][parity] partials read by the finisher
  unsigned char* ring = smem + L.ring;
  __shared__ int nU_s;
  __shared__ volatile int abort_s;
  __shared__ int fin_cnt[kGroups][2];  // warps of a group that have deposited an item's partials

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  // This launch's barrier tag: the workspace's epoch + 1 (read before this
  // CTA publishes anything; see the barrier below).
  const unsigned long long tag = (warp == 0) ? ld_relaxed_gpu(p.flags + kMaxGrid) + 1 : 0;
  if (tid == 0) {
    abort_s = 0;
    for (int s = 0; s < RS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kMath);
    }
    for (int i = 0; i < 2 * kGroups; ++i) {
      mbar_init(&rfree[i], 1);
      fin_cnt[i >> 1][i & 1] = 0;
    }
    fence_mbar_init();
  }
  prologue(p, lut, ids_s, w_s, uidx, touched, slotmap, &nU_s);
  const int nU = nU_s;
  const int G = static_cast<int>(gridDim.x), bid = static_cast<int>(blockIdx.x);

  // Phase-1 items: a contiguous run per CTA (consecutive items = consecutive rows).
  const int ipe = I / 16;
  const int nitems = nU * ipe;
  const int q_it = nitems / G, rem_it = nitems % G;
  const int i0 = bid * q_it + min(bid, rem_it);
  const int n_gu = q_it + (bid < rem_it ? 1 : 0);
  // Phase-2 stages: row blocks bid, bid + G, ...; per row block ceil(nU / DPE) stages.
  const int nrb_all = H / 16;
  const int nrb = bid < nrb_all ? (nrb_all - bid + G - 1) / G : 0;
  const int nch = (nU + DPE - 1) / DPE;
  const int n_dn = nrb * nch;
  const int T = n_gu + n_dn;

  if (warp == kProducer) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = l2_evict_first_policy();
    int issued = 0;
    // Ring slot s and its pass ph of stage j; item (u, rb) of stage j < n_gu;
    // chunk ch and row-block round rq of stage j >= n_gu -- all advanced per
    // stage instead of divided out.
    int s = 0, ph = 0, u = i0 / ipe, rb = i0 % ipe, ch = 0, rq = 0;
    for (int j = 0; j < T; ++j) {
      if (j >= RS && !ring_wait(&empty[s], ph ^ 1, &abort_s, p.err, kErrWaitEmpty)) break;
      unsigned char* st = ring + static_cast<uint32_t>(s) * slot;
      if (j < n_gu) {
        // 16 gate rows (block 0) and the matching 16 up rows (block 1): lanes
        // 0-3 / 8-11 the gate / up packed copies, 4-7 / 12-15 their absmax.
        const int64_t grow = static_cast<int64_t>(touched[u]) * 2 * I + rb * 16;
        if (lane == 0) mbar_arrive_expect_tx(&full[s], 32u * (H / 2) + 32u * KB * 4);
        __syncwarp();
        if (lane < 16) {
          const int blk = lane >> 3;
          copy_block_part(lane & 7, st + blk * 4 * cs_gu, st + am_gu + blk * 16 * as_gu, &full[s], p.gu_packed,
                          p.gu_absmax, H, grow + blk * I, pol);
        }
        if (++rb == ipe) {
          rb = 0;
          ++u;
        }
      } else {
        // One block of 16 down rows per expert: lane 8 ei + c issues copy c of expert ei.
        const int rbd = bid + rq * G;
        const int u0 = ch * DPE, ne = min(DPE, nU - u0);
        if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(ne) * (16u * (I / 2) + 16u * KBI * 4));
        __syncwarp();
        if (lane < 8 * ne) {
          const int ei = lane >> 3;
          const int64_t row0 = static_cast<int64_t>(touched[u0 + ei]) * H + rbd * 16;
          copy_block_part(lane & 7, st + ei * exp_dn, st + ei * exp_dn + am_dn, &full[s], p.dn_packed, p.dn_absmax, I,
                          row0, pol);
        }
        if (++ch == nch) {
          ch = 0;
          ++rq;
        }
      }
      ++issued;
      if (++s == RS) {
        s = 0;
        ph ^= 1;
      }
    }
    // Every copy in flight lands before the CTA may exit.
    for (int j = max(0, issued - RS); j < issued; ++j)
      if (!mbar_wait(&full[j % RS], (j / RS) & 1)) record_error(p.err, kErrWaitDrain);
    return;
  }

  // ---------------------------------------------------------------- math warps
  const unsigned char* lut_b = smem + L.lut;
  const uint32_t lane4 = static_cast<uint32_t>(lane) * 4;
  const int S = p.M * p.k;
  if (p.r > 0 && n_gu > 0) {
    // LoRA first factor of the slots whose expert has items in this CTA:
    // xa[s, rho] = x[token(s)] . lora_A[e(s), rho]
    const int u_lo = i0 / ipe, u_hi = (i0 + n_gu - 1) / ipe;
    for (int qd = warp; qd < S * p.r; qd += kMath) {
      const int s = qd / p.r, rho = qd % p.r;
      const int u = uidx[ids_s[s]];
      if (u < u_lo || u > u_hi) continue;
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
    named_bar(kBarMath, kMath * 32);
  }

  // -------------------------------------------------------------- phase 1
  {
    const int gi = warp / kGW, wi = warp % kGW;
    // The warp's k-blocks are the same in every item: its slice of x (token g
    // of the MMA column) stays in registers.  Columns of tokens that do not
    // route to an item's expert compute values that are never stored.
    uint32_t xr[SPW][2][8];
#pragma unroll
    for (int q = 0; q < SPW; ++q) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int kb = 2 * (wi + kGW * q) + hh;
        uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
        if (g < p.M && kb < KB) {
          const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(g) * H + kb * 64 + 16 * t);
          a = src[0];
          b = src[1];
        }
        xr[q][hh][0] = a.x; xr[q][hh][1] = a.y; xr[q][hh][2] = a.z; xr[q][hh][3] = a.w;
        xr[q][hh][4] = b.x; xr[q][hh][5] = b.y; xr[q][hh][6] = b.z; xr[q][hh][7] = b.w;
      }
    }
    // Ring slot s and pass ph of item jj (the ring depth is even, so a group's
    // items stay on slots of one parity of index).
    int s = gi, ph = 0;
    for (int jj = gi; jj < n_gu; jj += kGroups, s += kGroups) {
      if (s >= RS) {
        s -= RS;
        ph ^= 1;
      }
      ring_wait(&full[s], ph, &abort_s, p.err, kErrWaitFull);
      const unsigned char* st = ring + static_cast<uint32_t>(s) * slot;
      const float* am = reinterpret_cast<const float*>(st + am_gu);
      // Tile T: MMA row g = gate column 4 (g % 4) + 2T + g / 4 of the item
      // (copy g % 4 of the gate block, row 2T + g / 4 in it); row g + 8 = the
      // same column's up row (copy 4 + g % 4).
      float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int q = 0; q < SPW; ++q) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int kb = 2 * (wi + kGW * q) + hh;
          if (kb < KB) {
            uint2 w0[2], w1[2];
            float a0[2], a1[2];
#pragma unroll
            for (int T = 0; T < 2; ++T) {
              const int r = 2 * T + (g >> 2), cg = g & 3;
              const uint32_t off = r * (H / 2) + kb * 32 + 8 * t;
              w0[T] = lds64(st + cg * cs_gu + off);
              w1[T] = lds64(st + (4 + cg) * cs_gu + off);
              a0[T] = am[cg * as_gu + r * KB + kb];
              a1[T] = am[(4 + cg) * as_gu + r * KB + kb];
            }
            float d[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            block_mma2(lut_b, lane4, w0[0], w1[0], xr[q][hh], w0[1], w1[1], xr[q][hh], d[0], d[1]);
#pragma unroll
            for (int T = 0; T < 2; ++T) {
              c[T][0] = fmaf(a0[T], d[T][0], c[T][0]);
              c[T][1] = fmaf(a0[T], d[T][1], c[T][1]);
              c[T][2] = fmaf(a1[T], d[T][2], c[T][2]);
              c[T][3] = fmaf(a1[T], d[T][3], c[T][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cnt(&empty[s], kMath / kGW);
      // Deposit the partials; the last warp of the group to do so finishes
      // the item while the others go on to their next one.  Items iq and
      // iq + 2 of the group share a buffer: wait until the finisher of iq - 2
      // has read it.
      const int iq = jj / kGroups, par = iq & 1;
      if (iq >= 2) ring_wait(&rfree[gi * 2 + par], ((iq >> 1) - 1) & 1, &abort_s, p.err, kErrWaitFull);
      const int ri = (((gi * 2 + par) * kGW + wi) * 2) * 32 + lane;
      *red_at(ri) = make_float4(c[0][0], c[0][1], c[0][2], c[0][3]);
      *red_at(ri + 32) = make_float4(c[1][0], c[1][1], c[1][2], c[1][3]);
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        __threadfence_block();
        last = atomicAdd(&fin_cnt[gi][par], 1) == kGW - 1;
      }
      if (__shfl_sync(0xffffffffu, last, 0)) {
        __threadfence_block();  // the other warps' partials, deposited before their increments
        // This warp finishes the item: the group's partials in warp order,
        // then SwiGLU (+ LoRA delta) for the tokens routed to the expert.
        const int it = i0 + jj, u = it / ipe, rb = it % ipe;
        const int e = touched[u];
#pragma unroll
        for (int T = 0; T < 2; ++T) {
          float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int w = 0; w < kGW; ++w) {
            const float4 v = *red_at((((gi * 2 + par) * kGW + w) * 2 + T) * 32 + lane);
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
          }
          const int col = rb * 16 + 4 * (g & 3) + 2 * T + (g >> 2);  // h column == gate row index
          const float gate_v[2] = {sum.x, sum.y}, up_v[2] = {sum.z, sum.w};
#pragma unroll
          for (int qq = 0; qq < 2; ++qq) {
            const int tok = 2 * t + qq;
            if (tok >= p.M) continue;
            const int sl = slotmap[u * kMaxM + tok];
            if (sl < 0) continue;
            float gv = gate_v[qq], uv = up_v[qq];
            if (p.r > 0) {
              const uint16_t* bg = p.lora_B + (static_cast<int64_t>(e) * 2 * I + col) * p.r;
              const uint16_t* bu = p.lora_B + (static_cast<int64_t>(e) * 2 * I + I + col) * p.r;
              float dg = 0.f, du = 0.f;
              for (int rho = 0; rho < p.r; ++rho) {
                const float xv = xa[sl * p.r + rho];
                dg = fmaf(xv, bf16_bits_to_float(bg[rho]), dg);
                du = fmaf(xv, bf16_bits_to_float(bu[rho]), du);
              }
              gv = fmaf(p.lora_scale, dg, gv);
              uv = fmaf(p.lora_scale, du, uv);
            }
            p.h[static_cast<int64_t>(sl) * I + col] = float_to_bf16_bits(silu_f32(gv) * uv);
          }
        }
        __syncwarp();
        if (lane == 0) {
          fin_cnt[gi][par] = 0;
          mbar_arrive(&rfree[gi * 2 + par]);  // the buffer may take item iq + 2's partials
        }
      }
    }
  }

  // --------------------------------------------------------- grid barrier
  named_bar(kBarMath, kMath * 32);  // every h store of this CTA is issued
  if (warp == 0) {
    // The block barrier above orders every h store of this CTA before this
    // release store (release is cumulative), so no full fence is needed: a
    // fence here measured 2-4 us on B200, waiting out the CTA's copies in flight.
    if (lane == 0) st_release_gpu(p.flags + bid, tag);
    __syncwarp();
    unsigned long long t0 = 0;
    for (uint32_t it = 0;; ++it) {
      // Independent relaxed loads of every slot (one round trip per poll),
      // then one fence once all are seen.
      bool ready = true;
      for (int base = 0; base < G; base += 256) {
        unsigned long long v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c = base + lane + 32 * i;
          v[i] = c < G ? ld_relaxed_gpu(p.flags + c) : tag;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) ready = ready && v[i] == tag;
      }
      if (__all_sync(0xffffffffu, ready)) {
        asm volatile("fence.acq_rel.gpu;" ::: "memory");  // acquire: the slots' releases before the h reads
        // Every CTA has read the old epoch: advance it for the next launch.
        if (bid == 0 && lane == 0) st_release_gpu(p.flags + kMaxGrid, tag);
        break;
      }
      if (abort_s) break;
      if ((it & 63u) == 0) {  // the clock only now and then: see mbar_wait
        const unsigned long long now = global_ns();
        if (it == 0) {
          t0 = now;
        } else if (now - t0 > kWaitLimitNs) {
          if (lane == 0) {
            abort_s = 1;
            record_error(p.err, kErrGridBarrier);
          }
          break;
        }
      }
    }
  }
  named_bar(kBarMath, kMath * 32);

  // -------------------------------------------------------------- phase 2
  {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    uint4 hA[PPW][2], hB[PPW][2];
    // h fragments of a stage for this warp's pairs (zeros where token g does
    // not route to the pair's expert), read from L2 one stage ahead of their use.
    // The warp's pair q is (expert pe[q] of the stage's chunk, k-block pk[q])
    // in every stage.
    int pe[PPW], pk[PPW];
#pragma unroll
    for (int q = 0; q < PPW; ++q) {
      pe[q] = (warp + kMath * q) / KBI;
      pk[q] = (warp + kMath * q) - pe[q] * KBI;
    }
    // h fragments of a stage of chunk ch (nothing when `live` is false).
    auto load_h = [&](int ch, bool live, uint4 (&hb)[PPW][2]) {
#pragma unroll
      for (int q = 0; q < PPW; ++q) hb[q][0] = hb[q][1] = make_uint4(0, 0, 0, 0);
      if (!live) return;
      const int u0 = ch * DPE, np = min(DPE, nU - u0) * KBI;
#pragma unroll
      for (int q = 0; q < PPW; ++q) {
        const int pi = warp + kMath * q;
        if (pi < np) {
          const int u = u0 + pe[q], kb = pk[q];
          const int sg = g < p.M ? slotmap[u * kMaxM + g] : -1;
          if (sg >= 0) {
            const uint4* src = reinterpret_cast<const uint4*>(p.h + static_cast<int64_t>(sg) * I + kb * 64 + 16 * t);
            hb[q][0] = __ldcg(src);
            hb[q][1] = __ldcg(src + 1);
          }
        }
      }
    };
    // Stage of ring slot s (pass ph), chunk ch of row-block round rbq.
    auto compute = [&](int s, int ph, int ch, int rbq, const uint4 (&hb)[PPW][2]) {
      ring_wait(&full[s], ph, &abort_s, p.err, kErrWaitFull);
      const unsigned char* st = ring + static_cast<uint32_t>(s) * slot;
      const int u0 = ch * DPE, np = min(DPE, nU - u0) * KBI;
      // The warp's pairs two at a time (independent MMA chains interleaved).
      auto pair_in = [&](int q, uint2& w0, uint2& w1, float& s0, float& s1, float& s2, float& s3) {
        const int ei = pe[q], kb = pk[q], u = u0 + ei;
        // MMA row g = block row 4 (g % 4) + g / 4, row g + 8 = that + 2.
        const unsigned char* base = st + ei * exp_dn;
        const float* am = reinterpret_cast<const float*>(base + am_dn);
        const int cg = g & 3, r = g >> 2;
        const uint32_t off = cg * cs_dn + r * (I / 2) + kb * 32 + 8 * t;
        w0 = lds64(base + off);
        w1 = lds64(base + off + I);  // two rows further
        const float a0 = am[cg * as_dn + r * KBI + kb], a1 = am[cg * as_dn + (r + 2) * KBI + kb];
        const int sl0 = (2 * t < p.M) ? slotmap[u * kMaxM + 2 * t] : -1;
        const int sl1 = (2 * t + 1 < p.M) ? slotmap[u * kMaxM + 2 * t + 1] : -1;
        const float wc0 = sl0 >= 0 ? w_s[sl0] : 0.f, wc1 = sl1 >= 0 ? w_s[sl1] : 0.f;
        s0 = a0 * wc0;
        s1 = a0 * wc1;
        s2 = a1 * wc0;
        s3 = a1 * wc1;
      };
#pragma unroll
      for (int q = 0; q < PPW; q += 2) {
        const bool va = warp + kMath * q < np, vb = q + 1 < PPW && warp + kMath * (q + 1) < np;
        if (va && vb) {
          uint2 w0a, w1a, w0b, w1b;
          float sa[4], sb[4];
          pair_in(q, w0a, w1a, sa[0], sa[1], sa[2], sa[3]);
          pair_in(q + 1, w0b, w1b, sb[0], sb[1], sb[2], sb[3]);
          float da[4] = {0.f, 0.f, 0.f, 0.f}, db[4] = {0.f, 0.f, 0.f, 0.f};
          block_mma2(lut_b, lane4, w0a, w1a, reinterpret_cast<const uint32_t*>(hb[q]), w0b, w1b,
                     reinterpret_cast<const uint32_t*>(hb[q + 1 < PPW ? q + 1 : q]), da, db);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] = fmaf(sb[i], db[i], fmaf(sa[i], da[i], acc[i]));
        } else if (va) {
          uint2 w0a, w1a;
          float sa[4];
          pair_in(q, w0a, w1a, sa[0], sa[1], sa[2], sa[3]);
          float da[4] = {0.f, 0.f, 0.f, 0.f};
          block_mma(lut_b, lane4, w0a, w1a, reinterpret_cast<const uint32_t*>(hb[q]), da);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] = fmaf(sa[i], da[i], acc[i]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (ch == nch - 1) {
        // End of a row block: the 16 warps' sums in warp order -> out.
        if (rbq > 0) named_bar(kBarMath, kMath * 32);  // the previous row block's sums are read
        *red_at(warp * 32 + lane) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        named_bar(kBarMath, kMath * 32);
        if (warp == rbq % kMath) {
          float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int w = 0; w < kMath; ++w) {
            const float4 v = *red_at(w * 32 + lane);
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
          }
          const int row0 = (bid + rbq * G) * 16 + 4 * (g & 3) + (g >> 2);
          const float v[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
          for (int q2 = 0; q2 < 4; ++q2) {
            const int tok = 2 * t + (q2 & 1);
            const int row = row0 + ((q2 >> 1) ? 2 : 0);
            if (tok < p.M) p.out[static_cast<int64_t>(tok) * H + row] = float_to_bf16_bits(v[q2]);
          }
        }
      }
    };
    // Stage jd is ring stage n_gu + jd: slot s, pass ph; chunk ch of round rbq.
    int s = n_gu % RS, ph = (n_gu / RS) & 1, ch = 0, rbq = 0;
    load_h(0, n_dn > 0, hA);
#pragma unroll 1
    for (int jd = 0; jd < n_dn; ++jd) {
      const int ch1 = ch + 1 == nch ? 0 : ch + 1;
      load_h(ch1, jd + 1 < n_dn, hB);
      compute(s, ph, ch, rbq, hA);
#pragma unroll
      for (int q = 0; q < PPW; ++q) {
        hA[q][0] = hB[q][0];
        hA[q][1] = hB[q][1];
      }
      if (++s == RS) {
        s = 0;
        ph ^= 1;
      }
      if (ch1 == 0) ++rbq;
      ch = ch1;
    }
  }
}

using KernelFn = void (*)(FusedParams);

template <int SPW>
KernelFn pick_ppw(int ppw) {
  switch (ppw) {
    case 1: return decode_fused_kernel<SPW, 1>;
    case 2: return decode_fused_kernel<SPW, 2>;
    default: return decode_fused_kernel<SPW, 3>;
  }
}

KernelFn pick_kernel(int spw, int ppw) {
  switch (spw) {
    case 1: return pick_ppw<1>(ppw);
    case 2: return pick_ppw<2>(ppw);
    case 3: return pick_ppw<3>(ppw);
    default: return pick_ppw<4>(ppw);
  }
}

// Launch plan of one shape.
struct Plan {
  int spw, ppw, dpe, stages, grid;
  uint32_t slot;
  size_t smem;
};

// Fills *pl; returns "" or why the shape does not fit the kernel.
std::string make_plan(int M, int k, int E, int H, int I, int r, size_t smem_limit, int sm_count, Plan* pl) {
  const int KB = H / 64, KBI = I / 64, nsp = (KB + 1) / 2;
  pl->spw = (nsp + kGW - 1) / kGW;
  if (pl->spw > kMaxSPW) return "the decode path takes H <= " + std::to_string(kGW * kMaxSPW * 128);
  if (KBI > kMaxKBI) return "the decode path takes I <= " + std::to_string(kMaxKBI * 64);
  const uint32_t gu = gu_stage_bytes(H), dn = dn_block_bytes(I);
  pl->dpe = std::max(1, std::min({static_cast<int>(gu / dn), kMaxDPE, kMaxKBI / KBI}));
  pl->ppw = (pl->dpe * KBI + kMath - 1) / kMath;
  pl->slot = al(std::max(gu, static_cast<uint32_t>(pl->dpe) * dn), 128);
  const size_t fixed = make_smem(M, k, E, r, I, 0, pl->slot).ring + 2 * kMaxStages * 8;
  if (fixed >= smem_limit) return "the decode kernel's shared-memory plan does not fit this shape";
  int st = static_cast<int>((smem_limit - fixed) / pl->slot);
  st = std::min(st, kMaxStages) & ~1;
  if (st < 2) return "the decode kernel's shared-memory ring does not fit this shape";
  pl->stages = st;
  pl->smem = make_smem(M, k, E, r, I, st, pl->slot).total;
  const int items_upper = std::min(M * k, E) * (I / 16);
  pl->grid = std::max(1, std::min({sm_count, kMaxGrid, std::max(items_upper, H / 16)}));
  return "";
}

struct DecodeWs {
  size_t flags, h, total;
};

// Workspace: the error word every workspace begins with (256-byte slot), the
// grid barrier's slots (one 64-bit word per CTA) and its epoch word, h [M*k, I] bf16.
DecodeWs decode_ws(int64_t M, int k, int64_t I) {
  DecodeWs w;
  w.flags = 256;
  w.h = w.flags + align_up(static_cast<size_t>(kMaxGrid + 1) * 8, 256);
  w.total = w.h + align_up(static_cast<size_t>(M * k * I * 2), 256);
  return w;
}

}  // namespace

std::string decode_unsupported_reason(int64_t M, int64_t E, int k, int64_t H, int64_t I) {
  if (M < 1 || M > kMaxM) return "the decode path takes 1 to " + std::to_string(kMaxM) + " tokens (M=" + std::to_string(M) + ")";
  if (k > 32) return "the decode path takes k <= 32 (k=" + std::to_string(k) + ")";
  if (E > 512) return "the decode path takes at most 512 experts (E=" + std::to_string(E) + ")";
  if (H > kGW * kMaxSPW * 128)
    return "the decode path takes H <= " + std::to_string(kGW * kMaxSPW * 128) + " (H=" + std::to_string(H) + ")";
  if (I > kMaxKBI * 64) return "the decode path takes I <= " + std::to_string(kMaxKBI * 64) + " (I=" + std::to_string(I) + ")";
  DeviceInfo di;
  if (device_info(&di) != cudaSuccess) return "device query failed";
  Plan pl;
  return make_plan(static_cast<int>(M), k, static_cast<int>(E), static_cast<int>(H), static_cast<int>(I), 16,
                   di.smem_optin - 1024, di.sm_count, &pl);
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
  FusedParams p{};
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
  p.err = static_cast<int*>(a.workspace);
  p.flags = reinterpret_cast<unsigned long long*>(static_cast<char*>(a.workspace) + ws.flags);
  p.h = reinterpret_cast<uint16_t*>(static_cast<char*>(a.workspace) + ws.h);
  p.out = a.out;
  Plan pl;
  if (!make_plan(p.M, p.k, p.E, p.H, p.I, r, di.smem_optin - 1024, di.sm_count, &pl).empty())
    return cudaErrorInvalidConfiguration;
  p.stages = pl.stages;
  p.dpe = pl.dpe;
  const KernelFn fn = pick_kernel(pl.spw, pl.ppw);
  err = ensure_smem_limit(reinterpret_cast<const void*>(fn), pl.smem);
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  LaunchScope ls("decode.fused", stream);
  return cudaLaunchKernelEx(&cfg, fn, p);
}

}  // namespace e4b
