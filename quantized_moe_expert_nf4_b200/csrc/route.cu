// Router top-k and the token/expert permutation.
//
// Follows experts4bit-qlora 0.22.0, "Which training path?": the token/expert
// pairs are sorted into per-expert groups so that each group runs as one GEMM.
// Top-k orders experts by (logit descending, index ascending); the weights are
// the softmax over the selected logits (renormalised) or the full softmax.
//
// The permutation is a stable counting sort without atomics, so it is
// deterministic:
//   * one warp per token selects the top k with 64-bit (value, ~index) keys;
//   * the slots of a tile are ranked within their expert in slot order by one
//     warp with __match_any_sync (peers share an expert; rank = peers below);
//   * positions = offsets[e] + (slots of e in earlier tiles) + local rank.
// Small calls (<= 4096 slots) run all of it in one CTA, one launch.  Larger
// calls use a tile kernel (top-k, local ranks, per-tile counts), a column scan
// per expert over the tiles, and a scatter kernel whose CTAs each scan the
// expert totals into the offsets.
#include <algorithm>

#include "common.cuh"
#include "e4b_internal.h"
#include "topk.cuh"

namespace e4b {
namespace {

constexpr int kSmallMaxSlots = 4096;
constexpr int kTileTokens = 16;  // tokens per tile of the large path

// Ranks slots [0, n) of `ids_s` within their expert in slot order, by one warp.
// counts[e] must be zero on entry; on exit it holds the per-expert totals.
__device__ __forceinline__ void warp_rank_slots(const int* ids_s, int n, int* rank_s, int* counts) {
  const int lane = threadIdx.x & 31;
  for (int base = 0; base < n; base += 32) {
    const int f = base + lane;
    const bool valid = f < n;
    const int e = valid ? ids_s[f] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int before = __popc(peers & lanemask_lt());
    const int c = valid ? counts[e] : 0;
    if (valid) rank_s[f] = c + before;
    __syncwarp();
    // The highest lane of each peer group bumps the count.
    const bool last = (peers >> lane) == 1u;
    if (valid && last) counts[e] = c + __popc(peers);
    __syncwarp();
  }
}

// Exclusive scan over counts[0..E) by the whole block (blockDim a multiple of 32,
// at most 1024; E of any size is handled in chunks).  Result in offs[0..E].
__device__ void block_exclusive_scan(const int* counts, int E, int* offs, int* warp_sums) {
  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  int carry = 0;
  for (int base = 0; base < E; base += blockDim.x) {
    const int e = base + tid;
    const int v = (e < E) ? counts[e] : 0;
    const int incl = warp_inclusive_scan(v);
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      const int ws = (lane < nwarps) ? warp_sums[lane] : 0;
      const int wi = warp_inclusive_scan(ws);
      if (lane < nwarps) warp_sums[lane] = wi - ws;
      if (lane == 31) warp_sums[32] = wi;  // block total
    }
    __syncthreads();
    if (e < E) offs[e] = carry + warp_sums[wid] + incl - v;
    const int total = warp_sums[32];
    __syncthreads();
    carry += total;
  }
  if (tid == 0) offs[E] = carry;
  __syncthreads();
}

template <int MAXJ>
__global__ void __launch_bounds__(512) route_small_kernel(const float* __restrict__ logits, int M, int E, int k,
                                                           bool renormalize, RouteOut o) {
  extern __shared__ int smem[];
  const int S = M * k;
  int* ids_s = smem;              // [S]
  int* rank_s = ids_s + S;        // [S]
  int* counts = rank_s + S;       // [E]
  int* offs = counts + E;         // [E+1]
  int* warp_sums = offs + E + 1;  // [33]
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nwarps = blockDim.x >> 5;

  for (int e = tid; e < E; e += blockDim.x) counts[e] = 0;
  for (int t = wid; t < M; t += nwarps) {
    const int id = route_token<MAXJ>(logits, t, E, k, renormalize, o.ids, o.w);
    if (lane < k) ids_s[t * k + lane] = id;
  }
  __syncthreads();
  if (wid == 0) warp_rank_slots(ids_s, S, rank_s, counts);
  __syncthreads();
  block_exclusive_scan(counts, E, offs, warp_sums);
  for (int e = tid; e <= E; e += blockDim.x) o.offsets[e] = offs[e];
  for (int f = tid; f < S; f += blockDim.x) {
    const int pos = offs[ids_s[f]] + rank_s[f];
    o.perm[pos] = f;
    o.inv[f] = pos;
    if (o.row_token) o.row_token[pos] = f / k;
  }
}

// Large path, kernel 1: one CTA per tile of kTileTokens tokens.
template <int MAXJ>
__global__ void __launch_bounds__(256) route_tile_kernel(const float* __restrict__ logits, int M, int E, int k,
                                                         bool renormalize, RouteOut o,
                                                         int* __restrict__ local_rank,
                                                         int* __restrict__ tile_counts) {
  extern __shared__ int smem[];
  const int tile_slots = kTileTokens * k;
  int* ids_s = smem;                 // [tile_slots]
  int* rank_s = ids_s + tile_slots;  // [tile_slots]
  int* counts = rank_s + tile_slots; // [E]
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int t0 = blockIdx.x * kTileTokens;
  const int ntok = min(kTileTokens, M - t0);
  for (int e = tid; e < E; e += blockDim.x) counts[e] = 0;
  for (int i = wid; i < ntok; i += (blockDim.x >> 5)) {
    const int id = route_token<MAXJ>(logits, t0 + i, E, k, renormalize, o.ids, o.w);
    if (lane < k) ids_s[i * k + lane] = id;
  }
  __syncthreads();
  if (wid == 0) warp_rank_slots(ids_s, ntok * k, rank_s, counts);
  __syncthreads();
  for (int i = tid; i < ntok * k; i += blockDim.x) local_rank[t0 * k + i] = rank_s[i];
  for (int e = tid; e < E; e += blockDim.x) tile_counts[static_cast<int64_t>(blockIdx.x) * E + e] = counts[e];
}

// Large path, kernel 2: one CTA per expert scans that expert's per-tile counts
// over the tiles, in place (tile_counts[t][e] becomes the slots of e in tiles
// before t), and writes the expert's total.
__global__ void __launch_bounds__(1024) route_colscan_kernel(int ntiles, int E, int* __restrict__ tile_counts,
                                                             int* __restrict__ totals) {
  __shared__ int warp_sums[33];
  const int e = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  int carry = 0;
  for (int base = 0; base < ntiles; base += blockDim.x) {
    const int t = base + tid;
    int* cell = tile_counts + static_cast<int64_t>(t) * E + e;
    const int v = (t < ntiles) ? *cell : 0;
    const int incl = warp_inclusive_scan(v);
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      const int ws = (lane < nwarps) ? warp_sums[lane] : 0;
      const int wi = warp_inclusive_scan(ws);
      if (lane < nwarps) warp_sums[lane] = wi - ws;
      if (lane == 31) warp_sums[32] = wi;  // block total
    }
    __syncthreads();
    if (t < ntiles) *cell = carry + warp_sums[wid] + incl - v;
    const int total = warp_sums[32];
    __syncthreads();
    carry += total;
  }
  if (tid == 0) totals[e] = carry;
}

// Large path, kernel 3: every CTA scans the expert totals into the offsets and
// places its tile's slots.
__global__ void __launch_bounds__(1024) route_scatter_kernel(int M, int E, int k, RouteOut o,
                                                             const int* __restrict__ local_rank,
                                                             const int* __restrict__ tile_before,
                                                             const int* __restrict__ totals) {
  extern __shared__ int smem[];
  int* offs = smem;               // [E+1]
  int* warp_sums = offs + E + 1;  // [33]
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  block_exclusive_scan(totals, E, offs, warp_sums);
  if (tile == 0)
    for (int e = tid; e <= E; e += blockDim.x) o.offsets[e] = offs[e];
  const int* before = tile_before + static_cast<int64_t>(tile) * E;
  const int f0 = tile * kTileTokens * k;
  const int nslots = min(kTileTokens, M - tile * kTileTokens) * k;
  for (int i = tid; i < nslots; i += blockDim.x) {
    const int f = f0 + i;
    const int e = o.ids[f];
    const int pos = offs[e] + before[e] + local_rank[f];
    o.perm[pos] = f;
    o.inv[f] = pos;
    if (o.row_token) o.row_token[pos] = f / k;
  }
}

template <int MAXJ>
cudaError_t launch_route_t(const float* logits, int64_t M, int E, int k, bool renormalize, const RouteOut& o,
                           void* workspace, cudaStream_t stream) {
  const int64_t S = M * k;
  if (S <= kSmallMaxSlots) {
    const size_t smem = (2 * S + 2 * E + 1 + 33) * sizeof(int);
    LaunchScope ls("route.small", stream);
    route_small_kernel<MAXJ><<<1, 512, smem, stream>>>(logits, static_cast<int>(M), E, k, renormalize, o);
    set_path("route.small");
    return cudaGetLastError();
  }
  const int ntiles = static_cast<int>((M + kTileTokens - 1) / kTileTokens);
  int* local_rank = static_cast<int*>(workspace);
  int* tile_counts = local_rank + align_up(S, 64);
  const size_t smem1 = (2 * kTileTokens * k + E) * sizeof(int);
  {
    LaunchScope ls("route.tile", stream);
    route_tile_kernel<MAXJ><<<ntiles, 256, smem1, stream>>>(logits, static_cast<int>(M), E, k, renormalize, o,
                                                            local_rank, tile_counts);
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  int* totals = tile_counts + static_cast<int64_t>(ntiles) * E;
  {
    const int threads = std::min(1024, (ntiles + 31) / 32 * 32);
    LaunchScope ls("route.colscan", stream);
    route_colscan_kernel<<<E, threads, 0, stream>>>(ntiles, E, tile_counts, totals);
  }
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t smem2 = (E + 1 + 33) * sizeof(int);
  LaunchScope ls("route.scatter", stream);
  route_scatter_kernel<<<ntiles, 1024, smem2, stream>>>(static_cast<int>(M), E, k, o, local_rank, tile_counts,
                                                        totals);
  set_path("route.tiled");
  return cudaGetLastError();
}

// Token gather: out[p, :] = A[row_index[p], :K], one warp per routed row,
// 16-byte vectors (K % 8 == 0, lda % 8 == 0, 16-byte aligned bases).  Indices
// out of range are clamped.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ A, int64_t a_rows,
                                                          int64_t lda, const int32_t* __restrict__ row_index,
                                                          int64_t S, int K, uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int vecs = K / 8;
  for (int64_t p = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; p < S; p += nwarps) {
    const int64_t src = clampv<int64_t>(row_index[p], 0, a_rows - 1);
    const uint4* s = reinterpret_cast<const uint4*>(A + src * lda);
    uint4* d = reinterpret_cast<uint4*>(out + p * K);
    for (int i0 = 0; i0 < vecs; i0 += 8 * 32) {  // eight 16-byte loads per lane in flight
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * 32 + lane;
        if (i < vecs) v[u] = __ldg(s + i);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * 32 + lane;
        if (i < vecs) d[i] = v[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_gather_rows(const uint16_t* A, int64_t a_rows, int64_t lda, const int32_t* row_index, int64_t S,
                               int K, uint16_t* out, cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int64_t want = (S + 7) / 8;
  const int64_t cap = static_cast<int64_t>(di.sm_count) * 16;
  LaunchScope ls("gather", stream);
  gather_rows_kernel<<<static_cast<int>(want < cap ? want : cap), 256, 0, stream>>>(A, a_rows, lda, row_index, S, K,
                                                                                   out);
  return cudaGetLastError();
}

size_t route_workspace_bytes(int64_t M, int64_t E, int k) {
  const int64_t S = M * k;
  if (S <= kSmallMaxSlots) return 0;
  const int64_t ntiles = (M + kTileTokens - 1) / kTileTokens;
  return (align_up(S, 64) + ntiles * E + align_up(E, 64)) * sizeof(int);
}

cudaError_t launch_route(const float* logits, int64_t M, int E, int k, bool renormalize, const RouteOut& o,
                         void* workspace, cudaStream_t stream) {
  if (M == 0) return cudaMemsetAsync(o.offsets, 0, (E + 1) * sizeof(int32_t), stream);
  if (E <= 32) return launch_route_t<1>(logits, M, E, k, renormalize, o, workspace, stream);
  if (E <= 64) return launch_route_t<2>(logits, M, E, k, renormalize, o, workspace, stream);
  if (E <= 128) return launch_route_t<4>(logits, M, E, k, renormalize, o, workspace, stream);
  if (E <= 256) return launch_route_t<8>(logits, M, E, k, renormalize, o, workspace, stream);
  if (E <= 512) return launch_route_t<16>(logits, M, E, k, renormalize, o, workspace, stream);
  return launch_route_t<32>(logits, M, E, k, renormalize, o, workspace, stream);
}

}  // namespace e4b
