// Elementwise and per-row steps of the layer backward through frozen NF4 experts.
//
// The layer backward (routing ids held fixed) recomputes the gate_up output
// a = [g | u] and the per-slot expert outputs z, then runs two grouped dgrad
// products with the SwiGLU derivative between them (experts4bit-qlora 0.22.0,
// "Which training path?": the frozen base is decoded again inside backward,
// one dgrad launch per projection).  These kernels are the steps between the
// GEMMs, all in group order p (perm[p] = flat slot t*k + j, row_token[p] = t):
//
//   swiglu_h      h_p    = bf16(SiLU(g_p) * u_p)
//   slot_grads    dz_p   = bf16(w_p * dout_t)          dw_(t,j) = dout_t . z_p
//   swiglu_bwd    da_p   = bf16([dh * u * SiLU'(g) | dh * SiLU(g)]),  SiLU'(g) = s (1 + g (1 - s))
//   token_sum     dx_t   = sum_j dxg_(inv[t*k + j])   (j ascending)
//   router_grad   dlogits_t through the routing weights: with renormalisation
//                 w_j (dw_j - sum_i w_i dw_i) on the selected experts; without
//                 it sum_j dw_j w_j (delta(e, id_j) - p_e) over the full softmax p.
#include "common.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

__device__ __forceinline__ float sigmoid_f32(float z) { return 1.0f / (1.0f + __expf(-z)); }

__global__ void swiglu_h_kernel(const float* __restrict__ a, int64_t S, int I, uint16_t* __restrict__ h) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // one 4-wide column group
  const int64_t per_row = I / 4;
  if (i >= S * per_row) return;
  const int64_t p = i / per_row, c = (i % per_row) * 4;
  const float4 g = *reinterpret_cast<const float4*>(a + p * 2 * I + c);
  const float4 u = *reinterpret_cast<const float4*>(a + p * 2 * I + I + c);
  const uint32_t lo = pack_bf16x2(silu_f32(g.x) * u.x, silu_f32(g.y) * u.y);
  const uint32_t hi = pack_bf16x2(silu_f32(g.z) * u.z, silu_f32(g.w) * u.w);
  *reinterpret_cast<uint2*>(h + p * I + c) = make_uint2(lo, hi);
}

// One warp per grouped row p: dz_p and the slot's dw.
__global__ void slot_grads_kernel(const uint16_t* __restrict__ dout, const float* __restrict__ z,
                                  const int32_t* __restrict__ perm, const int32_t* __restrict__ row_token,
                                  const float* __restrict__ w, int64_t S, int64_t M, int H,
                                  uint16_t* __restrict__ dz, float* __restrict__ dw) {
  const int lane = threadIdx.x & 31;
  const int64_t p = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (p >= S) return;
  const int64_t f = clampv<int64_t>(perm[p], 0, S - 1);
  const int64_t t = clampv<int64_t>(row_token[p], 0, M - 1);
  const float wp = w[f];
  const uint16_t* d = dout + t * H;
  const float* zp = z + p * H;
  float acc = 0.f;
  for (int c = lane * 8; c < H; c += 256) {
    const uint4 dv = *reinterpret_cast<const uint4*>(d + c);
    const float4 z0 = *reinterpret_cast<const float4*>(zp + c);
    const float4 z1 = *reinterpret_cast<const float4*>(zp + c + 4);
    const uint32_t dw4[4] = {dv.x, dv.y, dv.z, dv.w};
    const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(dw4[i] << 16), hi = __uint_as_float(dw4[i] & 0xffff0000u);
      acc = fmaf(lo, zz[2 * i], acc);
      acc = fmaf(hi, zz[2 * i + 1], acc);
      o[i] = pack_bf16x2(wp * lo, wp * hi);
    }
    *reinterpret_cast<uint4*>(dz + p * H + c) = make_uint4(o[0], o[1], o[2], o[3]);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) dw[f] = acc;
}

__global__ void swiglu_bwd_kernel(const float* __restrict__ a, const float* __restrict__ dh, int64_t S, int I,
                                  uint16_t* __restrict__ da) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_row = I / 4;
  if (i >= S * per_row) return;
  const int64_t p = i / per_row, c = (i % per_row) * 4;
  const float4 g4 = *reinterpret_cast<const float4*>(a + p * 2 * I + c);
  const float4 u4 = *reinterpret_cast<const float4*>(a + p * 2 * I + I + c);
  const float4 d4 = *reinterpret_cast<const float4*>(dh + p * I + c);
  const float g[4] = {g4.x, g4.y, g4.z, g4.w}, u[4] = {u4.x, u4.y, u4.z, u4.w}, d[4] = {d4.x, d4.y, d4.z, d4.w};
  float dg[4], du[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float s = sigmoid_f32(g[j]);
    dg[j] = d[j] * u[j] * (s * (1.0f + g[j] * (1.0f - s)));
    du[j] = d[j] * (g[j] * s);
  }
  *reinterpret_cast<uint2*>(da + p * 2 * I + c) = make_uint2(pack_bf16x2(dg[0], dg[1]), pack_bf16x2(dg[2], dg[3]));
  *reinterpret_cast<uint2*>(da + p * 2 * I + I + c) =
      make_uint2(pack_bf16x2(du[0], du[1]), pack_bf16x2(du[2], du[3]));
}

__global__ void token_sum_kernel(const float* __restrict__ dxg, const int32_t* __restrict__ inv, int64_t M, int k,
                                 int H, float* __restrict__ dx) {
  const int64_t t = blockIdx.x;
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (t >= M || c >= H) return;
  const int64_t S = M * k;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const int64_t p = clampv<int64_t>(inv[t * k + j], 0, S - 1);
    const float4 v = *reinterpret_cast<const float4*>(dxg + p * H + c);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  *reinterpret_cast<float4*>(dx + t * H + c) = acc;
}

// One warp per token.
__global__ void router_grad_kernel(const float* __restrict__ logits, const int32_t* __restrict__ ids,
                                   const float* __restrict__ w, const float* __restrict__ dw, int64_t M, int E, int k,
                                   int renormalize, float* __restrict__ dlogits) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (t >= M) return;
  // C = sum_j w_j dw_j over the token's k slots (k <= 32: one slot per lane)
  const float cj = lane < k ? w[t * k + lane] * dw[t * k + lane] : 0.f;
  float C = cj;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) C += __shfl_xor_sync(0xffffffffu, C, off);
  const int idl = lane < k ? ids[t * k + lane] : -1;
  float* out = dlogits + t * E;
  if (renormalize) {
    for (int e = lane; e < E; e += 32) out[e] = 0.f;
    __syncwarp();
    if (lane < k && idl >= 0 && idl < E) out[idl] = cj - w[t * k + lane] * C;
    return;
  }
  // full softmax p over the E logits
  const float* lg = logits + t * E;
  float mx = -INFINITY;
  for (int e = lane; e < E; e += 32) mx = fmaxf(mx, lg[e]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float sum = 0.f;
  for (int e = lane; e < E; e += 32) sum += expf(lg[e] - mx);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  for (int e = lane; e < E; e += 32) out[e] = -(expf(lg[e] - mx) / sum) * C;
  __syncwarp();
  // the selected experts (distinct ids) add their own coefficient, one lane each
  if (lane < k && idl >= 0 && idl < E) out[idl] += cj;
}

}  // namespace

cudaError_t launch_swiglu_h(const float* a, int64_t S, int I, uint16_t* h, cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  const int64_t n = S * (I / 4);
  LaunchScope ls("backward.swiglu_h", stream);
  swiglu_h_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(a, S, I, h);
  return cudaGetLastError();
}

cudaError_t launch_slot_grads(const uint16_t* dout, const float* z, const int32_t* perm, const int32_t* row_token,
                              const float* w, int64_t S, int64_t M, int H, uint16_t* dz, float* dw,
                              cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  LaunchScope ls("backward.slot_grads", stream);
  slot_grads_kernel<<<static_cast<unsigned>((S * 32 + 255) / 256), 256, 0, stream>>>(dout, z, perm, row_token, w, S,
                                                                                     M, H, dz, dw);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_bwd(const float* a, const float* dh, int64_t S, int I, uint16_t* da, cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  const int64_t n = S * (I / 4);
  LaunchScope ls("backward.swiglu_bwd", stream);
  swiglu_bwd_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(a, dh, S, I, da);
  return cudaGetLastError();
}

cudaError_t launch_token_sum(const float* dxg, const int32_t* inv, int64_t M, int k, int H, float* dx,
                             cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>(M), static_cast<unsigned>((H / 4 + 127) / 128));
  LaunchScope ls("backward.token_sum", stream);
  token_sum_kernel<<<grid, 128, 0, stream>>>(dxg, inv, M, k, H, dx);
  return cudaGetLastError();
}

cudaError_t launch_router_grad(const float* logits, const int32_t* ids, const float* w, const float* dw, int64_t M,
                               int E, int k, bool renormalize, float* dlogits, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  LaunchScope ls("backward.router_grad", stream);
  router_grad_kernel<<<static_cast<unsigned>((M * 32 + 255) / 256), 256, 0, stream>>>(logits, ids, w, dw, M, E, k,
                                                                                      renormalize ? 1 : 0, dlogits);
  return cudaGetLastError();
}

}  // namespace e4b
