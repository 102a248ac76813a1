// The extern "C" boundary of libe4b: argument checks, workspace layout, launches.
//
// Every call validates its arguments on the host before launching anything
// and reports failures through a status code plus a per-thread message; no
// call allocates or frees, and none synchronises except the diagnostic read of
// a workspace's error word.  See include/e4b.h for the contract.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "async.cuh"
#include "e4b_internal.h"

namespace e4b {

namespace {
thread_local std::string g_error;
thread_local const char* g_path = "";
thread_local int g_launches = 0;

struct TimingRec {
  const char* name;
  cudaEvent_t start, stop;
};
struct TimingState {
  bool on = false;
  std::vector<TimingRec> recs;
  std::vector<cudaEvent_t> pool;  // events reused across enable cycles
  size_t pool_used = 0;
  cudaEvent_t take() {
    if (pool_used == pool.size()) {
      cudaEvent_t ev;
      if (cudaEventCreate(&ev) != cudaSuccess) return nullptr;
      pool.push_back(ev);
    }
    return pool[pool_used++];
  }
};
thread_local TimingState g_timing;

constexpr size_t kAlign = 256;

struct Carve {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  }
};

// Workspace of the grouped forward path.
struct GroupedLayout {
  size_t err, ids, w, offsets, perm, inv, row_token, route_ws, xa, xg, h, z, total;
};

GroupedLayout grouped_layout(int64_t M, int64_t E, int64_t H, int64_t I, int k, int r) {
  const int64_t S = M * k;
  Carve c;
  GroupedLayout L;
  L.err = c.take(sizeof(int32_t));
  L.ids = c.take(S * sizeof(int32_t));
  L.w = c.take(S * sizeof(float));
  L.offsets = c.take((E + 1) * sizeof(int32_t));
  L.perm = c.take(S * sizeof(int32_t));
  L.inv = c.take(S * sizeof(int32_t));
  L.row_token = c.take(S * sizeof(int32_t));
  L.route_ws = c.take(route_workspace_bytes(M, E, k));
  L.xa = c.take(r > 0 ? S * 128 : 0);  // LoRA products, either layout (r <= 16)
  L.xg = c.take(S * H * sizeof(uint16_t));
  L.h = c.take(S * I * sizeof(uint16_t));
  L.z = c.take(S * H * sizeof(uint16_t));
  L.total = c.off;
  return L;
}

// Workspace of the layer backward (grouped order throughout).
struct BackwardLayout {
  size_t err, ids, w, offsets, perm, inv, row_token, route_ws, xa, xg, a, h, z, dz, dw, dh, da, dxg, yb, lg_xa, total;
};

BackwardLayout backward_layout(int64_t M, int64_t E, int64_t H, int64_t I, int k, int r) {
  const int64_t S = M * k;
  Carve c;
  BackwardLayout L;
  L.err = c.take(sizeof(int32_t));
  L.ids = c.take(S * sizeof(int32_t));
  L.w = c.take(S * sizeof(float));
  L.offsets = c.take((E + 1) * sizeof(int32_t));
  L.perm = c.take(S * sizeof(int32_t));
  L.inv = c.take(S * sizeof(int32_t));
  L.row_token = c.take(S * sizeof(int32_t));
  L.route_ws = c.take(route_workspace_bytes(M, E, k));
  L.xa = c.take(r > 0 ? S * 128 : 0);
  L.xg = c.take(S * H * sizeof(uint16_t));
  L.a = c.take(S * 2 * I * sizeof(float));
  L.h = c.take(S * I * sizeof(uint16_t));
  L.z = c.take(S * H * sizeof(float));
  L.dz = c.take(S * H * sizeof(uint16_t));
  L.dw = c.take(S * sizeof(float));
  L.dh = c.take(S * I * sizeof(float));
  L.da = c.take(S * 2 * I * sizeof(uint16_t));
  L.dxg = c.take(S * H * sizeof(float));
  L.yb = c.take(r > 0 ? S * r * sizeof(float) : 0);
  L.lg_xa = c.take(r > 0 ? S * r * sizeof(float) : 0);
  L.total = c.off;
  return L;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

e4b_status fail(e4b_status s, const std::string& msg) {
  g_error = msg;
  return s;
}

e4b_status cuda_fail(cudaError_t err, const char* where) {
  g_error = std::string(where) + ": " + cudaGetErrorName(err) + " (" + cudaGetErrorString(err) + ")";
  return E4B_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool quant_type_ok(int q) { return q == E4B_QUANT_NF4 || q == E4B_QUANT_FP4; }

// Size, presence and alignment of a caller's workspace.
e4b_status check_workspace(const char* what, size_t need, const void* workspace, size_t workspace_bytes) {
  if (workspace_bytes < need || (need > 0 && !workspace))
    return fail(E4B_ERR_WORKSPACE, std::string(what) + " workspace needs " + std::to_string(need) + " bytes");
  if (workspace && !aligned16(workspace))
    return fail(E4B_ERR_INVALID_ARGUMENT, std::string(what) + " workspace must be 16-byte aligned");
  return E4B_OK;
}

static_assert(kErrNone == E4B_KERNEL_ERR_NONE && kErrWaitFull == E4B_KERNEL_ERR_WAIT_FULL &&
                  kErrWaitEmpty == E4B_KERNEL_ERR_WAIT_EMPTY && kErrWaitDrain == E4B_KERNEL_ERR_WAIT_DRAIN &&
                  kErrGridBarrier == E4B_KERNEL_ERR_GRID_BARRIER,
              "device error codes match the header");

e4b_status check_device() {
  DeviceInfo di;
  const cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return cuda_fail(err, "device query");
  if (di.major != 10 || di.minor != 0)
    return fail(E4B_ERR_UNSUPPORTED, "libe4b is built for sm_100a (B200); current device is sm_" +
                                         std::to_string(di.major) + std::to_string(di.minor));
  return E4B_OK;
}

std::string shape_str(const char* name, int64_t v) { return std::string(name) + "=" + std::to_string(v); }

}  // namespace

void set_error(const std::string& msg) { g_error = msg; }
void set_path(const char* path) { g_path = path; }
void begin_call() {
  g_launches = 0;
  g_error.clear();
}

LaunchScope::LaunchScope(const char* name, cudaStream_t stream) : rec_(-1), stream_(stream) {
  ++g_launches;
  if (!g_timing.on) return;
  TimingRec r{name, g_timing.take(), g_timing.take()};
  if (!r.start || !r.stop) return;
  if (cudaEventRecord(r.start, stream) != cudaSuccess) return;
  g_timing.recs.push_back(r);
  rec_ = static_cast<int>(g_timing.recs.size()) - 1;
}

LaunchScope::~LaunchScope() {
  if (rec_ >= 0) cudaEventRecord(g_timing.recs[rec_].stop, stream_);
}

cudaError_t ensure_smem_limit(const void* func, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, size_t> raised;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lk(mu);
  size_t& cur = raised[{dev, func}];
  if (bytes <= cur) return cudaSuccess;
  err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (err != cudaSuccess) return err;
  cur = bytes;
  return cudaSuccess;
}

cudaError_t device_info(DeviceInfo* out) {
  static std::mutex mu;
  static std::vector<DeviceInfo> cache;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  {
    std::lock_guard<std::mutex> lk(mu);
    for (const auto& d : cache)
      if (d.device == dev) {
        *out = d;
        return cudaSuccess;
      }
  }
  DeviceInfo d{};
  d.device = dev;
  int v = 0;
  if ((err = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
  d.sm_count = v;
  if ((err = cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return err;
  d.major = v;
  if ((err = cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return err;
  d.minor = v;
  if ((err = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return err;
  d.smem_optin = static_cast<size_t>(v);
  std::lock_guard<std::mutex> lk(mu);
  cache.push_back(d);
  *out = d;
  return cudaSuccess;
}

cudaError_t launch_lora_xa(const GemmArgs& a, cudaStream_t stream);

e4b_status check_stack(const e4b_expert_stack* w, int k) {
  if (!w) return fail(E4B_ERR_INVALID_ARGUMENT, "null expert stack");
  if (w->E < 1 || w->E > 1024) return fail(E4B_ERR_UNSUPPORTED, "E must be in [1, 1024]");
  if (w->H < 64 || w->H % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "H must be a positive multiple of 64");
  if (w->I < 64 || w->I % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "I must be a positive multiple of 64");
  if (k < 1 || k > w->E || k > 32) return fail(E4B_ERR_INVALID_ARGUMENT, "k must be in [1, min(E, 32)]");
  if (!w->gu_packed || !w->gu_absmax || !w->dn_packed || !w->dn_absmax)
    return fail(E4B_ERR_INVALID_ARGUMENT, "null packed stack pointer");
  if (!quant_type_ok(w->quant_type)) return fail(E4B_ERR_INVALID_ARGUMENT, "quant_type must be NF4 or FP4");
  if ((w->lora_A == nullptr) != (w->lora_B == nullptr))
    return fail(E4B_ERR_INVALID_ARGUMENT, "lora_A and lora_B must be both set or both NULL");
  if (w->lora_A && (w->lora_r < 1 || w->lora_r > 16)) return fail(E4B_ERR_UNSUPPORTED, "LoRA rank must be in [1, 16]");
  if (w->lora_A && (!aligned16(w->lora_A) || !aligned16(w->lora_B)))
    return fail(E4B_ERR_INVALID_ARGUMENT, "lora_A and lora_B must be 16-byte aligned");
  if (!aligned16(w->gu_packed) || !aligned16(w->dn_packed) || !aligned16(w->gu_absmax) || !aligned16(w->dn_absmax))
    return fail(E4B_ERR_INVALID_ARGUMENT, "packed stacks and absmax must be 16-byte aligned");
  return E4B_OK;
}

e4b_status check_sm100() { return check_device(); }

}  // namespace e4b

using namespace e4b;

extern "C" {

const char* e4b_status_string(e4b_status s) {
  switch (s) {
    case E4B_OK: return "E4B_OK";
    case E4B_ERR_INVALID_ARGUMENT: return "E4B_ERR_INVALID_ARGUMENT";
    case E4B_ERR_UNSUPPORTED: return "E4B_ERR_UNSUPPORTED";
    case E4B_ERR_WORKSPACE: return "E4B_ERR_WORKSPACE";
    case E4B_ERR_CUDA: return "E4B_ERR_CUDA";
  }
  return "E4B_ERR_UNKNOWN";
}

const char* e4b_last_error(void) { return g_error.c_str(); }
const char* e4b_last_path(void) { return g_path; }
int e4b_version(void) { return E4B_VERSION; }
int e4b_last_launches(void) { return g_launches; }

// The two error-word calls leave the last call's path and launch count alone.
e4b_status e4b_workspace_error(const void* workspace, int32_t* code) {
  if (!workspace || !code) return fail(E4B_ERR_INVALID_ARGUMENT, "null workspace or code");
  if (!aligned16(workspace)) return fail(E4B_ERR_INVALID_ARGUMENT, "workspace must be 16-byte aligned");
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  cudaError_t err = cudaDeviceSynchronize();
  if (err != cudaSuccess) return cuda_fail(err, "synchronise before reading the error word");
  err = cudaMemcpy(code, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (err != cudaSuccess) return cuda_fail(err, "read of the error word");
  return E4B_OK;
}

e4b_status e4b_workspace_clear_error(void* workspace, e4b_stream stream) {
  if (!workspace) return fail(E4B_ERR_INVALID_ARGUMENT, "null workspace");
  if (!aligned16(workspace)) return fail(E4B_ERR_INVALID_ARGUMENT, "workspace must be 16-byte aligned");
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  cudaError_t err = cudaMemsetAsync(workspace, 0, sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "clear of the error word");
  return E4B_OK;
}

e4b_status e4b_timing_enable(int on) {
  g_timing.on = on != 0;
  g_timing.recs.clear();
  g_timing.pool_used = 0;
  return E4B_OK;
}

int e4b_timing_kernels(void) {
  std::vector<const char*> names;
  for (const auto& r : g_timing.recs)
    if (std::find_if(names.begin(), names.end(), [&](const char* n) { return std::strcmp(n, r.name) == 0; }) ==
        names.end())
      names.push_back(r.name);
  return static_cast<int>(names.size());
}

e4b_status e4b_timing_get(int i, const char** name, double* total_ms, int* launches) {
  std::vector<const char*> names;
  for (const auto& r : g_timing.recs)
    if (std::find_if(names.begin(), names.end(), [&](const char* n) { return std::strcmp(n, r.name) == 0; }) ==
        names.end())
      names.push_back(r.name);
  if (i < 0 || i >= static_cast<int>(names.size()) || !name || !total_ms || !launches)
    return fail(E4B_ERR_INVALID_ARGUMENT, "timing index out of range or null output");
  double ms = 0.0;
  int n = 0;
  for (const auto& r : g_timing.recs) {
    if (std::strcmp(r.name, names[i]) != 0) continue;
    cudaError_t err = cudaEventSynchronize(r.stop);
    if (err != cudaSuccess) return cuda_fail(err, "timing event sync");
    float t = 0.f;
    err = cudaEventElapsedTime(&t, r.start, r.stop);
    if (err != cudaSuccess) return cuda_fail(err, "timing elapsed");
    ms += t;
    ++n;
  }
  *name = names[i];
  *total_ms = ms;
  *launches = n;
  return E4B_OK;
}

e4b_status e4b_nf4_quantize_stack(const void* W, e4b_dtype w_dtype, int64_t E, int64_t N, int64_t K,
                                  int blocksize, uint8_t* packed, float* absmax, e4b_stream stream) {
  return e4b_quantize_stack(W, w_dtype, E, N, K, blocksize, E4B_QUANT_NF4, packed, absmax, stream);
}

e4b_status e4b_quantize_stack(const void* W, e4b_dtype w_dtype, int64_t E, int64_t N, int64_t K, int blocksize,
                              e4b_quant_type quant_type, uint8_t* packed, float* absmax, e4b_stream stream) {
  begin_call();
  if (!quant_type_ok(quant_type)) return fail(E4B_ERR_INVALID_ARGUMENT, "quant_type must be NF4 or FP4");
  if (blocksize != 64) return fail(E4B_ERR_UNSUPPORTED, "blocksize must be 64, got " + std::to_string(blocksize));
  if (w_dtype != E4B_F32 && w_dtype != E4B_BF16) return fail(E4B_ERR_INVALID_ARGUMENT, "w_dtype must be F32 or BF16");
  if (E < 1 || N < 1 || K < 1)
    return fail(E4B_ERR_INVALID_ARGUMENT, "E, N, K must be >= 1 (" + shape_str("E", E) + ", " + shape_str("N", N) +
                                              ", " + shape_str("K", K) + ")");
  if ((N * K) % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "N*K must be a multiple of 64 (blocks stay inside an expert)");
  if (!W || !packed || !absmax) return fail(E4B_ERR_INVALID_ARGUMENT, "null pointer (W, packed or absmax)");
  if (!aligned16(W) || !aligned16(packed) || !aligned16(absmax))
    return fail(E4B_ERR_INVALID_ARGUMENT, "W, packed and absmax must be 16-byte aligned");
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  const int64_t nblocks = E * N * K / 64;
  cudaError_t err = launch_quantize(W, w_dtype == E4B_BF16, nblocks, static_cast<int>(quant_type), packed, absmax, stream);
  if (err != cudaSuccess) return cuda_fail(err, "quantize launch");
  set_path("quantize");
  return E4B_OK;
}

size_t e4b_moe_route_permute_workspace_size(int64_t M, int64_t E, int k) {
  if (M < 0 || E < 1 || k < 1) return 0;
  return route_workspace_bytes(M, E, k);
}

e4b_status e4b_moe_route_permute(const float* logits, int64_t M, int64_t E, int k, int renormalize,
                                 int32_t* topk_ids, float* topk_w, int32_t* expert_offsets, int32_t* perm,
                                 int32_t* inv_perm, void* workspace, size_t workspace_bytes, e4b_stream stream) {
  begin_call();
  if (M < 0) return fail(E4B_ERR_INVALID_ARGUMENT, "M must be >= 0");
  if (E < 1 || E > 1024) return fail(E4B_ERR_UNSUPPORTED, "E must be in [1, 1024], got " + std::to_string(E));
  if (k < 1 || k > E || k > 32) return fail(E4B_ERR_INVALID_ARGUMENT, "k must be in [1, min(E, 32)]");
  if (M * k > INT32_MAX) return fail(E4B_ERR_UNSUPPORTED, "M*k exceeds int32 slot indices");
  if (!expert_offsets) return fail(E4B_ERR_INVALID_ARGUMENT, "null expert_offsets");
  if (M > 0 && (!logits || !topk_ids || !topk_w || !perm || !inv_perm))
    return fail(E4B_ERR_INVALID_ARGUMENT, "null pointer (logits, topk_ids, topk_w, perm or inv_perm)");
  if (e4b_status s = check_workspace("route", route_workspace_bytes(M, E, k), workspace, workspace_bytes);
      s != E4B_OK)
    return s;
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  RouteOut o{topk_ids, topk_w, expert_offsets, perm, inv_perm, nullptr};
  cudaError_t err = launch_route(logits, M, static_cast<int>(E), k, renormalize != 0, o, workspace, stream);
  if (err != cudaSuccess) return cuda_fail(err, "route launch");
  if (M == 0) set_path("route.empty");
  return E4B_OK;
}

size_t e4b_grouped_nf4_gemm_workspace_size(int64_t total_rows, int64_t N, int64_t K, int r) {
  (void)N;
  if (total_rows <= 0 || r < 0 || K < 0) return 0;  // no rows: nothing launches, nothing waits
  return gemm_workspace_bytes(total_rows, K, r);
}

e4b_status e4b_grouped_nf4_gemm(const uint16_t* A, int64_t a_rows, int64_t lda, const int32_t* row_index,
                                const int32_t* expert_offsets, int64_t E, int64_t total_rows, const uint8_t* packed,
                                const float* absmax, int64_t N, int64_t K, const uint16_t* lora_A,
                                const uint16_t* lora_B, int r, float lora_scale, e4b_epilogue epi, void* out,
                                e4b_dtype out_dtype, void* workspace, size_t workspace_bytes, e4b_stream stream) {
  return e4b_grouped_4bit_gemm(A, a_rows, lda, row_index, expert_offsets, E, total_rows, packed, absmax,
                               E4B_QUANT_NF4, N, K, lora_A, lora_B, r, lora_scale, epi, out, out_dtype, workspace,
                               workspace_bytes, stream);
}

e4b_status e4b_grouped_4bit_gemm(const uint16_t* A, int64_t a_rows, int64_t lda, const int32_t* row_index,
                                 const int32_t* expert_offsets, int64_t E, int64_t total_rows, const uint8_t* packed,
                                 const float* absmax, e4b_quant_type quant_type, int64_t N, int64_t K,
                                 const uint16_t* lora_A, const uint16_t* lora_B, int r, float lora_scale,
                                 e4b_epilogue epi, void* out, e4b_dtype out_dtype, void* workspace,
                                 size_t workspace_bytes, e4b_stream stream) {
  begin_call();
  if (!quant_type_ok(quant_type)) return fail(E4B_ERR_INVALID_ARGUMENT, "quant_type must be NF4 or FP4");
  if (E < 1 || E > 65536) return fail(E4B_ERR_INVALID_ARGUMENT, "E must be in [1, 65536]");
  if (total_rows < 0 || a_rows < 0) return fail(E4B_ERR_INVALID_ARGUMENT, "total_rows and a_rows must be >= 0");
  if (total_rows > 0 && a_rows < 1) return fail(E4B_ERR_INVALID_ARGUMENT, "a_rows must be >= 1 when rows exist");
  if (K < 64 || K % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "K must be a positive multiple of 64");
  if (N < 64 || N % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "N must be a positive multiple of 64");
  if (lda < K || lda % 8 != 0) return fail(E4B_ERR_INVALID_ARGUMENT, "lda must be >= K and a multiple of 8");
  if (epi != E4B_EPI_NONE && epi != E4B_EPI_SWIGLU) return fail(E4B_ERR_INVALID_ARGUMENT, "unknown epilogue");
  if (out_dtype != E4B_F32 && out_dtype != E4B_BF16) return fail(E4B_ERR_INVALID_ARGUMENT, "out_dtype must be F32 or BF16");
  if ((lora_A == nullptr) != (lora_B == nullptr))
    return fail(E4B_ERR_INVALID_ARGUMENT, "lora_A and lora_B must be both set or both NULL");
  if (lora_A && (r < 1 || r > 16)) return fail(E4B_ERR_UNSUPPORTED, "LoRA rank must be in [1, 16]");
  if (!lora_A) r = 0;
  if (!expert_offsets || !packed || !absmax) return fail(E4B_ERR_INVALID_ARGUMENT, "null expert_offsets, packed or absmax");
  if (total_rows > 0 && (!A || !out)) return fail(E4B_ERR_INVALID_ARGUMENT, "null A or out");
  if (total_rows > INT32_MAX) return fail(E4B_ERR_UNSUPPORTED, "total_rows exceeds int32");
  if ((A && !aligned16(A)) || !aligned16(packed) || (out && !aligned16(out)))
    return fail(E4B_ERR_INVALID_ARGUMENT, "A, packed and out must be 16-byte aligned");
  if (lora_A && (!aligned16(lora_A) || !aligned16(lora_B)))
    return fail(E4B_ERR_INVALID_ARGUMENT, "lora_A and lora_B must be 16-byte aligned");
  if (e4b_status s = check_workspace("gemm", total_rows > 0 ? gemm_workspace_bytes(total_rows, K, r) : 0, workspace,
                                     workspace_bytes);
      s != E4B_OK)
    return s;
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  if (total_rows == 0) {
    set_path("gemm.empty");
    return E4B_OK;
  }
  GemmArgs g{};
  g.A = A;
  g.a_rows = a_rows;
  g.lda = lda;
  g.row_index = row_index;
  g.offsets = expert_offsets;
  g.E = static_cast<int>(E);
  g.total_rows = total_rows;
  g.packed = packed;
  g.absmax = absmax;
  g.quant = quant_type;
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.lora_A = lora_A;
  g.lora_B = lora_B;
  g.r = r;
  g.lora_scale = lora_scale;
  g.err = static_cast<int*>(workspace);
  g.xa = r > 0 ? reinterpret_cast<float*>(static_cast<char*>(workspace) + gemm_workspace_xa_offset()) : nullptr;
  g.a_gathered = row_index ? reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) +
                                                         gemm_workspace_gather_offset(total_rows, r))
                           : nullptr;
  g.epi = epi;
  g.out = out;
  g.out_bf16 = out_dtype == E4B_BF16;
  const char* path = "";
  cudaError_t err = launch_grouped_gemm(g, stream, &path);
  if (err != cudaSuccess) return cuda_fail(err, "grouped gemm launch");
  set_path(path);
  return E4B_OK;
}

size_t e4b_grouped_nf4_gemm_dgrad_workspace_size(int64_t total_rows, int64_t N, int64_t K, int r) {
  (void)N;
  (void)K;
  if (total_rows <= 0 || r < 0 || N < 0) return 0;  // no rows: nothing launches, nothing waits
  return dgrad_workspace_bytes(total_rows, N, r);
}

e4b_status e4b_grouped_nf4_gemm_dgrad(const uint16_t* dY, int64_t dy_rows, int64_t lddy, const int32_t* row_index,
                                      const int32_t* expert_offsets, int64_t E, int64_t total_rows,
                                      const uint8_t* packed, const float* absmax, int64_t N, int64_t K,
                                      const uint16_t* lora_A, const uint16_t* lora_B, int r, float lora_scale,
                                      void* out, e4b_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                      e4b_stream stream) {
  return e4b_grouped_4bit_gemm_dgrad(dY, dy_rows, lddy, row_index, expert_offsets, E, total_rows, packed, absmax,
                                     E4B_QUANT_NF4, N, K, lora_A, lora_B, r, lora_scale, out, out_dtype, workspace,
                                     workspace_bytes, stream);
}

e4b_status e4b_grouped_4bit_gemm_dgrad(const uint16_t* dY, int64_t dy_rows, int64_t lddy, const int32_t* row_index,
                                       const int32_t* expert_offsets, int64_t E, int64_t total_rows,
                                       const uint8_t* packed, const float* absmax, e4b_quant_type quant_type,
                                       int64_t N, int64_t K, const uint16_t* lora_A, const uint16_t* lora_B, int r,
                                       float lora_scale, void* out, e4b_dtype out_dtype, void* workspace,
                                       size_t workspace_bytes, e4b_stream stream) {
  begin_call();
  if (!quant_type_ok(quant_type)) return fail(E4B_ERR_INVALID_ARGUMENT, "quant_type must be NF4 or FP4");
  if (E < 1 || E > 65536) return fail(E4B_ERR_INVALID_ARGUMENT, "E must be in [1, 65536]");
  if (total_rows < 0 || dy_rows < 0) return fail(E4B_ERR_INVALID_ARGUMENT, "total_rows and dy_rows must be >= 0");
  if (total_rows > 0 && dy_rows < 1) return fail(E4B_ERR_INVALID_ARGUMENT, "dy_rows must be >= 1 when rows exist");
  if (K < 64 || K % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "K must be a positive multiple of 64");
  if (N < 64 || N % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "N must be a positive multiple of 64");
  if (lddy < N || lddy % 8 != 0) return fail(E4B_ERR_INVALID_ARGUMENT, "lddy must be >= N and a multiple of 8");
  if (out_dtype != E4B_F32 && out_dtype != E4B_BF16) return fail(E4B_ERR_INVALID_ARGUMENT, "out_dtype must be F32 or BF16");
  if ((lora_A == nullptr) != (lora_B == nullptr))
    return fail(E4B_ERR_INVALID_ARGUMENT, "lora_A and lora_B must be both set or both NULL");
  if (lora_A && (r < 1 || r > 16)) return fail(E4B_ERR_UNSUPPORTED, "LoRA rank must be in [1, 16]");
  if (!lora_A) r = 0;
  if (!expert_offsets || !packed || !absmax) return fail(E4B_ERR_INVALID_ARGUMENT, "null expert_offsets, packed or absmax");
  if (total_rows > 0 && (!dY || !out)) return fail(E4B_ERR_INVALID_ARGUMENT, "null dY or out");
  if (total_rows > INT32_MAX) return fail(E4B_ERR_UNSUPPORTED, "total_rows exceeds int32");
  if ((dY && !aligned16(dY)) || !aligned16(packed) || !aligned16(absmax) || (out && !aligned16(out)))
    return fail(E4B_ERR_INVALID_ARGUMENT, "dY, packed, absmax and out must be 16-byte aligned");
  if (lora_A && (!aligned16(lora_A) || !aligned16(lora_B)))
    return fail(E4B_ERR_INVALID_ARGUMENT, "lora_A and lora_B must be 16-byte aligned");
  if (e4b_status s = check_workspace("dgrad", total_rows > 0 ? dgrad_workspace_bytes(total_rows, N, r) : 0, workspace,
                                     workspace_bytes);
      s != E4B_OK)
    return s;
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  if (total_rows == 0) {
    set_path("dgrad.empty");
    return E4B_OK;
  }
  DgradArgs d{};
  d.dY = dY;
  d.dy_rows = dy_rows;
  d.lddy = lddy;
  d.row_index = row_index;
  d.offsets = expert_offsets;
  d.E = static_cast<int>(E);
  d.total_rows = total_rows;
  d.packed = packed;
  d.absmax = absmax;
  d.quant = quant_type;
  d.N = static_cast<int>(N);
  d.K = static_cast<int>(K);
  d.lora_A = r ? lora_A : nullptr;
  d.lora_B = r ? lora_B : nullptr;
  d.r = r;
  d.lora_scale = lora_scale;
  d.yb = r ? reinterpret_cast<float*>(static_cast<char*>(workspace) + dgrad_workspace_yb_offset()) : nullptr;
  d.gathered = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) + dgrad_workspace_gather_offset(total_rows, r));
  d.err = static_cast<int*>(workspace);
  d.out = out;
  d.out_bf16 = out_dtype == E4B_BF16;
  const char* path = "";
  cudaError_t err = launch_grouped_dgrad(d, reinterpret_cast<cudaStream_t>(stream), &path);
  if (err != cudaSuccess) return cuda_fail(err, "grouped dgrad launch");
  set_path(path);
  return E4B_OK;
}

size_t e4b_grouped_lora_grads_workspace_size(int64_t total_rows, int r) {
  if (total_rows < 0 || r < 1 || r > 16) return 0;
  return lora_grads_workspace_bytes(total_rows, r);
}

e4b_status e4b_grouped_lora_grads(const uint16_t* x, int64_t x_rows, int64_t ldx, const int32_t* row_index,
                                  const int32_t* expert_offsets, int64_t E, int64_t total_rows, const uint16_t* da,
                                  int64_t ldda, int64_t N, int64_t K, const uint16_t* lora_A,
                                  const uint16_t* lora_B, int r, float lora_scale, float* dA, float* dB,
                                  void* workspace, size_t workspace_bytes, e4b_stream stream) {
  begin_call();
  if (E < 1 || E > 65536) return fail(E4B_ERR_INVALID_ARGUMENT, "E must be in [1, 65536]");
  if (total_rows < 0 || x_rows < 0) return fail(E4B_ERR_INVALID_ARGUMENT, "total_rows and x_rows must be >= 0");
  if (total_rows > 0 && x_rows < 1) return fail(E4B_ERR_INVALID_ARGUMENT, "x_rows must be >= 1 when rows exist");
  if (K < 64 || K % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "K must be a positive multiple of 64");
  if (N < 64 || N % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "N must be a positive multiple of 64");
  if (r < 1 || r > 16) return fail(E4B_ERR_UNSUPPORTED, "LoRA rank must be in [1, 16]");
  if (ldx < K || ldx % 8 != 0) return fail(E4B_ERR_INVALID_ARGUMENT, "ldx must be >= K and a multiple of 8");
  if (ldda < N) return fail(E4B_ERR_INVALID_ARGUMENT, "ldda must be >= N");
  if (!expert_offsets || !lora_A || !lora_B || !dA || !dB)
    return fail(E4B_ERR_INVALID_ARGUMENT, "null expert_offsets, lora_A, lora_B, dA or dB");
  if (total_rows > 0 && (!x || !da)) return fail(E4B_ERR_INVALID_ARGUMENT, "null x or da");
  if (total_rows > INT32_MAX) return fail(E4B_ERR_UNSUPPORTED, "total_rows exceeds int32");
  if ((x && !aligned16(x)) || !aligned16(lora_A) || !aligned16(lora_B) || !aligned16(dA) || !aligned16(dB) ||
      (da && !aligned16(da)))
    return fail(E4B_ERR_INVALID_ARGUMENT, "x, da, lora_A, lora_B, dA and dB must be 16-byte aligned");
  if (e4b_status s = check_workspace("lora grads", lora_grads_workspace_bytes(total_rows, r), workspace,
                                     workspace_bytes);
      s != E4B_OK)
    return s;
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* xa = reinterpret_cast<float*>(static_cast<char*>(workspace) + 256);
  float* yb = reinterpret_cast<float*>(static_cast<char*>(workspace) + lora_grads_workspace_yb_offset(total_rows, r));
  if (total_rows > 0) {
    GemmArgs g{};
    g.A = x;
    g.a_rows = x_rows;
    g.lda = ldx;
    g.row_index = row_index;
    g.offsets = expert_offsets;
    g.E = static_cast<int>(E);
    g.total_rows = total_rows;
    g.N = static_cast<int>(N);
    g.K = static_cast<int>(K);
    g.lora_A = lora_A;
    g.lora_B = lora_B;
    g.r = r;
    g.xa = xa;
    cudaError_t err = launch_lora_xa(g, st);
    if (err != cudaSuccess) return cuda_fail(err, "lora grads: x . A^T");
    DgradArgs d{};
    d.dY = da;
    d.dy_rows = total_rows;
    d.lddy = ldda;
    d.offsets = expert_offsets;
    d.E = static_cast<int>(E);
    d.total_rows = total_rows;
    d.N = static_cast<int>(N);
    d.K = static_cast<int>(K);
    d.lora_B = lora_B;
    d.r = r;
    d.yb = yb;
    err = launch_dgrad_lora_yb(d, st);
    if (err != cudaSuccess) return cuda_fail(err, "lora grads: da . B");
  }
  LoraGradArgs a{};
  a.x = x;
  a.x_rows = x_rows;
  a.ldx = ldx;
  a.row_index = row_index;
  a.offsets = expert_offsets;
  a.E = static_cast<int>(E);
  a.total_rows = total_rows;
  a.da = da;
  a.ldda = ldda;
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.r = r;
  a.lora_scale = lora_scale;
  a.xa = xa;
  a.yb = yb;
  a.dA = dA;
  a.dB = dB;
  cudaError_t err = launch_lora_grads(a, st);
  if (err != cudaSuccess) return cuda_fail(err, "lora grads launch");
  set_path("lora_grads");
  return E4B_OK;
}

size_t e4b_grouped_mxfp4_gemm_workspace_size(int64_t total_rows, int64_t N, int64_t K) {
  (void)N;
  if (total_rows <= 0 || K < 0) return 0;  // no rows: nothing launches, nothing waits
  return gemm_workspace_bytes(total_rows, K, 0);
}

e4b_status e4b_grouped_mxfp4_gemm(const uint16_t* A, int64_t a_rows, int64_t lda, const int32_t* row_index,
                                  const int32_t* expert_offsets, int64_t E, int64_t total_rows,
                                  const uint8_t* blocks, const uint8_t* scales, int64_t N, int64_t K,
                                  e4b_epilogue epi, void* out, e4b_dtype out_dtype, void* workspace,
                                  size_t workspace_bytes, e4b_stream stream) {
  begin_call();
  if (E < 1 || E > 65536) return fail(E4B_ERR_INVALID_ARGUMENT, "E must be in [1, 65536]");
  if (total_rows < 0 || a_rows < 0) return fail(E4B_ERR_INVALID_ARGUMENT, "total_rows and a_rows must be >= 0");
  if (total_rows > 0 && a_rows < 1) return fail(E4B_ERR_INVALID_ARGUMENT, "a_rows must be >= 1 when rows exist");
  if (K < 64 || K % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "K must be a positive multiple of 64");
  if (N < 64 || N % 64 != 0) return fail(E4B_ERR_UNSUPPORTED, "N must be a positive multiple of 64");
  if (lda < K || lda % 8 != 0) return fail(E4B_ERR_INVALID_ARGUMENT, "lda must be >= K and a multiple of 8");
  if (epi != E4B_EPI_NONE && epi != E4B_EPI_SWIGLU) return fail(E4B_ERR_INVALID_ARGUMENT, "unknown epilogue");
  if (out_dtype != E4B_F32 && out_dtype != E4B_BF16) return fail(E4B_ERR_INVALID_ARGUMENT, "out_dtype must be F32 or BF16");
  if (!expert_offsets || !blocks || !scales) return fail(E4B_ERR_INVALID_ARGUMENT, "null expert_offsets, blocks or scales");
  if (total_rows > 0 && (!A || !out)) return fail(E4B_ERR_INVALID_ARGUMENT, "null A or out");
  if (total_rows > INT32_MAX) return fail(E4B_ERR_UNSUPPORTED, "total_rows exceeds int32");
  if ((A && !aligned16(A)) || !aligned16(blocks) || (out && !aligned16(out)))
    return fail(E4B_ERR_INVALID_ARGUMENT, "A, blocks and out must be 16-byte aligned");
  if (e4b_status s = check_workspace("mxfp4 gemm", total_rows > 0 ? gemm_workspace_bytes(total_rows, K, 0) : 0,
                                     workspace, workspace_bytes);
      s != E4B_OK)
    return s;
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  if (total_rows == 0) {
    set_path("mxfp4.empty");
    return E4B_OK;
  }
  Mxfp4Args m{};
  m.A = A;
  m.a_rows = a_rows;
  m.lda = lda;
  m.row_index = row_index;
  m.offsets = expert_offsets;
  m.E = static_cast<int>(E);
  m.total_rows = total_rows;
  m.blocks = blocks;
  m.scales = scales;
  m.N = static_cast<int>(N);
  m.K = static_cast<int>(K);
  m.epi = epi;
  m.out = out;
  m.out_bf16 = out_dtype == E4B_BF16;
  GemmArgs g{};
  g.A = A;
  g.a_rows = a_rows;
  g.lda = lda;
  g.row_index = row_index;
  g.offsets = expert_offsets;
  g.E = static_cast<int>(E);
  g.total_rows = total_rows;
  g.packed = blocks;
  g.mx_scales = scales;
  g.quant = kQuantMxfp4;
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.err = static_cast<int*>(workspace);
  g.a_gathered = row_index ? reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) +
                                                         gemm_workspace_gather_offset(total_rows, 0))
                           : nullptr;
  g.epi = epi;
  g.out = out;
  g.out_bf16 = out_dtype == E4B_BF16;
  const char* path = "";
  cudaError_t err = launch_grouped_mxfp4(g, m, reinterpret_cast<cudaStream_t>(stream), &path);
  if (err != cudaSuccess) return cuda_fail(err, "grouped mxfp4 gemm launch");
  set_path(path);
  return E4B_OK;
}

static int stack_r(const e4b_expert_stack* w) { return w->lora_A ? w->lora_r : 0; }

size_t e4b_moe_expert_forward_workspace_size(int64_t M, const e4b_expert_stack* w, int k) {
  if (!w || M <= 0 || k < 1) return 0;
  const size_t g = grouped_layout(M, w->E, w->H, w->I, k, stack_r(w)).total;
  const size_t d = decode_workspace_bytes(M, w->E, k, w->H, w->I, stack_r(w));
  return g > d ? g : d;
}

static e4b_status forward_grouped(const uint16_t* x, int64_t M, const float* logits, int k, int renormalize,
                                  const e4b_expert_stack* w, uint16_t* out, void* ws, cudaStream_t stream) {
  const int r = stack_r(w);
  const GroupedLayout L = grouped_layout(M, w->E, w->H, w->I, k, r);
  RouteOut o{at<int32_t>(ws, L.ids), at<float>(ws, L.w), at<int32_t>(ws, L.offsets),
             at<int32_t>(ws, L.perm), at<int32_t>(ws, L.inv), at<int32_t>(ws, L.row_token)};
  cudaError_t err = launch_route(logits, M, static_cast<int>(w->E), k, renormalize != 0, o,
                                 at<void>(ws, L.route_ws), stream);
  if (err != cudaSuccess) return cuda_fail(err, "route launch");
  const int64_t S = M * k;
  GemmArgs g{};
  g.A = x;
  g.a_rows = M;
  g.lda = w->H;
  g.row_index = o.row_token;
  g.offsets = o.offsets;
  g.E = static_cast<int>(w->E);
  g.total_rows = S;
  g.packed = w->gu_packed;
  g.absmax = w->gu_absmax;
  g.quant = w->quant_type;
  g.N = static_cast<int>(2 * w->I);
  g.K = static_cast<int>(w->H);
  g.lora_A = r ? w->lora_A : nullptr;
  g.lora_B = r ? w->lora_B : nullptr;
  g.r = r;
  g.lora_scale = r ? w->lora_alpha / static_cast<float>(r) : 0.0f;
  g.xa = r ? at<float>(ws, L.xa) : nullptr;
  g.a_gathered = at<uint16_t>(ws, L.xg);
  g.err = at<int>(ws, L.err);
  g.epi = E4B_EPI_SWIGLU;
  g.out = at<uint16_t>(ws, L.h);
  g.out_bf16 = true;
  const char* p1 = "";
  if ((err = launch_grouped_gemm(g, stream, &p1)) != cudaSuccess) return cuda_fail(err, "gate_up gemm launch");
  GemmArgs d{};
  d.A = at<uint16_t>(ws, L.h);
  d.a_rows = S;
  d.lda = w->I;
  d.row_index = nullptr;
  d.offsets = o.offsets;
  d.E = static_cast<int>(w->E);
  d.total_rows = S;
  d.packed = w->dn_packed;
  d.absmax = w->dn_absmax;
  d.quant = w->quant_type;
  d.N = static_cast<int>(w->H);
  d.K = static_cast<int>(w->I);
  d.err = at<int>(ws, L.err);
  d.epi = E4B_EPI_NONE;
  d.out = at<uint16_t>(ws, L.z);
  d.out_bf16 = true;  // per-slot expert outputs in bf16 (the combine sums them in fp32)
  const char* p2 = "";
  if ((err = launch_grouped_gemm(d, stream, &p2)) != cudaSuccess) return cuda_fail(err, "down gemm launch");
  if ((err = launch_combine(at<uint16_t>(ws, L.z), o.inv, o.w, M, k, static_cast<int>(w->H), out, stream)) != cudaSuccess)
    return cuda_fail(err, "combine launch");
  set_path("forward.grouped");
  return E4B_OK;
}

e4b_status e4b_moe_expert_forward_path(const uint16_t* x, int64_t M, const float* router_logits, int k,
                                       int renormalize, const e4b_expert_stack* w, uint16_t* out, void* workspace,
                                       size_t workspace_bytes, e4b_path path, e4b_stream stream) {
  begin_call();
  if (e4b_status s = check_stack(w, k); s != E4B_OK) return s;
  if (M < 0) return fail(E4B_ERR_INVALID_ARGUMENT, "M must be >= 0");
  if (M * k > INT32_MAX) return fail(E4B_ERR_UNSUPPORTED, "M*k exceeds int32 slot indices");
  if (M > 0 && (!x || !router_logits || !out)) return fail(E4B_ERR_INVALID_ARGUMENT, "null x, router_logits or out");
  if (M > 0 && (!aligned16(x) || !aligned16(out))) return fail(E4B_ERR_INVALID_ARGUMENT, "x and out must be 16-byte aligned");
  if (path != E4B_PATH_AUTO && path != E4B_PATH_DECODE && path != E4B_PATH_GROUPED)
    return fail(E4B_ERR_INVALID_ARGUMENT, "unknown path");
  if (e4b_status s = check_workspace("forward", e4b_moe_expert_forward_workspace_size(M, w, k), workspace,
                                     workspace_bytes);
      s != E4B_OK)
    return s;
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  if (M == 0) {
    set_path("forward.empty");
    return E4B_OK;
  }
  const std::string dec_why = decode_unsupported_reason(M, w->E, k, w->H, w->I);
  const bool dec_ok = dec_why.empty();
  if (path == E4B_PATH_DECODE && !dec_ok) return fail(E4B_ERR_UNSUPPORTED, dec_why);
  if (path == E4B_PATH_DECODE || (path == E4B_PATH_AUTO && dec_ok)) {
    DecodeArgs a{x, M, router_logits, k, renormalize != 0, w, out, workspace};
    cudaError_t err = launch_decode_forward(a, stream);
    if (err != cudaSuccess) return cuda_fail(err, "decode forward launch");
    set_path("forward.decode");
    return E4B_OK;
  }
  return forward_grouped(x, M, router_logits, k, renormalize, w, out, workspace, stream);
}

e4b_status e4b_moe_expert_forward(const uint16_t* x, int64_t M, const float* router_logits, int k, int renormalize,
                                  const e4b_expert_stack* w, uint16_t* out, void* workspace, size_t workspace_bytes,
                                  e4b_stream stream) {
  return e4b_moe_expert_forward_path(x, M, router_logits, k, renormalize, w, out, workspace, workspace_bytes,
                                     E4B_PATH_AUTO, stream);
}

size_t e4b_moe_expert_backward_workspace_size(int64_t M, const e4b_expert_stack* w, int k) {
  if (!w || M <= 0 || k < 1 || w->E < 1 || w->H < 1 || w->I < 1) return 0;
  return backward_layout(M, w->E, w->H, w->I, k, stack_r(w)).total;
}

e4b_status e4b_moe_expert_backward(const uint16_t* x, int64_t M, const float* router_logits, int k, int renormalize,
                                   const e4b_expert_stack* w, const uint16_t* dout, float* dx, float* dlogits,
                                   float* dA, float* dB, void* workspace, size_t workspace_bytes,
                                   e4b_stream stream) {
  begin_call();
  if (e4b_status s = check_stack(w, k); s != E4B_OK) return s;
  if (M < 0) return fail(E4B_ERR_INVALID_ARGUMENT, "M must be >= 0");
  if (M * k > INT32_MAX) return fail(E4B_ERR_UNSUPPORTED, "M*k exceeds int32 slot indices");
  if (M > 0 && (!x || !router_logits || !dout || !dx || !dlogits))
    return fail(E4B_ERR_INVALID_ARGUMENT, "null x, router_logits, dout, dx or dlogits");
  const int r = stack_r(w);
  if (r > 0 && (!dA || !dB)) return fail(E4B_ERR_INVALID_ARGUMENT, "a stack with an adapter needs dA and dB");
  if (M > 0 && (!aligned16(x) || !aligned16(dout) || !aligned16(dx) || !aligned16(dlogits) ||
                (dA && !aligned16(dA)) || (dB && !aligned16(dB))))
    return fail(E4B_ERR_INVALID_ARGUMENT, "x, dout, dx, dlogits, dA and dB must be 16-byte aligned");
  if (e4b_status s = check_workspace("backward", e4b_moe_expert_backward_workspace_size(M, w, k), workspace,
                                     workspace_bytes);
      s != E4B_OK)
    return s;
  if (e4b_status s = check_device(); s != E4B_OK) return s;
  const cudaStream_t stream_ = reinterpret_cast<cudaStream_t>(stream);
  if (M == 0) {
    if (r > 0) {  // no rows: the adapter gradients are zero
      cudaError_t err = cudaMemsetAsync(dA, 0, static_cast<size_t>(w->E) * r * w->H * sizeof(float), stream_);
      if (err == cudaSuccess)
        err = cudaMemsetAsync(dB, 0, static_cast<size_t>(w->E) * 2 * w->I * r * sizeof(float), stream_);
      if (err != cudaSuccess) return cuda_fail(err, "backward: zero adapter gradients");
    }
    set_path("backward.empty");
    return E4B_OK;
  }
  void* ws = workspace;
  const BackwardLayout L = backward_layout(M, w->E, w->H, w->I, k, r);
  const int64_t S = M * k;
  const int E = static_cast<int>(w->E), H = static_cast<int>(w->H), I = static_cast<int>(w->I);
  const float scale = r ? w->lora_alpha / static_cast<float>(r) : 0.0f;
  RouteOut o{at<int32_t>(ws, L.ids), at<float>(ws, L.w), at<int32_t>(ws, L.offsets),
             at<int32_t>(ws, L.perm), at<int32_t>(ws, L.inv), at<int32_t>(ws, L.row_token)};
  cudaError_t err = launch_route(router_logits, M, E, k, renormalize != 0, o, at<void>(ws, L.route_ws), stream_);
  if (err != cudaSuccess) return cuda_fail(err, "backward: route");
  // Recompute a = [g | u] (fp32) and z (fp32) per grouped row.
  GemmArgs g{};
  g.A = x;
  g.a_rows = M;
  g.lda = H;
  g.row_index = o.row_token;
  g.offsets = o.offsets;
  g.E = E;
  g.total_rows = S;
  g.packed = w->gu_packed;
  g.absmax = w->gu_absmax;
  g.quant = w->quant_type;
  g.N = 2 * I;
  g.K = H;
  g.lora_A = r ? w->lora_A : nullptr;
  g.lora_B = r ? w->lora_B : nullptr;
  g.r = r;
  g.lora_scale = scale;
  g.xa = r ? at<float>(ws, L.xa) : nullptr;
  g.a_gathered = at<uint16_t>(ws, L.xg);
  g.err = at<int>(ws, L.err);
  g.epi = E4B_EPI_NONE;
  g.out = at<float>(ws, L.a);
  g.out_bf16 = false;
  const char* path = "";
  if ((err = launch_grouped_gemm(g, stream_, &path)) != cudaSuccess) return cuda_fail(err, "backward: gate_up gemm");
  if ((err = launch_swiglu_h(at<float>(ws, L.a), S, I, at<uint16_t>(ws, L.h), stream_)) != cudaSuccess)
    return cuda_fail(err, "backward: swiglu");
  GemmArgs d{};
  d.A = at<uint16_t>(ws, L.h);
  d.a_rows = S;
  d.lda = I;
  d.offsets = o.offsets;
  d.E = E;
  d.total_rows = S;
  d.packed = w->dn_packed;
  d.absmax = w->dn_absmax;
  d.quant = w->quant_type;
  d.N = H;
  d.K = I;
  d.err = at<int>(ws, L.err);
  d.epi = E4B_EPI_NONE;
  d.out = at<float>(ws, L.z);
  d.out_bf16 = false;
  if ((err = launch_grouped_gemm(d, stream_, &path)) != cudaSuccess) return cuda_fail(err, "backward: down gemm");
  // dz = w * dout per grouped row, dw = dout . z per slot
  if ((err = launch_slot_grads(dout, at<float>(ws, L.z), o.perm, o.row_token, o.w, S, M, H, at<uint16_t>(ws, L.dz),
                               at<float>(ws, L.dw), stream_)) != cudaSuccess)
    return cuda_fail(err, "backward: slot gradients");
  // dh = dz . Wd (dgrad through down), da by the SwiGLU derivative
  DgradArgs dd{};
  dd.dY = at<uint16_t>(ws, L.dz);
  dd.dy_rows = S;
  dd.lddy = H;
  dd.offsets = o.offsets;
  dd.E = E;
  dd.total_rows = S;
  dd.packed = w->dn_packed;
  dd.absmax = w->dn_absmax;
  dd.quant = w->quant_type;
  dd.N = H;
  dd.K = I;
  dd.out = at<float>(ws, L.dh);
  dd.out_bf16 = false;
  dd.err = at<int>(ws, L.err);
  if ((err = launch_grouped_dgrad(dd, stream_, &path)) != cudaSuccess) return cuda_fail(err, "backward: dgrad down");
  if ((err = launch_swiglu_bwd(at<float>(ws, L.a), at<float>(ws, L.dh), S, I, at<uint16_t>(ws, L.da), stream_)) !=
      cudaSuccess)
    return cuda_fail(err, "backward: swiglu derivative");
  // dx per grouped row through gate_up (with the adapter's share), then per token
  DgradArgs dg{};
  dg.dY = at<uint16_t>(ws, L.da);
  dg.dy_rows = S;
  dg.lddy = 2 * I;
  dg.offsets = o.offsets;
  dg.E = E;
  dg.total_rows = S;
  dg.packed = w->gu_packed;
  dg.absmax = w->gu_absmax;
  dg.quant = w->quant_type;
  dg.N = 2 * I;
  dg.K = H;
  dg.lora_A = r ? w->lora_A : nullptr;
  dg.lora_B = r ? w->lora_B : nullptr;
  dg.r = r;
  dg.lora_scale = scale;
  dg.yb = r ? at<float>(ws, L.yb) : nullptr;
  dg.out = at<float>(ws, L.dxg);
  dg.out_bf16 = false;
  dg.err = at<int>(ws, L.err);
  if ((err = launch_grouped_dgrad(dg, stream_, &path)) != cudaSuccess) return cuda_fail(err, "backward: dgrad gate_up");
  if ((err = launch_token_sum(at<float>(ws, L.dxg), o.inv, M, k, H, dx, stream_)) != cudaSuccess)
    return cuda_fail(err, "backward: token sum");
  if ((err = launch_router_grad(router_logits, o.ids, o.w, at<float>(ws, L.dw), M, E, k, renormalize != 0, dlogits,
                                stream_)) != cudaSuccess)
    return cuda_fail(err, "backward: router gradient");
  if (r > 0) {
    // adapter gradients of gate_up: xa = x . A^T here, yb = da . B from the
    // gate_up dgrad above, then the per-group sums
    GemmArgs gx = g;
    gx.xa = at<float>(ws, L.lg_xa);
    if ((err = launch_lora_xa(gx, stream_)) != cudaSuccess) return cuda_fail(err, "backward: x . A^T");
    LoraGradArgs la{};
    la.x = x;
    la.x_rows = M;
    la.ldx = H;
    la.row_index = o.row_token;
    la.offsets = o.offsets;
    la.E = E;
    la.total_rows = S;
    la.da = at<uint16_t>(ws, L.da);
    la.ldda = 2 * I;
    la.N = 2 * I;
    la.K = H;
    la.r = r;
    la.lora_scale = scale;
    la.xa = at<float>(ws, L.lg_xa);
    la.yb = at<float>(ws, L.yb);
    la.dA = dA;
    la.dB = dB;
    if ((err = launch_lora_grads(la, stream_)) != cudaSuccess) return cuda_fail(err, "backward: adapter gradients");
  }
  set_path("backward.grouped");
  return E4B_OK;
}

}  // extern "C"
