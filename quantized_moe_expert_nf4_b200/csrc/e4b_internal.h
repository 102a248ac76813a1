// Internal declarations shared by the translation units of libe4b.
// Host-side launchers only; each kernel lives in its own .cu file.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "e4b.h"

namespace e4b {

// Per-thread error / path reporting (set by the C-ABI layer).
void set_error(const std::string& msg);
void set_path(const char* path);

// Every kernel launch of the library is wrapped in a LaunchScope: it counts the
// launches of the current call and, while kernel timing is enabled on this
// thread, brackets the launch with CUDA events recorded on its stream.
class LaunchScope {
 public:
  LaunchScope(const char* name, cudaStream_t stream);
  ~LaunchScope();
  LaunchScope(const LaunchScope&) = delete;
  LaunchScope& operator=(const LaunchScope&) = delete;

 private:
  int rec_;
  cudaStream_t stream_;
};
void begin_call();  // resets the per-call launch counter

// The NF4 codebook as the library holds it (QLoRA table, ascending).
extern const float kNf4Codebook[16];

// Quantiser decision thresholds: T[c] is the smallest float strictly above
// the exact midpoint (cb[c] + cb[c+1]) / 2, so that for any float s,
// s > midpoint  <=>  s >= T[c].  T[15] = +inf.
struct Nf4Thresholds {
  float t[16];
};
Nf4Thresholds nf4_thresholds();

cudaError_t launch_quantize(const void* W, bool bf16, int64_t nblocks, uint8_t* packed,
                            float* absmax, cudaStream_t stream);

// ---- routing -------------------------------------------------------------
struct RouteOut {
  int32_t* ids;        // [M, k]
  float* w;            // [M, k]
  int32_t* offsets;    // [E+1]
  int32_t* perm;       // [S]
  int32_t* inv;        // [S]
  int32_t* row_token;  // [S] perm[p] / k, or nullptr
};
size_t route_workspace_bytes(int64_t M, int64_t E, int k);
cudaError_t launch_route(const float* logits, int64_t M, int E, int k, bool renormalize,
                         const RouteOut& o, void* workspace, cudaStream_t stream);
// out[p, :] = A[row_index[p], :K] for p < S (the routed rows, contiguous).
cudaError_t launch_gather_rows(const uint16_t* A, int64_t a_rows, int64_t lda, const int32_t* row_index, int64_t S,
                               int K, uint16_t* out, cudaStream_t stream);

// ---- grouped GEMM --------------------------------------------------------
struct GemmArgs {
  const uint16_t* A;
  int64_t a_rows, lda;
  const int32_t* row_index;  // nullable
  const int32_t* offsets;    // [E+1]
  int E;
  int64_t total_rows;
  const uint8_t* packed;
  const float* absmax;
  int N, K;
  const uint16_t* lora_A;  // [E, r, K] or nullptr
  const uint16_t* lora_B;  // [E, N, r] or nullptr
  int r;
  float lora_scale;
  float* xa;  // workspace LoRA products: [total_rows, r] fp32 (warp-MMA path) or [total_rows, 64] bf16 (tensor cores)
  uint16_t* a_gathered;  // workspace [total_rows, K]: routed rows gathered for the tensor-core kernel
  int* err;   // workspace error word of the tensor-core kernel's bounded waits
  int epi;    // e4b_epilogue
  void* out;
  bool out_bf16;
};
// Workspace: [error word, 256 B][LoRA x.A^T, 128 B per row, 256-B aligned]
// [gathered rows, total_rows * K bf16].
size_t gemm_workspace_bytes(int64_t total_rows, int64_t K, int r);
size_t gemm_workspace_xa_offset();
size_t gemm_workspace_gather_offset(int64_t total_rows, int r);
bool tc_supported(const GemmArgs& a);
cudaError_t launch_grouped_gemm_tc(const GemmArgs& a, int* err_word, cudaStream_t stream);
// Gathers the routed rows (when a.row_index is set) and writes the LoRA
// products the tensor-core kernel reads: xa as [total_rows, 64] bf16,
// scale * x . lora_A^T, zero past r.
cudaError_t launch_tc_lora_prep(const GemmArgs& a, cudaStream_t stream);
// Picks the implementation; reports the path name through set_path.
cudaError_t launch_grouped_gemm(const GemmArgs& a, cudaStream_t stream, const char** path);

// ---- combine ---------------------------------------------------------------
cudaError_t launch_combine(const uint16_t* z, const int32_t* inv, const float* w, int64_t M, int k,
                           int H, uint16_t* out, cudaStream_t stream);

// ---- fused small-M forward ---------------------------------------------------
struct DecodeArgs {
  const uint16_t* x;
  int64_t M;
  const float* logits;
  int k;
  bool renormalize;
  const e4b_expert_stack* w;
  uint16_t* out;
  void* workspace;
};
bool decode_supported(int64_t M, int64_t E, int k, int64_t H, int64_t I);
// Why the decode kernels cannot take this shape ("" when they can).
std::string decode_unsupported_reason(int64_t M, int64_t E, int k, int64_t H, int64_t I);
size_t decode_workspace_bytes(int64_t M, int64_t E, int k, int64_t H, int64_t I, int r);
cudaError_t launch_decode_forward(const DecodeArgs& a, cudaStream_t stream);

// Device properties cached per device.
struct DeviceInfo {
  int device;
  int sm_count;
  int major, minor;
  size_t smem_optin;
};
cudaError_t device_info(DeviceInfo* out);

// Raises `func`'s dynamic shared-memory limit on the current device to at least
// `bytes`.  The attribute belongs to one function on one device; it is only ever
// raised, under a lock, so a call needing less never lowers what another relies on.
cudaError_t ensure_smem_limit(const void* func, size_t bytes);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace e4b
