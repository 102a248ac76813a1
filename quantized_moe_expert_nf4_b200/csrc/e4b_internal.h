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

// Host-side argument checks shared by the C-ABI entry points; on failure they
// record the message (e4b_last_error) and return the status.
e4b_status check_stack(const e4b_expert_stack* w, int k);  // stack pointers, shapes, alignment, LoRA rank, k
e4b_status check_sm100();                                 // the current device is sm_100

// The codebooks as the library holds them, indexed by e4b_quant_type: NF4
// (QLoRA table, ascending) and FP4 (e2m1 / 6, in code order).
extern const float kCodebooks[2][16];

// Quantiser tables of one storage type.  The distinct codebook values in
// ascending order are the levels; T[l] is the smallest float strictly above
// the exact midpoint of levels l and l+1, so that for any float s,
// s > midpoint  <=>  s >= T[l]; the unused tail of T is +inf.  The level of s
// is the number of thresholds <= s; code[level] is the code written for it
// (the lowest code holding that value); zero_code is written for an all-zero
// block.
struct QuantTables {
  float t[16];
  uint32_t code[16];
  uint32_t zero_code;
};
QuantTables quant_tables(int quant);

// The quantiser kernel's lookup of a level: 128 cells of width 1/64 over s in
// [-1, 1], each widened by kQuantCellSlack on both sides.  Cell c holds the one
// decision threshold inside it (+inf if none; both codebooks' thresholds are
// at least 0.079 apart, wider than a cell) and the codes written below and at
// or above it.  Any s in the widened cell gets its code from one comparison.
constexpr int kQuantCells = 128;
constexpr double kQuantCellSlack = 1e-5;
struct QuantCellTable {
  uint2 cell[kQuantCells];  // x: threshold (float bits), y: code below | code at or above << 4
  uint32_t zero_code;
  int ok;                   // 0 if some widened cell held two thresholds
};
QuantCellTable quant_cell_table(int quant);

cudaError_t launch_quantize(const void* W, bool bf16, int64_t nblocks, int quant, uint8_t* packed,
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
// Internal storage index of MXFP4 weights on the tensor-core kernel: e2m1 codes
// (element 2i in the low nibble) with one e8m0 scale byte per 32 elements of a
// row instead of an fp32 absmax per 64 (not an e4b_quant_type).
constexpr int kQuantMxfp4 = 2;

struct GemmArgs {
  const uint16_t* A;
  int64_t a_rows, lda;
  const int32_t* row_index;  // nullable
  const int32_t* offsets;    // [E+1]
  int E;
  int64_t total_rows;
  const uint8_t* packed;
  const float* absmax;       // [E, N*K/64] (NF4, FP4)
  const uint8_t* mx_scales;  // [E, N*K/32] e8m0 (quant == kQuantMxfp4; tensor-core kernel only)
  int quant;  // e4b_quant_type of packed, or kQuantMxfp4
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

// ---- grouped dgrad ---------------------------------------------------------
struct DgradArgs {
  const uint16_t* dY;
  int64_t dy_rows, lddy;
  const int32_t* row_index;  // nullable
  const int32_t* offsets;    // [E+1]
  int E;
  int64_t total_rows;
  const uint8_t* packed;
  const float* absmax;
  int quant;  // e4b_quant_type of packed
  int N, K;
  const uint16_t* lora_A;  // [E, r, K] or nullptr
  const uint16_t* lora_B;  // [E, N, r] or nullptr
  int r;
  float lora_scale;
  float* yb;  // workspace [total_rows, r] fp32: dY . lora_B
  uint16_t* gathered;  // workspace [total_rows, N] bf16: dY rows in group order (tensor-core path)
  int* err;            // workspace error word
  void* out;  // [total_rows, K]
  bool out_bf16;
};
// Workspace: [error word, 256 B][dY . lora_B, total_rows * r fp32][dY rows gathered,
// total_rows * N bf16], parts 256-B aligned.
size_t dgrad_workspace_bytes(int64_t total_rows, int64_t N, int r);
size_t dgrad_workspace_yb_offset();
size_t dgrad_workspace_gather_offset(int64_t total_rows, int r);
// Warp-MMA kernel below 512 routed rows (and with an adapter and bf16 output),
// the tensor-core kernel otherwise; E4B_DGRAD=mma|tc forces one.
cudaError_t launch_grouped_dgrad(const DgradArgs& a, cudaStream_t stream, const char** path);
bool dgrad_tc_supported(const DgradArgs& a, int64_t lddy);
cudaError_t launch_grouped_dgrad_tc(const DgradArgs& a, const uint16_t* dy, int64_t dy_rows, int64_t lddy,
                                    int* err_word, cudaStream_t stream);
// yb = dY . lora_B per routed row (into a.yb); a.lora_B, a.r, a.N, a.dY, a.lddy used.
cudaError_t launch_dgrad_lora_yb(const DgradArgs& a, cudaStream_t stream);

// ---- grouped LoRA gradients ---------------------------------------------------
struct LoraGradArgs {
  const uint16_t* x;  // input rows of the projection (gathered by row_index)
  int64_t x_rows, ldx;
  const int32_t* row_index;  // nullable
  const int32_t* offsets;    // [E+1]
  int E;
  int64_t total_rows;
  const uint16_t* da;  // [total_rows, ldda] gradient of the projection's output rows
  int64_t ldda;
  int N, K, r;
  float lora_scale;
  const float* xa;  // [total_rows, r] x . A_e^T
  const float* yb;  // [total_rows, r] da . B_e
  float* dA;        // [E, r, K]
  float* dB;        // [E, N, r]
};
// Workspace: [error word, 256 B][xa, total_rows * r fp32][yb, total_rows * r fp32], 256-B aligned parts.
size_t lora_grads_workspace_bytes(int64_t total_rows, int r);
size_t lora_grads_workspace_yb_offset(int64_t total_rows, int r);
cudaError_t launch_lora_grads(const LoraGradArgs& a, cudaStream_t stream);

// ---- layer backward steps (csrc/backward.cu) -------------------------------------
cudaError_t launch_swiglu_h(const float* a, int64_t S, int I, uint16_t* h, cudaStream_t stream);
cudaError_t launch_slot_grads(const uint16_t* dout, const float* z, const int32_t* perm, const int32_t* row_token,
                              const float* w, int64_t S, int64_t M, int H, uint16_t* dz, float* dw,
                              cudaStream_t stream);
cudaError_t launch_swiglu_bwd(const float* a, const float* dh, int64_t S, int I, uint16_t* da, cudaStream_t stream);
cudaError_t launch_token_sum(const float* dxg, const int32_t* inv, int64_t M, int k, int H, float* dx,
                             cudaStream_t stream);
cudaError_t launch_router_grad(const float* logits, const int32_t* ids, const float* w, const float* dw, int64_t M,
                               int E, int k, bool renormalize, float* dlogits, cudaStream_t stream);

// ---- grouped MXFP4 GEMM -------------------------------------------------------
struct Mxfp4Args {
  const uint16_t* A;
  int64_t a_rows, lda;
  const int32_t* row_index;  // nullable
  const int32_t* offsets;    // [E+1]
  int E;
  int64_t total_rows;
  const uint8_t* blocks;  // [E, N*K/2] e2m1 codes, element 2i in the low nibble
  const uint8_t* scales;  // [E, N*K/32] e8m0
  int N, K;
  int epi;
  void* out;
  bool out_bf16;
};
cudaError_t launch_grouped_mxfp4_gemm(const Mxfp4Args& a, cudaStream_t stream);
// Picks the kernel for an MXFP4 call as launch_grouped_gemm does for NF4 (the
// tensor-core kernel from 512 routed rows, E4B_GEMM=mma|tc forces one): `a`
// describes it for the tensor-core kernel (quant kQuantMxfp4, mx_scales, error
// word and gather room in the workspace), `m` for the warp-MMA kernel.
cudaError_t launch_grouped_mxfp4(const GemmArgs& a, const Mxfp4Args& m, cudaStream_t stream, const char** path);

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
