// Small-batch layer forward that needs no device allocation and no workspace.
//
// Some hosts cannot hand this library scratch memory: serving engines that
// carve every byte of device memory out of a fixed pool planned at start-up,
// and runtimes that forbid any allocator call (cudaMalloc included) once the
// decode loop is running.  For them this file keeps the decode path's scratch
// -- the SwiGLU activations h of the routed slots and the kernels' error word
// -- in a
// statically sized device array that exists from the moment the library is
// loaded on a GPU until the process exits.  The caller still passes x, the
// router logits, the packed stacks and the output buffer.
#include <mutex>
#include <string>

#include "e4b_internal.h"

namespace e4b {
namespace {

// h holds M*k*I bf16 values; the limit below allows e.g. M=8, k=8, I=4096.
constexpr int64_t kNoAllocMaxHElems = 256 * 1024;
constexpr size_t kNoAllocHBytes = static_cast<size_t>(kNoAllocMaxHElems) * 2;
constexpr size_t kNoAllocBytes = kNoAllocHBytes + 16 * 1024;  // + the error word and the routing the kernels share

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device.  The host-side name of the array is not a device address.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

e4b_status nofail(e4b_status s, const std::string& msg) {
  set_error(msg);
  return s;
}

}  // namespace
}  // namespace e4b

using namespace e4b;

extern "C" e4b_status e4b_moe_expert_forward_decode_noalloc(const uint16_t* x, int64_t M, const float* router_logits,
                                                            int k, int renormalize, const e4b_expert_stack* w,
                                                            uint16_t* out, e4b_stream stream) {
  begin_call();
  if (!w) return nofail(E4B_ERR_INVALID_ARGUMENT, "null expert stack");
  if (M < 1 || M > 8) return nofail(E4B_ERR_UNSUPPORTED, "the allocation-free forward takes 1 to 8 tokens");
  if (k < 1 || k > 32 || k > w->E) return nofail(E4B_ERR_INVALID_ARGUMENT, "k must be in [1, min(E, 32)]");
  if (w->E < 1 || w->H < 64 || w->H % 64 != 0 || w->I < 64 || w->I % 64 != 0)
    return nofail(E4B_ERR_UNSUPPORTED, "E >= 1 and H, I positive multiples of 64 required");
  if (M * k * w->I > kNoAllocMaxHElems)
    return nofail(E4B_ERR_UNSUPPORTED, "M*k*I = " + std::to_string(M * k * w->I) +
                                           " exceeds the static scratch of the allocation-free forward (" +
                                           std::to_string(kNoAllocMaxHElems) + " activations)");
  if (!x || !router_logits || !out || !w->gu_packed || !w->gu_absmax || !w->dn_packed || !w->dn_absmax)
    return nofail(E4B_ERR_INVALID_ARGUMENT, "null pointer argument");
  if ((w->lora_A == nullptr) != (w->lora_B == nullptr))
    return nofail(E4B_ERR_INVALID_ARGUMENT, "lora_A and lora_B must be both set or both NULL");
  if (w->lora_A && (w->lora_r < 1 || w->lora_r > 16)) return nofail(E4B_ERR_UNSUPPORTED, "LoRA rank must be in [1, 16]");
  if (w->quant_type != E4B_QUANT_NF4 && w->quant_type != E4B_QUANT_FP4)
    return nofail(E4B_ERR_INVALID_ARGUMENT, "quant_type must be NF4 or FP4");
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(x) || !a16(out) || !a16(w->gu_packed) || !a16(w->dn_packed) || !a16(w->gu_absmax) || !a16(w->dn_absmax))
    return nofail(E4B_ERR_INVALID_ARGUMENT, "x, out, packed stacks and absmax must be 16-byte aligned");
  if (w->lora_A && (!a16(w->lora_A) || !a16(w->lora_B)))
    return nofail(E4B_ERR_INVALID_ARGUMENT, "lora_A and lora_B must be 16-byte aligned");
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return nofail(E4B_ERR_CUDA, std::string("device query: ") + cudaGetErrorString(err));
  if (di.major != 10 || di.minor != 0) return nofail(E4B_ERR_UNSUPPORTED, "libe4b is built for sm_100a (B200)");
  if (const std::string why = decode_unsupported_reason(M, w->E, k, w->H, w->I); !why.empty())
    return nofail(E4B_ERR_UNSUPPORTED, why);
  if (decode_workspace_bytes(M, w->E, k, w->H, w->I, w->lora_A ? w->lora_r : 0) > kNoAllocBytes)
    return nofail(E4B_ERR_UNSUPPORTED, "decode scratch layout exceeds the static array");
  void* scratch = nullptr;
  err = scratch_address(&scratch);
  if (err != cudaSuccess)
    return nofail(E4B_ERR_CUDA, std::string("cudaGetSymbolAddress of the static scratch: ") + cudaGetErrorString(err));
  DecodeArgs a{x, M, router_logits, k, renormalize != 0, w, out, scratch};
  err = launch_decode_forward(a, reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return nofail(E4B_ERR_CUDA, std::string("decode forward launch: ") + cudaGetErrorString(err));
  set_path("forward.decode.noalloc");
  return E4B_OK;
}
