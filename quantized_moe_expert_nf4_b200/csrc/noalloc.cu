// Small-batch layer forward that needs no device allocation and no workspace.
//
// Some hosts cannot hand this library scratch memory: serving engines that
// carve every byte of device memory out of a fixed pool planned at start-up,
// and runtimes that forbid any allocator call (cudaMalloc included) once the
// decode loop is running.  For them this file keeps the decode path's scratch
// -- the SwiGLU activations h of the routed slots and the slots of the decode
// kernel's grid barrier -- in a statically sized device array that exists from
// the moment the library is loaded on a GPU until the process exits.  The caller still passes x, the
// router logits, the packed stacks and the output buffer.
#include <cuda.h>

#include <mutex>
#include <string>
#include <vector>

#include "e4b_internal.h"

namespace e4b {
namespace {

// h holds M*k*I bf16 values; the limit below allows e.g. M=8, k=8, I=4096.
constexpr int64_t kNoAllocMaxHElems = 256 * 1024;
constexpr size_t kNoAllocHBytes = static_cast<size_t>(kNoAllocMaxHElems) * 2;
constexpr size_t kNoAllocBytes = kNoAllocHBytes + 16 * 1024;  // + the error word and the grid-barrier slots

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of the scratch array in the current context.  The host-side
// name of the array is not a device address.  The address belongs to the
// module instance of one CUDA context: after cudaDeviceReset, or with another
// context current on the same device, the module is loaded again and the
// array may sit elsewhere, so the cache is keyed by the context's unique id
// (cuCtxGetId), never by the device index alone.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct ScratchEntry {
  unsigned long long ctx_id;
  void* addr;
};

std::mutex g_mu;
std::vector<ScratchEntry> g_scratch;

template <class Fn>
Fn driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &ptr, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(ptr);
}

cudaError_t scratch_address(void** out) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return cudaErrorNotSupported;
  cudaError_t err = cudaSuccess;
  void* p = nullptr;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  if (!ctx) {
    // No context on this thread yet: the runtime's symbol lookup makes the
    // device's primary context current (and loads the module).
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  std::lock_guard<std::mutex> lk(g_mu);
  for (const ScratchEntry& e : g_scratch)
    if (e.ctx_id == id) {
      *out = e.addr;
      return cudaSuccess;
    }
  err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (err != cudaSuccess) return err;
  g_scratch.push_back({id, p});
  *out = p;
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
  if (e4b_status st = check_stack(w, k); st != E4B_OK) return st;
  if (M < 1 || M > 8) return nofail(E4B_ERR_UNSUPPORTED, "the allocation-free forward takes 1 to 8 tokens");
  if (M * k * w->I > kNoAllocMaxHElems)
    return nofail(E4B_ERR_UNSUPPORTED, "M*k*I = " + std::to_string(M * k * w->I) +
                                           " exceeds the static scratch of the allocation-free forward (" +
                                           std::to_string(kNoAllocMaxHElems) + " activations)");
  if (!x || !router_logits || !out) return nofail(E4B_ERR_INVALID_ARGUMENT, "null x, router_logits or out");
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(x) || !a16(out)) return nofail(E4B_ERR_INVALID_ARGUMENT, "x and out must be 16-byte aligned");
  if (e4b_status st = check_sm100(); st != E4B_OK) return st;
  if (const std::string why = decode_unsupported_reason(M, w->E, k, w->H, w->I); !why.empty())
    return nofail(E4B_ERR_UNSUPPORTED, why);
  if (decode_workspace_bytes(M, w->E, k, w->H, w->I, w->lora_A ? w->lora_r : 0) > kNoAllocBytes)
    return nofail(E4B_ERR_UNSUPPORTED, "decode scratch layout exceeds the static array");
  void* scratch = nullptr;
  cudaError_t err = scratch_address(&scratch);
  if (err != cudaSuccess)
    return nofail(E4B_ERR_CUDA, std::string("cudaGetSymbolAddress of the static scratch: ") + cudaGetErrorString(err));
  DecodeArgs a{x, M, router_logits, k, renormalize != 0, w, out, scratch};
  err = launch_decode_forward(a, reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return nofail(E4B_ERR_CUDA, std::string("decode forward launch: ") + cudaGetErrorString(err));
  set_path("forward.decode.noalloc");
  return E4B_OK;
}
