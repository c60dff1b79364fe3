// Allocation-free entry point of the In-Place W_down update.
//
// Some callers cannot hand the library a workspace: host runtimes that plan every device buffer
// before they start serving and refuse allocations afterwards, and plugin interfaces that pass
// only input and output pointers. This entry point serves them: its scratch (the two bf16
// copies of the running W_down and the per-chunk tile counters) lives in a fixed-size static
// device array that is part of the library image. Every GPU that loads the library holds the
// array until the process exits; all calls share it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "internal.h"
#include "ttt.h"

namespace ttt {
namespace {

constexpr size_t kNoAllocScratchBytes = 32ull << 20;  // 32 MiB

__device__ __align__(256) unsigned char g_inplace_scratch[kNoAllocScratchBytes];

// Device address of the scratch array, looked up once per device and context (host code must
// not use the array's name as a device pointer). The context's unique id is kept beside the
// address: after a device reset the device gets a new primary context, with the array at an
// address of its own, and the lookup is made again.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct ScratchSlot {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;
};
std::mutex g_scratch_mu;
constexpr int kMaxDevices = 256;
ScratchSlot g_scratch[kMaxDevices];

// Id of the calling thread's current context, 0 when there is none or the driver cannot say.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

int scratch_address(void** out, std::string* msg) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *msg = std::string("cudaGetDevice: ") + cudaGetErrorString(e);
    return TTT_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *msg = "device number " + std::to_string(dev) + " is beyond the " +
           std::to_string(kMaxDevices) + " devices this entry point keeps scratch addresses for";
    return TTT_ERR_UNSUPPORTED;
  }
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  if (!slot.addr || id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_inplace_scratch);
    if (e != cudaSuccess || !p) {
      *msg = std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e);
      return TTT_ERR_CUDA;
    }
    slot.addr = p;
    slot.ctx_id = current_context_id();  // the lookup made the primary context current
  }
  *out = slot.addr;
  return TTT_OK;
}

}  // namespace
}  // namespace ttt

extern "C" {

size_t inplace_ttt_noalloc_max_scratch_bytes(void) { return ttt::kNoAllocScratchBytes; }

int inplace_ttt_chunk_fwd_noalloc(const void* Z, const void* Vhat, const void* W0, float eta,
                                  void* O, float* W_out, int T, int Dff, int D, int C,
                                  cudaStream_t stream) {
  if (T > 0 && Dff > 0 && D > 0 && C > 0 && T % C == 0) {
    const size_t need = inplace_ttt_workspace_size(T, Dff, D, C);
    if (need > ttt::kNoAllocScratchBytes) {
      ttt::set_last_error("inplace_ttt_chunk_fwd_noalloc: this shape needs " +
                          std::to_string(need) + " bytes of scratch, more than the " +
                          std::to_string(ttt::kNoAllocScratchBytes) +
                          " bytes built into the library; use inplace_ttt_chunk_fwd with a "
                          "caller-provided workspace");
      return TTT_ERR_UNSUPPORTED;
    }
  }
  void* scratch = nullptr;
  std::string msg;
  const int st = ttt::scratch_address(&scratch, &msg);
  if (st != TTT_OK) {
    ttt::set_last_error("inplace_ttt_chunk_fwd_noalloc: " + msg);
    return st;
  }
  // Same validation and kernels as the workspace entry point; the scratch array is the
  // workspace. The tile counters in it are zeroed on the stream at the start of every call.
  const int rc = inplace_ttt_chunk_fwd(Z, Vhat, W0, eta, O, W_out, T, Dff, D, C, scratch,
                                      ttt::kNoAllocScratchBytes, stream);
  if (rc != TTT_OK)  // name the function the caller used in the message
    ttt::set_last_error(std::string("inplace_ttt_chunk_fwd_noalloc: ") + ttt_last_error_message());
  return rc;
}

}  // extern "C"
