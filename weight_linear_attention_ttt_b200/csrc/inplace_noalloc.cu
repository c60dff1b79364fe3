// Allocation-free entry point of the In-Place W_down update.
//
// Some callers cannot hand the library a workspace: host runtimes that plan every device buffer
// before they start serving and refuse allocations afterwards, and plugin interfaces that pass
// only input and output pointers. This entry point serves them: its scratch (the two bf16
// copies of the running W_down and the per-chunk tile counters) lives in a fixed-size static
// device array that is part of the library image. Every GPU that loads the library holds the
// array until the process exits; all calls share it.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "internal.h"
#include "ttt.h"

namespace ttt {
namespace {

constexpr size_t kNoAllocScratchBytes = 32ull << 20;  // 32 MiB

__device__ __align__(256) unsigned char g_inplace_scratch[kNoAllocScratchBytes];

// Device address of the scratch array, looked up once per device (host code must not use the
// array's name as a device pointer).
std::mutex g_scratch_mu;
void* g_scratch_addr[256] = {};

int scratch_address(void** out, std::string* msg) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 256) {
    *msg = std::string("cudaGetDevice: ") + cudaGetErrorString(e);
    return TTT_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_inplace_scratch);
    if (e != cudaSuccess || !p) {
      *msg = std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e);
      return TTT_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
  return inplace_ttt_chunk_fwd(Z, Vhat, W0, eta, O, W_out, T, Dff, D, C, scratch,
                               ttt::kNoAllocScratchBytes, stream);
}

}  // extern "C"
