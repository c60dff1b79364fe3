// Prefix combination of per-slice state increments for context parallelism: a device that owns
// sequence slice r starts from S0 + (increments of slices 0 .. r-1), and the state after the
// whole sequence is S0 + (all increments) ("In-Place 테스트 시점 학습", associative-scan paragraph:
// per-chunk deltas combined by a prefix sum give the sequential result).
#include "internal.h"
#include "ttt.h"

namespace ttt {
namespace {

__global__ void state_prefix_kernel(const float* __restrict__ S0, const float* __restrict__ inc,
                                    int upto, size_t n_state, float* __restrict__ out) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_state) return;
  float acc = S0 ? S0[i] : 0.f;
  for (int r = 0; r < upto; ++r) acc += inc[(size_t)r * n_state + i];
  out[i] = acc;
}

}  // namespace
}  // namespace ttt

extern "C" int ttt_state_prefix_sum(const float* S0, const float* increments, int n_increments,
                                    int upto, int B, int H, int d, float* out,
                                    cudaStream_t stream) {
  if (!increments || !out || n_increments <= 0 || upto < 0 || upto > n_increments || B <= 0 ||
      H <= 0 || d <= 0) {
    ttt::set_last_error("ttt_state_prefix_sum: null pointer or bad sizes");
    return TTT_ERR_INVALID_ARG;
  }
  const size_t n = (size_t)B * H * d * d;
  const uintptr_t o = reinterpret_cast<uintptr_t>(out);
  const uintptr_t lo = reinterpret_cast<uintptr_t>(increments);
  if (o < lo + n * n_increments * 4 && lo < o + n * 4) {
    ttt::set_last_error("ttt_state_prefix_sum: out must not overlap the increments");
    return TTT_ERR_INVALID_ARG;
  }
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  ttt::state_prefix_kernel<<<blocks, threads, 0, stream>>>(S0, increments, upto, n, out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    ttt::set_last_error(std::string("ttt_state_prefix_sum launch: ") + cudaGetErrorString(e));
    return TTT_ERR_CUDA;
  }
  ttt::count_launch();
  return TTT_OK;
}
