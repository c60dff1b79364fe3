// LM-aligned target for the In-Place W_down update.
//
// Source: "In-Place 테스트 시점 학습: LLM을 위한 원활한 동적 적응 프레임워크", LM-aligned objective
// paragraph: the target Vhat is made from the token embeddings by a 1D convolution and a
// projection, so that it carries the next token's information. Reading (the page gives it in
// words): a depthwise convolution over tokens whose tap i multiplies token t + 1 - i (the next
// token, the current one and k - 2 before it; zeros outside the sequence), then a bias-free
// projection:
//     U[t, j] = sum_i Wc[i, j] X[t + 1 - i, j],     Vhat = U Wp.
// The convolution is a memory-bound pass (one bf16 write of U); the projection runs on the
// tcgen05 read tiles of the In-Place kernel.
#include <cuda_bf16.h>

#include <algorithm>
#include <string>

#include "internal.h"

namespace ttt {
namespace {

constexpr int KMAX = 8;      // taps supported
constexpr int ROWS = 64;     // tokens per thread block row

__device__ __forceinline__ void bf16x8_to_f(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Thread = eight consecutive channels of ROWS consecutive tokens.
__global__ void lm_conv_kernel(const uint4* __restrict__ X, const float* __restrict__ Wc,
                               uint4* __restrict__ U, int T, int Dm, int k) {
  const int c8 = blockIdx.x * blockDim.x + threadIdx.x;   // channel group
  const int ng = Dm / 8;
  if (c8 >= ng) return;
  float w[KMAX][8];
#pragma unroll
  for (int i = 0; i < KMAX; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) w[i][e] = i < k ? Wc[(size_t)i * Dm + 8 * c8 + e] : 0.f;
  const int t0 = blockIdx.y * ROWS;
  for (int t = t0; t < min(T, t0 + ROWS); ++t) {
    float acc[8] = {};
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      const int src = t + 1 - i;
      if (i < k && src >= 0 && src < T) {
        float x[8];
        bf16x8_to_f(X[(size_t)src * ng + c8], x);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += w[i][e] * x[e];
      }
    }
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
      ow[e] = *reinterpret_cast<const uint32_t*>(&v);
    }
    U[(size_t)t * ng + c8] = o;
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t lm_target_workspace_bytes(int T, int Dm, int D, int k) {
  (void)D;
  (void)k;
  return align256((size_t)T * Dm * 2) + 256;
}

int launch_lm_target(const void* X, const float* Wc, const void* Wp, void* Vhat, int T, int Dm,
                     int D, int k, void* ws, size_t ws_bytes, const LaunchCtx& ctx) {
  if (ws_bytes < lm_target_workspace_bytes(T, Dm, D, k)) {
    *ctx.msg = "lm target: workspace too small";
    return kWorkspace;
  }
  void* U = ws;
  int* counter = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + align256((size_t)T * Dm * 2));
  const dim3 grid((Dm / 8 + 127) / 128, (T + ROWS - 1) / ROWS);
  lm_conv_kernel<<<grid, 128, 0, ctx.stream>>>(static_cast<const uint4*>(X), Wc,
                                               static_cast<uint4*>(U), T, Dm, k);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("lm conv launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return launch_projection(U, Wp, Vhat, T, Dm, D, counter, ctx);
}

}  // namespace ttt
