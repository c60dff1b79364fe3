// TTT-Linear mini-batch dual form on CUDA cores, exact fp32 arithmetic (no TF32).
//
// Serves fp32 inputs (where the tolerance is too tight for tensor-core bf16/TF32 operands) and
// any chunk size 1 <= C <= 64 the tensor-core path does not take. One CTA per (batch, head)
// stream keeps W (d x d fp32) in shared memory for the whole sequence. Per chunk (source:
// "Learning to (Learn at Test Time)" reading, mini-batch TTT / dual-form section):
//     G   = K_c W - V_c
//     A   = tril(Q_c K_c^T) diag(eta_c)            (diagonal included)
//     O_c = Q_c W - A G
//     W   = W - K_c^T diag(eta_c) G
#include <cuda_bf16.h>

#include "internal.h"

namespace ttt {
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

constexpr int kSimtThreads = 256;

template <typename TIn, int D>
__global__ void __launch_bounds__(kSimtThreads)
    dual_simt_kernel(const TIn* __restrict__ Q, const TIn* __restrict__ K,
                     const TIn* __restrict__ V, const float* __restrict__ eta, float eta_scalar,
                     const float* W0, TIn* __restrict__ O, float* Wout, int T, int C) {
  extern __shared__ float sm[];
  float* W = sm;                 // [D][D]
  float* Qs = W + D * D;         // [C][D]
  float* Ks = Qs + C * D;        // [C][D]
  float* Vs = Ks + C * D;        // [C][D]
  float* Gs = Vs + C * D;        // [C][D]
  float* As = Gs + C * D;        // [C][C]
  float* es = As + C * C;        // [C]
  const int stream = blockIdx.x;
  const int tid = threadIdx.x;
  const size_t base = (size_t)stream * T * D;

  for (int i = tid; i < D * D; i += kSimtThreads)
    W[i] = W0 ? W0[(size_t)stream * D * D + i] : 0.f;
  __syncthreads();

  for (int c0 = 0; c0 < T; c0 += C) {
    for (int i = tid; i < C * D; i += kSimtThreads) {
      const size_t gi = base + (size_t)c0 * D + i;
      Qs[i] = to_f(Q[gi]);
      Ks[i] = to_f(K[gi]);
      Vs[i] = to_f(V[gi]);
    }
    for (int i = tid; i < C; i += kSimtThreads)
      es[i] = eta ? eta[(size_t)stream * T + c0 + i] : eta_scalar;
    __syncthreads();
    // G = K W - V
    for (int idx = tid; idx < C * D; idx += kSimtThreads) {
      const int s = idx / D, j = idx % D;
      float acc = 0.f;
      for (int i = 0; i < D; ++i) acc = fmaf(Ks[s * D + i], W[i * D + j], acc);
      Gs[idx] = acc - Vs[idx];
    }
    // A = tril(Q K^T) diag(eta)
    for (int idx = tid; idx < C * C; idx += kSimtThreads) {
      const int t = idx / C, s = idx % C;
      float acc = 0.f;
      if (s <= t) {
        for (int i = 0; i < D; ++i) acc = fmaf(Qs[t * D + i], Ks[s * D + i], acc);
        acc *= es[s];
      }
      As[idx] = acc;
    }
    __syncthreads();
    // O = Q W - A G
    for (int idx = tid; idx < C * D; idx += kSimtThreads) {
      const int t = idx / D, j = idx % D;
      float acc = 0.f;
      for (int i = 0; i < D; ++i) acc = fmaf(Qs[t * D + i], W[i * D + j], acc);
      float corr = 0.f;
      for (int s = 0; s <= t; ++s) corr = fmaf(As[t * C + s], Gs[s * D + j], corr);
      O[base + (size_t)(c0 + t) * D + j] = from_f<TIn>(acc - corr);
    }
    __syncthreads();
    // W -= K^T diag(eta) G
    for (int idx = tid; idx < D * D; idx += kSimtThreads) {
      const int i = idx / D, j = idx % D;
      float acc = 0.f;
      for (int s = 0; s < C; ++s) acc = fmaf(Ks[s * D + i] * es[s], Gs[s * D + j], acc);
      W[idx] -= acc;
    }
    __syncthreads();
  }
  for (int i = tid; i < D * D; i += kSimtThreads) Wout[(size_t)stream * D * D + i] = W[i];
}

template <typename TIn, int D>
int launch_t(const StateArgs& a, const LaunchCtx& ctx) {
  const size_t smem = sizeof(float) * ((size_t)D * D + 4ull * a.C * D + (size_t)a.C * a.C + a.C);
  auto kern = dual_simt_kernel<TIn, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  kern<<<a.B * a.H, kSimtThreads, smem, ctx.stream>>>(
      static_cast<const TIn*>(a.Q), static_cast<const TIn*>(a.K), static_cast<const TIn*>(a.V),
      a.eta, a.eta_scalar, a.S0, static_cast<TIn*>(a.O), a.S_out, a.T, a.C);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual_simt launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

template <typename TIn>
int launch_d(const StateArgs& a, const LaunchCtx& ctx) {
  switch (a.d) {
    case 32: return launch_t<TIn, 32>(a, ctx);
    case 64: return launch_t<TIn, 64>(a, ctx);
    case 128: return launch_t<TIn, 128>(a, ctx);
  }
  *ctx.msg = "dual_simt: unsupported head dim";
  return kUnsupported;
}

}  // namespace

int launch_dual_simt(const StateArgs& a, const LaunchCtx& ctx) {
  return a.dt == 0 ? launch_d<float>(a, ctx) : launch_d<__nv_bfloat16>(a, ctx);
}

}  // namespace ttt
