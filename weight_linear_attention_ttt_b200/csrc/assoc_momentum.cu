// Associative mode with a momentum inner loop: the dispatch between the one-pass form
// (assoc_mom.cu, the default) and the two-pass form below (tuning key "momentum_form" = 1, kept
// for comparison; beta in [0.25, 0.9]).
//
// Two-pass form. Source: "KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다", momentum paragraph: with
// momentum SGD the inner loop is still a weighted sum of linear-attention terms. Per stream,
//     M_t = beta M_(t-1) + eta_t k_t^T v_t,   S_t = S_(t-1) + M_t,   o_t = q_t S_t.
// Summing the momentum terms, with A_t = sum_{s<=t} eta_s k_s^T v_s (the plain associative
// state) and M_t the momentum itself,
//     S_t = S0 + (beta M0 + A_t - beta M_t) / (1 - beta),
// so the layer is one plain associative pass with rates eta / (1 - beta) from
// S0 + beta M0 / (1 - beta), then one decayed pass (the chunk kernel's decay mode) that forms
// q_t M_t and M_T and writes O = O_plain - beta / (1 - beta) q_t M_t in its epilogue (the
// decayed output is not rounded before the subtraction); S_T = S_plain - beta / (1 - beta) M_T
// elementwise.
#include <cuda_bf16.h>

#include <algorithm>
#include <string>

#include "internal.h"

namespace ttt {
namespace {

// out = (a ? a : 0) + c * b over n fp32 elements
__global__ void axpy_states_kernel(const float* a, const float* __restrict__ b, float c,
                                   float* out, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    out[i] = (a ? a[i] : 0.f) + c * b[i];
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t assoc_momentum_split_workspace_bytes(int B, int H, int T, int d, int C) {
  const size_t BH = (size_t)B * H;
  return align256(assoc_workspace_bytes(B, H, T, d, C)) + BH * d * d * sizeof(float);
}

// Enough for either form, so that a size queried before a form is chosen stays valid.
size_t assoc_momentum_workspace_bytes(int B, int H, int T, int d, int C) {
  return std::max(assoc_momentum_split_workspace_bytes(B, H, T, d, C),
                  assoc_momentum_fused_workspace_bytes(B, H, T, d, C));
}

int launch_assoc_momentum(const AssocMomentumArgs& a, const LaunchCtx& ctx) {
  return tuning(kTuneMomentumForm) == 1 ? launch_assoc_momentum_split(a, ctx)
                                         : launch_assoc_momentum_fused(a, ctx);
}

int launch_assoc_momentum_split(const AssocMomentumArgs& a, const LaunchCtx& ctx) {
  const size_t BH = (size_t)a.B * a.H, d = a.d;
  const size_t fwd = align256(assoc_workspace_bytes(a.B, a.H, a.T, a.d, a.C));
  if (a.ws_bytes < fwd + BH * d * d * sizeof(float)) {
    *ctx.msg = "ttt_assoc_momentum_fwd: workspace smaller than "
               "ttt_assoc_momentum_workspace_size()";
    return kWorkspace;
  }
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  float* S0p = reinterpret_cast<float*>(ws + fwd);
  const float inv = 1.f / (1.f - a.beta), c = -a.beta * inv;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const float* start = a.S0;
  if (a.M0) {   // S0 + beta M0 / (1 - beta)
    axpy_states_kernel<<<sms * 4, 256, 0, ctx.stream>>>(a.S0, a.M0, a.beta * inv, S0p,
                                                        BH * d * d);
    count_launch();
    start = S0p;
  }
  StateArgs plain{a.Q, a.K, a.V, a.eta, a.eta_scalar, start, a.O, a.S_out, a.B, a.H, a.T,
                  a.d, a.C, 1, a.ws, fwd};
  plain.eta_mul = inv;
  int r = launch_assoc(plain, ctx);
  if (r != kOk) return r;
  StateArgs decay{a.Q, a.K, a.V, a.eta, a.eta_scalar, a.M0, a.O, a.M_out, a.B, a.H, a.T, a.d,
                  a.C, 1, a.ws, fwd};
  decay.decay = 1;
  decay.beta = a.beta;
  decay.Oadd = a.O;         // read back, combined and rewritten row by row in the epilogue
  decay.add_scale = c;
  r = launch_assoc(decay, ctx);
  if (r != kOk) return r;
  axpy_states_kernel<<<sms * 4, 256, 0, ctx.stream>>>(a.S_out, a.M_out, c, a.S_out, BH * d * d);
  count_launch();
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("assoc momentum launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  return kOk;
}

}  // namespace ttt
