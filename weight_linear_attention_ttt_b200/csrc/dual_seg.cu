// Sequence-parallel dual form: the segment-affine scan.
//
// Without weight normalisation the dual form's chunk update is affine in the state
// ("KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다", associativity paragraph, applied
// to the update of "Learning to (Learn at Test Time)", mini-batch section):
//     W' = (I - K_c^T diag(eta_c) K_c) W + K_c^T diag(eta_c) V_c,
// so a segment of chunks maps its start state to its end state by W_end = A_s W_start + B_s, and
// maps compose. The sequence of each stream is cut into S segments of L = T / S tokens, which
// the dual-form kernels run as B*H*S independent streams (the tensors are viewed as
// [B*H*S, 1, L, d]; nothing is copied):
//   1. B_s: the segment run from W = 0 (its end state);
//   2. A_s + B_s: the segment run from W = I;
//   3. fold, per stream and in segment order, in fp32: W_start(s+1) = A_s W_start(s) + B_s;
//   4. every segment run from W_start(s), writing O; the last segment's end state is W_out.
// Passes 1 and 2 write O as scratch (pass 4 overwrites it). The work is three dual-form passes
// instead of one, spread over S times as many chains: it pays when B*H leaves most SMs idle.
#include <algorithm>

#include "internal.h"

namespace ttt {
namespace {

__global__ void identity_states_kernel(float* __restrict__ W, size_t n, int d) {
  const size_t total = n * d * d;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(i % ((size_t)d * d));
    W[i] = (e / d == e % d) ? 1.f : 0.f;
  }
}

// One CTA per stream: W (fp32, d x d) and A_s = (A_s + B_s) - B_s in shared memory; segment s
// stores its start state, then W <- A_s W + B_s. Each thread owns d*d/256 outputs.
template <int D>
__global__ void __launch_bounds__(256) fold_segments_kernel(const float* __restrict__ W0,
                                                            const float* __restrict__ Bm,
                                                            const float* __restrict__ ABm,
                                                            float* __restrict__ Wstart, int S) {
  constexpr int E = D * D / 256;   // outputs per thread
  extern __shared__ float fsm[];
  float* W = fsm;                  // [D][D]
  float* A = fsm + D * D;          // [D][D]
  const size_t bh = blockIdx.x;
  for (int i = threadIdx.x; i < D * D; i += 256) W[i] = W0 ? W0[bh * D * D + i] : 0.f;
  __syncthreads();
  for (int s = 0; s < S; ++s) {
    const size_t seg = (bh * S + s) * D * D;
    for (int i = threadIdx.x; i < D * D; i += 256) {
      Wstart[seg + i] = W[i];
      A[i] = ABm[seg + i] - Bm[seg + i];
    }
    __syncthreads();
    float out[E];
#pragma unroll
    for (int q = 0; q < E; ++q) {
      const int idx = threadIdx.x + 256 * q, i = idx / D, j = idx % D;
      float acc = Bm[seg + idx];
#pragma unroll 8
      for (int k = 0; k < D; ++k) acc = fmaf(A[i * D + k], W[k * D + j], acc);
      out[q] = acc;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < E; ++q) W[threadIdx.x + 256 * q] = out[q];
    __syncthreads();
  }
}

__global__ void last_segment_state_kernel(const float* __restrict__ Wend, float* W_out, int S,
                                          int d, size_t bh_count) {
  const size_t per = (size_t)d * d, total = bh_count * per;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = i / per, e = i % per;
    W_out[i] = Wend[(bh * S + (S - 1)) * per + e];
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

int dual_seg_choose_segments(int B, int H, int T, int C, int requested) {
  const int nchunks = T / C;
  if (requested > 0) return (nchunks % requested == 0) ? requested : -1;
  // automatic: the most segments that keep one chain per SM; fewer than four segments do not
  // repay the two extra passes, so that case runs the sequential kernel (S = 1)
  const int bh = B * H, sms = sm_count();
  int best = 1;
  for (int s = 2; s <= nchunks && (long)bh * s <= sms; ++s)
    if (nchunks % s == 0) best = s;
  return best >= 4 ? best : 1;
}

size_t dual_seg_workspace_bytes(int B, int H, int d, int S) {
  if (S <= 1) return 0;
  // identity starts, B maps, A + B maps, segment start states, segment end states
  return 5 * (size_t)B * H * S * d * d * sizeof(float);
}

int launch_dual_seg(const StateArgs& a, int S, const LaunchCtx& ctx) {
  auto run = [&](const StateArgs& x) {
    return dual_mma_supported(x.d, x.C, x.dt) ? launch_dual_mma(x, ctx) : launch_dual_simt(x, ctx);
  };
  if (S <= 1) return run(a);
  const int d = a.d, bh = a.B * a.H;
  const size_t n = (size_t)bh * S, per = (size_t)d * d;
  if (a.ws_bytes < dual_seg_workspace_bytes(a.B, a.H, d, S)) {
    *ctx.msg = "ttt_linear_dual_seg_fwd: workspace smaller than ttt_linear_dual_seg_workspace_size()";
    return kWorkspace;
  }
  float* ws = static_cast<float*>(a.ws);
  float* Wid = ws;
  float* Bm = Wid + n * per;
  float* ABm = Bm + n * per;
  float* Wst = ABm + n * per;
  float* Wend = Wst + n * per;
  const int sms = sm_count();

  identity_states_kernel<<<sms * 4, 256, 0, ctx.stream>>>(Wid, n, d);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual seg identity launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  // segments as independent streams: [B*H*S, 1, T/S, d]
  StateArgs v = a;
  v.B = (int)n;
  v.H = 1;
  v.T = a.T / S;
  v.ws = nullptr;
  v.ws_bytes = 0;
  StateArgs pb = v;   // 1. from W = 0
  pb.S0 = nullptr;
  pb.S_out = Bm;
  int st = run(pb);
  if (st != kOk) return st;
  StateArgs pa = v;   // 2. from W = I
  pa.S0 = Wid;
  pa.S_out = ABm;
  st = run(pa);
  if (st != kOk) return st;
  // 3. fold
  const size_t smem = 2 * per * sizeof(float);
  if (d == 32) {
    fold_segments_kernel<32><<<bh, 256, smem, ctx.stream>>>(a.S0, Bm, ABm, Wst, S);
  } else if (d == 64) {
    fold_segments_kernel<64><<<bh, 256, smem, ctx.stream>>>(a.S0, Bm, ABm, Wst, S);
  } else if (d == 128) {
    e = cudaFuncSetAttribute(fold_segments_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      fold_segments_kernel<128><<<bh, 256, smem, ctx.stream>>>(a.S0, Bm, ABm, Wst, S);
  } else {
    *ctx.msg = "ttt_linear_dual_seg_fwd: unsupported head dim";
    return kUnsupported;
  }
  count_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual seg fold launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  // 4. outputs from the true segment starts
  StateArgs po = v;
  po.S0 = Wst;
  po.S_out = Wend;
  st = run(po);
  if (st != kOk) return st;
  last_segment_state_kernel<<<sms * 2, 256, 0, ctx.stream>>>(Wend, a.S_out, S, d, (size_t)bh);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual seg state launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  return kOk;
}

}  // namespace ttt
