// Backward pass of the associative (gradient-ascent linear-attention) mode.
//
// Forward, per stream (source: "KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다",
// one inner step with a linear bias-free last layer; associativity paragraph):
//     S_t = S_(t-1) + eta_t k_t^T v_t,   o_t = q_t S_t.
// Gradients of L = sum_t <dO_t, o_t> + <dS_out, S_T>, with A_t = dS_out + sum_{u >= t} q_u^T dO_u
// the gradient with respect to S_t:
//     dq_t   = dO_t S_t^T          = dO_t S0^T + sum_{s <= t} eta_s (dO_t . v_s) k_s
//     Y_t    = k_t A_t             = k_t dS_out + sum_{u >= t} (k_t . q_u) dO_u
//     Z_t    = v_t A_t^T           = v_t dS_out^T + sum_{u >= t} (v_t . dO_u) q_u
//     dv_t = eta_t Y_t,  dk_t = eta_t Z_t,  deta_t = Y_t . v_t,  dS0 = A_0.
// Each of dQ, Y and Z is the forward recurrence itself with other operands, so the three run
// on the forward kernel (assoc_scan.cu):
//     dQ: queries dO, keys V, values K, rates eta, start S0^T          (forward order)
//     Y : queries K,  keys Q, values dO, rate 1,   start dS_out         (reverse order)
//     Z : queries V,  keys dO, values Q, rate 1,   start dS_out^T       (reverse order)
// where reverse order walks the chunks from the last and keeps, inside a chunk, key tokens at
// or after the query token. The state the Y pass ends with is dS0. The Z pass scales its output
// rows by eta in its own epilogue (it writes dK); a last elementwise pass scales Y by eta in
// place and forms deta = Y . v. Y and Z carry the same state (A and its transpose), so by
// default they run as one reverse pass (assoc_yz.cu) that reads Q, K, V and dO once; the tuning
// key "assoc_bwd_form" = 1 runs them as the two separate scans.
#include <cuda_bf16.h>

#include <string>

#include "internal.h"

namespace ttt {
namespace {

// dst[b] = src[b]^T for n matrices of d x d fp32 (32 x 32 tiles through shared memory).
__global__ void transpose_states_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                        int d) {
  __shared__ float tile[32][33];
  const size_t base = (size_t)blockIdx.z * d * d;
  const int x0 = blockIdx.x * 32, y0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y)
    tile[i][threadIdx.x] = src[base + (size_t)(y0 + i) * d + x0 + threadIdx.x];
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y)
    dst[base + (size_t)(x0 + i) * d + y0 + threadIdx.x] = tile[threadIdx.x][i];
}

__device__ __forceinline__ float bf16_to_f(uint16_t h) {
  return __uint_as_float((uint32_t)h << 16);
}
__device__ __forceinline__ uint16_t f_to_bf16(float f) {
  const __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&b);
}

// One warp per token row of DV = 64 or 128 values (DV / 32 per lane): dV = eta Y in place,
// deta = Y . V.
template <int DV>
__global__ void assoc_bwd_finish_kernel(const uint16_t* __restrict__ V, const float* eta,
                                        float eta_scalar, uint16_t* dV,
                                        float* __restrict__ deta, size_t rows) {
  constexpr int PER = DV / 32;
  using Vec = typename std::conditional<PER == 4, uint2, uint32_t>::type;
  const int lane = threadIdx.x & 31;
  const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
  for (size_t row = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const size_t o = row * DV + PER * lane;
    const Vec y = *reinterpret_cast<const Vec*>(dV + o);
    const Vec v = *reinterpret_cast<const Vec*>(V + o);
    const float e = eta ? eta[row] : eta_scalar;
    const uint16_t* yh = reinterpret_cast<const uint16_t*>(&y);
    const uint16_t* vh = reinterpret_cast<const uint16_t*>(&v);
    Vec ov;
    uint16_t* ovh = reinterpret_cast<uint16_t*>(&ov);
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const float yf = bf16_to_f(yh[i]);
      dot += yf * bf16_to_f(vh[i]);
      ovh[i] = f_to_bf16(e * yf);
    }
    *reinterpret_cast<Vec*>(dV + o) = ov;
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, s);
    if (lane == 0) deta[row] = dot;
  }
}

}  // namespace

size_t assoc_bwd_workspace_bytes(int B, int H, int T, int d, int C) {
  const size_t fwd = assoc_workspace_bytes(B, H, T, d, C);
  const size_t st = (size_t)B * H * d * d * sizeof(float);
  return ((fwd + 255) & ~size_t(255)) + 3 * st;
}

int launch_assoc_bwd(const AssocBwdArgs& a, const LaunchCtx& ctx) {
  const int BH = a.B * a.H, d = a.d;
  const size_t fwd = (assoc_workspace_bytes(a.B, a.H, a.T, d, a.C) + 255) & ~size_t(255);
  const size_t st = (size_t)BH * d * d * sizeof(float);
  if (a.ws_bytes < fwd + 3 * st) {
    *ctx.msg = "ttt_assoc_scan_bwd: workspace smaller than ttt_assoc_scan_bwd_workspace_size()";
    return kWorkspace;
  }
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  float* s0t = reinterpret_cast<float*>(ws + fwd);           // S0^T
  float* gt = reinterpret_cast<float*>(ws + fwd + st);       // dS_out^T
  float* junk = reinterpret_cast<float*>(ws + fwd + 2 * st);  // final states nobody reads
  const dim3 tgrid(d / 32, d / 32, BH), tblock(32, 8);
  if (a.S0) {
    transpose_states_kernel<<<tgrid, tblock, 0, ctx.stream>>>(a.S0, s0t, d);
    count_launch();
  }
  const bool fused = tuning(kTuneAssocBwdForm) != 1;   // Y and Z in one reverse pass
  if (a.dS_out && !fused) {
    transpose_states_kernel<<<tgrid, tblock, 0, ctx.stream>>>(a.dS_out, gt, d);
    count_launch();
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("assoc bwd transpose launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  // dQ: the forward recurrence with queries dO, keys V, values K
  StateArgs q{a.dO, a.V, a.K, a.eta, a.eta_scalar, a.S0 ? s0t : nullptr, a.dQ, junk, a.B, a.H,
              a.T, d, a.C, 1, a.ws, fwd};
  int r = launch_assoc(q, ctx);
  if (r != kOk) return r;
  if (fused) {
    r = launch_assoc_yz(a, a.ws, fwd, ctx);
    if (r != kOk) return r;
  }
  // Y (into dV): queries K, keys Q, values dO, reverse order; ends with dS0
  StateArgs y{a.K, a.Q, a.dO, nullptr, 1.0f, a.dS_out, a.dV, a.dS0, a.B, a.H, a.T, d, a.C, 1,
              a.ws, fwd};
  y.reverse = 1;
  if (!fused && (r = launch_assoc(y, ctx)) != kOk) return r;
  // Z (into dK): queries V, keys dO, values Q, reverse order
  StateArgs z{a.V, a.dO, a.Q, nullptr, 1.0f, a.dS_out ? gt : nullptr, a.dK, junk, a.B, a.H, a.T,
              d, a.C, 1, a.ws, fwd};
  z.reverse = 1;
  z.orow = a.eta;                              // dK = eta Z, scaled in the pass's epilogue
  z.oscale = a.eta ? 1.f : a.eta_scalar;
  if (!fused && (r = launch_assoc(z, ctx)) != kOk) return r;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto finish = d == 64 ? assoc_bwd_finish_kernel<64> : assoc_bwd_finish_kernel<128>;
  finish<<<sms * 8, 256, 0, ctx.stream>>>(static_cast<const uint16_t*>(a.V), a.eta, a.eta_scalar,
                                          static_cast<uint16_t*>(a.dV), a.deta,
                                          (size_t)BH * a.T);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("assoc bwd finish launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace ttt
