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
// The backward (launch_dual_seg_bwd) reuses the maps and the start states and folds the state
// gradient's own affine recurrence in reverse.
#include <algorithm>
#include <string>

#include "internal.h"
#include "ptx.cuh"

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

// Register-tiled D x D fp32 product for the folds: thread t of 256 owns the TT x TT block of
// outputs at rows TT (t / 16), columns TT (t % 16) (TT = D / 16) and adds
//     acc[r][c] += sum_k op(A)[row r][k] * W[k][column c],   op(A) = A, or A^T if TRANS,
// with A and W row-major [D][D] in shared memory. Each k-step of 4 loads 4 TT-wide rows of W
// and the matching 4 x TT piece of op(A) as whole vectors, then does 16 TT^2 independent FMAs.
template <int N>
__device__ __forceinline__ void ld_row(const float* p, float (&v)[N]) {
  if constexpr (N == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x, v[1] = x.y;
  } else {
#pragma unroll
    for (int h = 0; h < N / 4; ++h) {
      const float4 x = *reinterpret_cast<const float4*>(p + 4 * h);
      v[4 * h] = x.x, v[4 * h + 1] = x.y, v[4 * h + 2] = x.z, v[4 * h + 3] = x.w;
    }
  }
}
template <int D, bool TRANS>
__device__ __forceinline__ void tile_product(const float* A, const float* W,
                                             float (&acc)[D / 16][D / 16]) {
  constexpr int TT = D / 16;
  const int i0 = TT * (threadIdx.x / 16), j0 = TT * (threadIdx.x % 16);
#pragma unroll 2
  for (int k = 0; k < D; k += 4) {
    float a[4][TT];   // a[kk][r] = op(A)[i0 + r][k + kk]
    if constexpr (TRANS) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) ld_row<TT>(A + (k + kk) * D + i0, a[kk]);
    } else {
#pragma unroll
      for (int r = 0; r < TT; ++r) {
        float v[4];
        ld_row<4>(A + (i0 + r) * D + k, v);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) a[kk][r] = v[kk];
      }
    }
    float w[4][TT];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) ld_row<TT>(W + (k + kk) * D + j0, w[kk]);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int r = 0; r < TT; ++r)
#pragma unroll
        for (int c = 0; c < TT; ++c) acc[r][c] = fmaf(a[kk][r], w[kk][c], acc[r][c]);
  }
}
// W <- op(A) W + bias (bias a global D x D matrix), all threads of the CTA.
template <int D, bool TRANS>
__device__ __forceinline__ void affine_step(const float* A, float* W,
                                            const float* __restrict__ bias) {
  constexpr int TT = D / 16;
  const int i0 = TT * (threadIdx.x / 16), j0 = TT * (threadIdx.x % 16);
  float acc[TT][TT];
#pragma unroll
  for (int r = 0; r < TT; ++r) ld_row<TT>(bias + (i0 + r) * D + j0, acc[r]);
  tile_product<D, TRANS>(A, W, acc);
  __syncthreads();
#pragma unroll
  for (int r = 0; r < TT; ++r)
#pragma unroll
    for (int c = 0; c < TT; ++c) W[(i0 + r) * D + j0 + c] = acc[r][c];
  __syncthreads();
}

// One CTA per stream: W (fp32, d x d) and A_s = (A_s + B_s) - B_s in shared memory; segment s
// stores its start state, then W <- A_s W + B_s.
template <int D>
__global__ void __launch_bounds__(256) fold_segments_kernel(const float* __restrict__ W0,
                                                            const float* __restrict__ Bm,
                                                            const float* __restrict__ ABm,
                                                            float* __restrict__ Wstart, int S) {
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
    affine_step<D, false>(A, W, Bm + seg);
  }
}

// Backward of the segment-affine evaluation: the state gradient X obeys
// X_before = (I - K^T diag(eta) K) X_after + Q^T dO - K^T A^T dO per chunk (no W in it), so a
// segment maps X_before = A_s^T X_after + N_s (each chunk factor is symmetric, so the segment's
// factor is the transpose of the forward's A_s). One CTA per stream, in reverse segment order:
// segment s stores its X_after, then X <- A_s^T X + N_s.
template <int D>
__global__ void __launch_bounds__(256) fold_segments_reverse_kernel(
    const float* __restrict__ dW_out, const float* __restrict__ Bm, const float* __restrict__ ABm,
    const float* __restrict__ Noff, float* __restrict__ Xafter, int S) {
  extern __shared__ float fsm[];
  float* X = fsm;                  // [D][D]
  float* A = fsm + D * D;          // [D][D] = A_s
  const size_t bh = blockIdx.x;
  for (int i = threadIdx.x; i < D * D; i += 256) X[i] = dW_out ? dW_out[bh * D * D + i] : 0.f;
  __syncthreads();
  for (int s = S - 1; s >= 0; --s) {
    const size_t seg = (bh * S + s) * D * D;
    for (int i = threadIdx.x; i < D * D; i += 256) {
      Xafter[seg + i] = X[i];
      A[i] = ABm[seg + i] - Bm[seg + i];
    }
    __syncthreads();
    affine_step<D, true>(A, X, Noff + seg);   // X <- A_s^T X + N_s
  }
}

// Column-sliced fold, d = 64: one CTA per (stream, 16-column slice of the state); the columns
// of W <- A W + B (and of the reverse X <- A^T X + N) evolve independently. The segment maps
// arrive as A itself (the caller subtracts B from the run from W = I beforehand), so a step
// needs A (16 KB) and the bias's 16 columns (4 KB): both stream in through a double-buffered
// cp.async ring one segment ahead while the CTA stores the slice of the incoming state and
// updates it. Thread t owns rows 4 (t / 16) .. +3 of slice column t % 16.
constexpr int FD = 64, FCW = 16, FCS = FD / FCW, FPITCH = FD + 4;   // padded map rows
constexpr int FBUF = FD * FPITCH + FD * FCW;                        // A, bias slice (floats)
constexpr int FOLD_COLS_SMEM = (FD * FCW + 2 * FBUF) * (int)sizeof(float);
template <bool REV>
__global__ void __launch_bounds__(256) fold_cols_kernel(const float* __restrict__ init,
                                                        const float* __restrict__ Am,
                                                        const float* __restrict__ bias,
                                                        float* __restrict__ out, int S) {
  extern __shared__ __align__(16) float fcm[];
  float* Wsl = fcm;                    // [FD][FCW] state slice
  float* bufs = fcm + FD * FCW;        // 2 buffers x {A [FD][FPITCH], bias slice [FD][FCW]}
  const size_t bh = blockIdx.x / FCS;
  const int c0 = (blockIdx.x % FCS) * FCW;
  const int c = threadIdx.x % 16, r0 = 4 * (threadIdx.x / 16);
  auto seg_of = [&](int i) { return REV ? S - 1 - i : i; };
  auto prefetch = [&](int i, int b) {
    const size_t seg = (bh * S + seg_of(i)) * FD * FD;
    float* d = bufs + b * FBUF;
#pragma unroll
    for (int k = 0; k < FD * FD / 4 / 256; ++k) {   // A: 16-byte pieces, 4 per thread
      const int e = threadIdx.x + 256 * k;
      cp_async16(smem_u32(d + (e / 16) * FPITCH + 4 * (e % 16)), Am + seg + 4 * e);
    }
    {   // bias columns c0 .. c0 + 15: one 16-byte piece per thread
      const int row = threadIdx.x / 4, q = threadIdx.x % 4;
      cp_async16(smem_u32(d + FD * FPITCH + row * FCW + 4 * q),
                 bias + seg + (size_t)row * FD + c0 + 4 * q);
    }
  };
  for (int e = threadIdx.x; e < FD * FCW; e += 256)
    Wsl[e] = init ? init[bh * FD * FD + (size_t)(e / FCW) * FD + c0 + e % FCW] : 0.f;
  if (S > 0) prefetch(0, 0);
  cp_async_commit();
  for (int i = 0; i < S; ++i) {
    const int b = i & 1;
    if (i + 1 < S) prefetch(i + 1, b ^ 1);
    cp_async_commit();
    cp_async_wait<1>();   // segment i's maps have landed (this thread's part) ...
    __syncthreads();      // ... and every thread's; the state slice is complete
    const size_t seg = (bh * S + seg_of(i)) * FD * FD;
    for (int e = threadIdx.x; e < FD * FCW; e += 256)
      out[seg + (size_t)(e / FCW) * FD + c0 + e % FCW] = Wsl[e];
    const float* A = bufs + b * FBUF;
    const float* bs = A + FD * FPITCH;
    float acc[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[r] = bs[(r0 + r) * FCW + c];
#pragma unroll 4
    for (int k = 0; k < FD; k += 4) {
      float w[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) w[kk] = Wsl[(k + kk) * FCW + c];
      if constexpr (REV) {   // A^T: row k of A, columns r0 .. r0+3
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const float4 a = *reinterpret_cast<const float4*>(A + (k + kk) * FPITCH + r0);
          acc[0] = fmaf(a.x, w[kk], acc[0]);
          acc[1] = fmaf(a.y, w[kk], acc[1]);
          acc[2] = fmaf(a.z, w[kk], acc[2]);
          acc[3] = fmaf(a.w, w[kk], acc[3]);
        }
      } else {               // A: rows r0 .. r0+3, columns k .. k+3
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 a = *reinterpret_cast<const float4*>(A + (r0 + r) * FPITCH + k);
          acc[r] = fmaf(a.x, w[0], fmaf(a.y, w[1], fmaf(a.z, w[2], fmaf(a.w, w[3], acc[r]))));
        }
      }
    }
    __syncthreads();      // every thread has read the slice and the maps of buffer b
#pragma unroll
    for (int r = 0; r < 4; ++r) Wsl[(r0 + r) * FCW + c] = acc[r];
  }
  cp_async_wait_all();
}

// dst[bh] = src[bh * S + s_pick] for bh_count d x d fp32 states
__global__ void pick_segment_state_kernel(const float* __restrict__ src, float* dst, int S,
                                          int s_pick, int d, size_t bh_count) {
  const size_t per = (size_t)d * d, total = bh_count * per;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = i / per, e = i % per;
    dst[i] = src[(bh * S + s_pick) * per + e];
  }
}

// a[i] -= b[i] over n elements
__global__ void sub_states_kernel(float* __restrict__ a, const float* __restrict__ b, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    a[i] -= b[i];
}

// Context parallelism: maps gathered from the ranks, [n_maps][BH][D][D] each (A and B apart).
// One CTA per stream: W = W0 (or 0), then W <- A_m W + B_m for m < upto; W_out = W.
template <int D>
__global__ void __launch_bounds__(256) fold_gathered_kernel(const float* __restrict__ W0,
                                                            const float* __restrict__ Am,
                                                            const float* __restrict__ Bm,
                                                            int upto, size_t bh_count,
                                                            float* __restrict__ W_out) {
  extern __shared__ float fsm[];
  float* W = fsm;
  float* A = fsm + D * D;
  const size_t bh = blockIdx.x;
  for (int i = threadIdx.x; i < D * D; i += 256) W[i] = W0 ? W0[bh * D * D + i] : 0.f;
  __syncthreads();
  for (int m = 0; m < upto; ++m) {
    const size_t off = ((size_t)m * bh_count + bh) * D * D;
    for (int i = threadIdx.x; i < D * D; i += 256) A[i] = Am[off + i];
    __syncthreads();
    affine_step<D, false>(A, W, Bm + off);
  }
  for (int i = threadIdx.x; i < D * D; i += 256) W_out[bh * D * D + i] = W[i];
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

namespace {

int run_dual(const StateArgs& x, const LaunchCtx& ctx) {
  return dual_mma_supported(x.d, x.C, x.dt) ? launch_dual_mma(x, ctx) : launch_dual_simt(x, ctx);
}

int check_launch(const LaunchCtx& ctx, const char* what, cudaError_t e = cudaSuccess) {
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) return kOk;
  *ctx.msg = std::string("dual seg ") + what + ": " + cudaGetErrorString(e);
  return kCuda;
}

// Per-stream fold over the segments, forward (start states) or reverse (state gradients).
int launch_fold(bool reverse, int d, int bh, const float* init, const float* Bm,
                const float* ABm, const float* Noff, float* dst, int S, const LaunchCtx& ctx) {
  const size_t smem = 2 * (size_t)d * d * sizeof(float);
  cudaError_t e = cudaSuccess;
  switch (d) {
    case 32:
      if (reverse)
        fold_segments_reverse_kernel<32><<<bh, 256, smem, ctx.stream>>>(init, Bm, ABm, Noff, dst, S);
      else
        fold_segments_kernel<32><<<bh, 256, smem, ctx.stream>>>(init, Bm, ABm, dst, S);
      break;
    case 64:
      // column-sliced, with the maps streamed one segment ahead (fold_cols_kernel); the maps
      // buffer holds A itself here (maps_and_fold subtracted B)
      if (reverse) {
        e = cudaFuncSetAttribute(fold_cols_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, FOLD_COLS_SMEM);
        if (e == cudaSuccess)
          fold_cols_kernel<true><<<bh * FCS, 256, FOLD_COLS_SMEM, ctx.stream>>>(init, ABm, Noff,
                                                                              dst, S);
      } else {
        e = cudaFuncSetAttribute(fold_cols_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, FOLD_COLS_SMEM);
        if (e == cudaSuccess)
          fold_cols_kernel<false><<<bh * FCS, 256, FOLD_COLS_SMEM, ctx.stream>>>(init, ABm, Bm,
                                                                               dst, S);
      }
      break;
    case 128:
      if (reverse) {
        e = cudaFuncSetAttribute(fold_segments_reverse_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
          fold_segments_reverse_kernel<128><<<bh, 256, smem, ctx.stream>>>(init, Bm, ABm, Noff,
                                                                           dst, S);
      } else {
        e = cudaFuncSetAttribute(fold_segments_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
          fold_segments_kernel<128><<<bh, 256, smem, ctx.stream>>>(init, Bm, ABm, dst, S);
      }
      break;
    default:
      *ctx.msg = "dual seg: unsupported head dim";
      return kUnsupported;
  }
  count_launch();
  return check_launch(ctx, "fold launch", e);
}

// Steps 1-3: the segment maps (B_s from W = 0, A_s + B_s from W = I) and the fold giving every
// segment's start state Wst. `v` is the segment view; the maps' outputs go to `Ojunk`.
int maps_and_fold(const StateArgs& v, int S, int bh, const float* W0, void* Ojunk, float* Wid,
                  float* Bm, float* ABm, float* Wst, const LaunchCtx& ctx) {
  const size_t n = (size_t)v.B;
  identity_states_kernel<<<sm_count() * 4, 256, 0, ctx.stream>>>(Wid, n, v.d);
  count_launch();
  int st = check_launch(ctx, "identity launch");
  if (st != kOk) return st;
  // the maps need only the final states: the state-only form where it exists, else the
  // outputs go to scratch
  void* const maps_O = dual_state_only_supported(v.d, v.C, v.dt) ? nullptr : Ojunk;
  StateArgs pb = v;
  pb.S0 = nullptr;
  pb.O = maps_O;
  pb.S_out = Bm;
  if ((st = run_dual(pb, ctx)) != kOk) return st;
  StateArgs pa = v;
  pa.S0 = Wid;
  pa.O = maps_O;
  pa.S_out = ABm;
  if ((st = run_dual(pa, ctx)) != kOk) return st;
  if (v.d == 64) {   // the column-sliced fold takes A itself: A + B -> A in place
    sub_states_kernel<<<sm_count() * 2, 256, 0, ctx.stream>>>(ABm, Bm, n * v.d * v.d);
    count_launch();
    if ((st = check_launch(ctx, "map difference launch")) != kOk) return st;
  }
  return launch_fold(false, v.d, bh, W0, Bm, ABm, nullptr, Wst, S, ctx);
}

int pick(const float* src, float* dst, int S, int s_pick, int d, int bh, const LaunchCtx& ctx) {
  pick_segment_state_kernel<<<sm_count() * 2, 256, 0, ctx.stream>>>(src, dst, S, s_pick, d,
                                                                     (size_t)bh);
  count_launch();
  return check_launch(ctx, "state launch");
}

}  // namespace

int launch_dual_seg(const StateArgs& a, int S, const LaunchCtx& ctx) {
  if (S <= 1) return run_dual(a, ctx);
  const int d = a.d, bh = a.B * a.H;
  const size_t n = (size_t)bh * S, per = (size_t)d * d;
  if (a.ws_bytes < dual_seg_workspace_bytes(a.B, a.H, d, S)) {
    *ctx.msg = "ttt_linear_dual_seg_fwd: workspace smaller than ttt_linear_dual_seg_workspace_size()";
    return kWorkspace;
  }
  float* Wid = static_cast<float*>(a.ws);
  float* Bm = Wid + n * per;
  float* ABm = Bm + n * per;
  float* Wst = ABm + n * per;
  float* Wend = Wst + n * per;
  // segments as independent streams: [B*H*S, 1, T/S, d]
  StateArgs v = a;
  v.B = (int)n;
  v.H = 1;
  v.T = a.T / S;
  v.ws = nullptr;
  v.ws_bytes = 0;
  int st = maps_and_fold(v, S, bh, a.S0, a.O, Wid, Bm, ABm, Wst, ctx);
  if (st != kOk) return st;
  // 4. outputs from the true segment starts; the last segment's end state is W_out
  StateArgs po = v;
  po.S0 = Wst;
  po.S_out = Wend;
  if ((st = run_dual(po, ctx)) != kOk) return st;
  return pick(Wend, a.S_out, S, S - 1, d, bh, ctx);
}

size_t dual_slice_maps_workspace_bytes(int B, int H, int T, int d, int dt) {
  // scratch outputs of the two passes, then the identity start states
  const size_t o = ((size_t)B * H * T * d * (dt ? 2 : 4) + 255) & ~size_t(255);
  return o + (size_t)B * H * d * d * sizeof(float);
}

// The maps of a token slice of every stream: B from W = 0, A = (end from W = I) - B.
int launch_dual_slice_maps(const StateArgs& a, float* A_out, float* B_out, const LaunchCtx& ctx) {
  const size_t bh = (size_t)a.B * a.H, per = (size_t)a.d * a.d;
  const size_t o = ((size_t)bh * a.T * a.d * (a.dt ? 2 : 4) + 255) & ~size_t(255);
  float* Wid = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) + o);
  identity_states_kernel<<<sm_count() * 4, 256, 0, ctx.stream>>>(Wid, bh, a.d);
  count_launch();
  int st = check_launch(ctx, "identity launch");
  if (st != kOk) return st;
  StateArgs x = a;   // final states only: the state-only form, else the outputs are scratch
  x.Q = a.K;
  x.O = dual_state_only_supported(a.d, a.C, a.dt) ? nullptr : a.ws;
  x.ws = nullptr;
  x.ws_bytes = 0;
  x.S0 = nullptr;
  x.S_out = B_out;
  if ((st = run_dual(x, ctx)) != kOk) return st;
  x.S0 = Wid;
  x.S_out = A_out;
  if ((st = run_dual(x, ctx)) != kOk) return st;
  sub_states_kernel<<<sm_count() * 2, 256, 0, ctx.stream>>>(A_out, B_out, bh * per);
  count_launch();
  return check_launch(ctx, "subtract launch");
}

int launch_dual_state_fold(const float* W0, const float* A, const float* B, int upto, int bh,
                           int d, float* W_out, const LaunchCtx& ctx) {
  const size_t smem = 2 * (size_t)d * d * sizeof(float);
  cudaError_t e = cudaSuccess;
  switch (d) {
    case 32:
      fold_gathered_kernel<32><<<bh, 256, smem, ctx.stream>>>(W0, A, B, upto, bh, W_out);
      break;
    case 64:
      fold_gathered_kernel<64><<<bh, 256, smem, ctx.stream>>>(W0, A, B, upto, bh, W_out);
      break;
    case 128:
      e = cudaFuncSetAttribute(fold_gathered_kernel<128>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess)
        fold_gathered_kernel<128><<<bh, 256, smem, ctx.stream>>>(W0, A, B, upto, bh, W_out);
      break;
    default:
      *ctx.msg = "dual state fold: unsupported head dim";
      return kUnsupported;
  }
  count_launch();
  return check_launch(ctx, "fold launch", e);
}

size_t dual_seg_bwd_workspace_bytes(int B, int H, int T, int d, int S) {
  if (S <= 1) return dual_bwd_workspace_bytes(B, H, T, d);
  // the backward kernel's checkpoints over the segment view, then seven fp32 states per segment
  const size_t ck = (dual_bwd_workspace_bytes(B * H * S, 1, T / S, d) + 255) & ~size_t(255);
  return ck + 7 * (size_t)B * H * S * d * d * sizeof(float);
}

// Backward: maps and start states as in the forward; a backward pass over the segments from a
// zero incoming state gradient gives each segment's offset N_s (its dW0 output); the reverse fold
// gives every segment's incoming state gradient X_after(s); a second backward pass from the
// true (W_start, X_after) gives the gradients, and segment 0's dW0 is the stream's.
int launch_dual_seg_bwd(const AssocBwdArgs& a, int S, const LaunchCtx& ctx) {
  if (S <= 1) return launch_dual_bwd(a, ctx);
  const int d = a.d, bh = a.B * a.H;
  const size_t n = (size_t)bh * S, per = (size_t)d * d;
  if (a.ws_bytes < dual_seg_bwd_workspace_bytes(a.B, a.H, a.T, d, S)) {
    *ctx.msg = "ttt_linear_dual_seg_bwd: workspace smaller than ttt_linear_dual_seg_bwd_workspace_size()";
    return kWorkspace;
  }
  const size_t ck = (dual_bwd_workspace_bytes((int)n, 1, a.T / S, d) + 255) & ~size_t(255);
  float* Wid = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) + ck);
  float* Bm = Wid + n * per;
  float* ABm = Bm + n * per;
  float* Wst = ABm + n * per;
  float* Noff = Wst + n * per;
  float* Xaft = Noff + n * per;
  float* dW0s = Xaft + n * per;
  StateArgs v{a.Q, a.K, a.V, a.eta, a.eta_scalar, nullptr, nullptr, nullptr, (int)n, 1,
              a.T / S, d, a.C, 1, nullptr, 0};
  // the forward maps write their (unused) outputs into dQ, which the last pass overwrites
  int st = maps_and_fold(v, S, bh, a.S0, a.dQ, Wid, Bm, ABm, Wst, ctx);
  if (st != kOk) return st;
  AssocBwdArgs b = a;
  b.B = (int)n;
  b.H = 1;
  b.T = a.T / S;
  b.S0 = Wst;
  b.ws = a.ws;
  b.ws_bytes = ck;
  b.dS_out = nullptr;   // offsets N_s (the gradients written here are overwritten below)
  b.dS0 = Noff;
  if ((st = launch_dual_bwd(b, ctx)) != kOk) return st;
  if ((st = launch_fold(true, d, bh, a.dS_out, Bm, ABm, Noff, Xaft, S, ctx)) != kOk) return st;
  b.dS_out = Xaft;
  b.dS0 = dW0s;
  if ((st = launch_dual_bwd(b, ctx)) != kOk) return st;
  return pick(dW0s, a.dS0, S, 0, d, bh, ctx);
}

}  // namespace ttt
