// Backward of the TTT-Linear mini-batch dual form, bf16 inputs, chunk C = 16, d in {32, 64, 128}.
//
// Forward, per (batch, head) stream and chunk c ("Learning to (Learn at Test Time)" reading,
// section on mini-batch TTT and its dual form):
//     G = K W - V,   O = Q W - A G  with  A = tril(Q K^T) diag(eta),   W' = W - K^T diag(eta) G.
// Given dO and the gradient dW_out of the final state, the chunk adjoint with X = dL/dW' is
//     U   = K X                         dG = -A^T dO - diag(eta) U        dV = -dG
//     dA  = -tril(dO G^T)               dS = dA diag(eta)                 (scores Q K^T)
//     dQ  = dO W^T + dS K               dK = dS^T Q - diag(eta) G X^T + dG W^T
//     deta_s = sum_t dA[t,s] (Q K^T)[t,s] - U_s . G_s
//     X  <- X + Q^T dO + K^T dG         (the gradient for the chunk before; dW0 after chunk 0)
// The state adjoint's recurrence does not involve W, but every gradient does, so the kernel runs
// two sweeps in one CTA per stream:
//   1. forward: the chunk-start states W_c are recomputed (fp32 in registers, bf16 operand copy
//      in shared memory, exactly the products of the forward kernel) and written to the
//      workspace as bf16, one d x d checkpoint per chunk;
//   2. reverse: chunks from last to first; X stays in fp32 registers (its bf16 copy
//      double-buffered in shared memory), and the chunk's twelve products run on mma.sync
//      m16n8k16 (bf16 operands, fp32 accumulation) in four phases separated by block barriers.
// Inputs (and in sweep 2 the checkpoints) stream through a ring of shared-memory slots filled by
// cp.async up to three chunks ahead, so that the serial chunk loop does not wait on HBM latency.
// Results (checkpoints, dQ, dK, dV) are staged in shared memory and leave as whole 16-byte
// pieces: written straight from the MMA fragments, every row would be an 8-byte scatter.
// Work split over 8 warps: a 16 x d result is cut into d/8 column tiles (n8) dealt round-robin
// to the warps; a warp owns the same columns of the state (all d/16 row tiles), so the state
// recurrences (column-independent) need no barrier of their own.
// Precision: W, X and all accumulations are fp32; operands (W_c, X, G, dG, A, dS) are rounded to
// bf16 once per chunk for the tensor cores.
#include <cuda_bf16.h>

#include <algorithm>

#include <string>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace ttt {
namespace {

constexpr int BC = 16;      // chunk length = MMA M
constexpr int NWARP = 8;
constexpr int THREADS = 32 * NWARP;

template <int D>
struct BwdCfg {
  static constexpr int LD = D + 8;                 // bf16 elements per padded shared row
  static constexpr int RS = LD * 2;                // bytes per row (a multiple of 16)
  static constexpr int TILE = BC * RS;             // one 16 x d operand
  static constexpr int WBYTES = D * RS;            // one d x d operand
  static constexpr int IN_Q = 0, IN_K = TILE, IN_V = 2 * TILE, IN_DO = 3 * TILE;
  static constexpr int IN_W = 4 * TILE;
  static constexpr int IN_ETA = IN_W + WBYTES;
  static constexpr int IN_BYTES = IN_ETA + 64;     // one chunk's inputs
  static constexpr int NBUF = D <= 64 ? 4 : 2;     // input ring: NBUF - 1 chunks in flight
  static constexpr int XB = NBUF * IN_BYTES;       // two bf16 state copies
  static constexpr int SG = XB + 2 * WBYTES;       // G (bf16)
  static constexpr int SEG = SG + TILE;            // diag(eta) G (bf16; negated in sweep 1)
  static constexpr int SDG = SEG + TILE;           // dG (bf16)
  static constexpr int SRS = 48;                   // row bytes of the 16 x 16 bf16 tiles
  static constexpr int SS = SDG + TILE;            // scores Q K^T, fp32 [16][20]
  static constexpr int SA = SS + BC * 20 * 4;      // A (bf16 [16][24])
  static constexpr int SDS = SA + BC * SRS;        // dS (bf16 [16][24])
  static constexpr int SDE2 = SDS + BC * SRS;      // per column tile: -sum_j U G  [NT][16]
  static constexpr int SDE1 = SDE2 + (D / 8) * 64; // sum_t dA (Q K^T)  [16]
  static constexpr int SOQ = SDE1 + 64;            // dQ, dV, dK staged for coalesced stores
  static constexpr int SOV = SOQ + TILE;
  static constexpr int SOK = SOV + TILE;
  static constexpr int SMEM = SOK + TILE;
  static constexpr int NT = D / 8, MT = D / 16, KS = D / 16;
  static constexpr int CT = (NT + NWARP - 1) / NWARP;  // column tiles per warp
  static_assert(IN_BYTES % 16 == 0 && RS % 16 == 0, "16-byte cp.async rows");
};

struct DualBwdParams {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const uint16_t* dO;
  const float* eta;     // [streams, T] or nullptr
  float eta_scalar;
  const float* W0;      // [streams, d, d] or nullptr
  const float* dW_out;  // [streams, d, d] or nullptr
  uint16_t* dQ;
  uint16_t* dK;
  uint16_t* dV;
  float* deta;
  float* dW0;
  uint16_t* ckpt;       // [streams, T / 16, d, d] bf16
  int T;
  int have_ckpt;        // the checkpoints are already written (sweep 1 is skipped)
};

// m16n8k16 operand fragments from padded shared tiles (row stride rs bytes).
// A (16 x 16) at (m0, k0) of a matrix stored [m][k].
__device__ __forceinline__ void frag_a(uint32_t base, int rs, int m0, int k0, uint32_t (&a)[4]) {
  const int l = threadIdx.x & 31, mi = l >> 3;
  ldsm_x4(base + (m0 + (l & 7) + (mi & 1) * 8) * rs + (k0 + (mi >> 1) * 8) * 2, a);
}
// A (16 x 16) at (m0, k0) of the transpose of a matrix stored [k][m].
__device__ __forceinline__ void frag_a_t(uint32_t base, int rs, int m0, int k0,
                                         uint32_t (&a)[4]) {
  const int l = threadIdx.x & 31, mi = l >> 3;
  ldsm_x4_t(base + (k0 + (l & 7) + (mi >> 1) * 8) * rs + (m0 + (mi & 1) * 8) * 2, a);
}
// B (16 x 8) at (k0, n0) of a matrix stored [n][k] (B^T row-major).
__device__ __forceinline__ void frag_b(uint32_t base, int rs, int n0, int k0, uint32_t (&b)[2]) {
  const int l = threadIdx.x & 15;
  ldsm_x2(base + (n0 + (l & 7)) * rs + (k0 + (l >> 3) * 8) * 2, b);
}
// B (16 x 8) at (k0, n0) of a matrix stored [k][n] (row-major).
__device__ __forceinline__ void frag_b_t(uint32_t base, int rs, int k0, int n0,
                                         uint32_t (&b)[2]) {
  const int l = threadIdx.x & 15;
  ldsm_x2_t(base + (k0 + (l & 7) + (l >> 3) * 8) * rs + n0 * 2, b);
}
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  mma16816(d, a[0], a[1], a[2], a[3], b[0], b[1]);
}

// rows x d bf16 from a padded shared tile (row stride rs bytes) to dense global rows, one
// 16-byte piece per thread and step (a warp writes four whole 128-byte rows at d = 64)
template <int D, int ROWS, int NTHR>
__device__ __forceinline__ void copy_out(uint32_t src, int rs, uint16_t* dst, int tid) {
  constexpr int PPR = D / 8, N = ROWS * PPR;
#pragma unroll
  for (int k = 0; k < (N + NTHR - 1) / NTHR; ++k) {
    const int i = tid + k * NTHR;
    if (N % NTHR == 0 || i < N)
      *reinterpret_cast<uint4*>(dst + (size_t)(i / PPR) * D + (i % PPR) * 8) =
          lds128(src + (i / PPR) * rs + (i % PPR) * 16);
  }
}

template <int D>
__global__ void __launch_bounds__(THREADS, 1) dual_bwd_kernel(const DualBwdParams p) {
  using L = BwdCfg<D>;
  constexpr int RS = L::RS;
  extern __shared__ __align__(16) unsigned char smem[];
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const int n = p.T / BC;
  const size_t s_tok = (size_t)blockIdx.x * p.T;           // first token row of this stream
  uint16_t* ck = p.ckpt + (size_t)blockIdx.x * n * D * D;

  // State tiles (W in sweep 1, X in sweep 2): warp w owns whole column tiles nt = w + 8 ct
  // (all d/16 row tiles of each). Columns of both recurrences are independent, so each warp
  // carries its own columns from chunk to chunk without block barriers.
  float st[L::CT][L::MT][4];
  auto load_state = [&](const float* src) {
#pragma unroll
    for (int ct = 0; ct < L::CT; ++ct) {
      const int nt = warp + NWARP * ct;
#pragma unroll
      for (int mt = 0; mt < L::MT; ++mt) {
        const int row = mt * 16 + g, col = nt * 8 + 2 * tq;
        if (src && nt < L::NT) {
          const float* s = src + (size_t)blockIdx.x * D * D;
          const float2 u = *reinterpret_cast<const float2*>(s + row * D + col);
          const float2 v = *reinterpret_cast<const float2*>(s + (row + 8) * D + col);
          st[ct][mt][0] = u.x, st[ct][mt][1] = u.y, st[ct][mt][2] = v.x, st[ct][mt][3] = v.y;
        } else {
          st[ct][mt][0] = st[ct][mt][1] = st[ct][mt][2] = st[ct][mt][3] = 0.f;
        }
      }
    }
  };
  auto put_state = [&](uint32_t dst, uint16_t* gdst) {   // bf16 copy (shared, and a checkpoint)
#pragma unroll
    for (int ct = 0; ct < L::CT; ++ct) {
      const int nt = warp + NWARP * ct;
      if (nt < L::NT) {
#pragma unroll
        for (int mt = 0; mt < L::MT; ++mt) {
          const int row = mt * 16 + g, col = nt * 8 + 2 * tq;
          const uint32_t w0 = pack_bf16(st[ct][mt][0], st[ct][mt][1]);
          const uint32_t w1 = pack_bf16(st[ct][mt][2], st[ct][mt][3]);
          sts32(dst + row * RS + col * 2, w0);
          sts32(dst + (row + 8) * RS + col * 2, w1);
          if (gdst) {
            *reinterpret_cast<uint32_t*>(gdst + row * D + col) = w0;
            *reinterpret_cast<uint32_t*>(gdst + (row + 8) * D + col) = w1;
          }
        }
      }
    }
  };
  // ROWS x d bf16 rows, dense in global memory, into padded shared rows (16-byte pieces)
  auto cp_rows = [&](auto rows_c, uint32_t dst, const uint16_t* src) {
    constexpr int ROWS = decltype(rows_c)::value, PPR = D / 8, N = ROWS * PPR;
#pragma unroll
    for (int k = 0; k < (N + THREADS - 1) / THREADS; ++k) {
      const int i = threadIdx.x + k * THREADS;
      if (N % THREADS == 0 || i < N)
        cp_async16(dst + (i / PPR) * RS + (i % PPR) * 16, src + (size_t)(i / PPR) * D + (i % PPR) * 8);
    }
  };
  using Rows16 = std::integral_constant<int, BC>;
  using RowsD = std::integral_constant<int, D>;
  auto cp_eta = [&](uint32_t dst, int c) {
    if (p.eta) {
      if (threadIdx.x < 4) cp_async16(dst + threadIdx.x * 16, p.eta + s_tok + c * BC + threadIdx.x * 4);
    } else if (threadIdx.x < BC) {
      stsf(dst + threadIdx.x * 4, p.eta_scalar);
    }
  };

  // ---------------------------------------------------------------- sweep 1: chunk-start states
  auto load_kv = [&](int c) {
    const uint32_t buf = sb + (c % L::NBUF) * L::IN_BYTES;
    cp_rows(Rows16{}, buf + L::IN_K, p.K + (s_tok + (size_t)c * BC) * D);
    cp_rows(Rows16{}, buf + L::IN_V, p.V + (s_tok + (size_t)c * BC) * D);
    cp_eta(buf + L::IN_ETA, c);
  };
  load_state(p.W0);
  put_state(sb + L::XB, nullptr);
#pragma unroll
  for (int s = 0; s < L::NBUF - 1; ++s) {   // one commit group per ring slot, empty past the end
    if (s < n && !p.have_ckpt) load_kv(s);
    cp_async_commit();
  }
  for (int c = 0; c < (p.have_ckpt ? 0 : n); ++c) {
    const uint32_t in = sb + (c % L::NBUF) * L::IN_BYTES;
    const uint32_t wb = sb + L::XB + (c & 1) * L::WBYTES;
    const uint32_t wn = sb + L::XB + ((c + 1) & 1) * L::WBYTES;
    cp_async_wait<L::NBUF - 2>();   // chunk c's group has landed (this thread's part)
    __syncthreads();                // ... and every thread's; slot (c - 1) % NBUF is free
    if (c + L::NBUF - 1 < n) load_kv(c + L::NBUF - 1);
    cp_async_commit();
    // checkpoint W_c (complete in wb since the barrier above), coalesced 16-byte stores
    copy_out<D, D, THREADS>(wb, RS, ck + (size_t)c * D * D, threadIdx.x);
    // -diag(eta) G = diag(eta) (V - K W), column tiles
#pragma unroll
    for (int ct = 0; ct < L::CT; ++ct) {
      const int nt = warp + NWARP * ct;
      if (nt < L::NT) {
        // two accumulators (even / odd k-steps) halve the dependent MMA chain
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < L::KS; ++ks) {
          uint32_t a[4], b[2];
          frag_a(in + L::IN_K, RS, 0, 16 * ks, a);
          frag_b_t(wb, RS, 16 * ks, 8 * nt, b);
          mma((ks & 1) ? acc2 : acc, a, b);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] += acc2[j];
        const int col = 8 * nt + 2 * tq;
        const uint32_t v0 = ldsu32(in + L::IN_V + g * RS + col * 2);
        const uint32_t v1 = ldsu32(in + L::IN_V + (g + 8) * RS + col * 2);
        const float e0 = ldsf(in + L::IN_ETA + 4 * g), e1 = ldsf(in + L::IN_ETA + 4 * (g + 8));
        sts32(sb + L::SEG + g * RS + col * 2,
              pack_bf16(e0 * (bf16_lo(v0) - acc[0]), e0 * (bf16_hi(v0) - acc[1])));
        sts32(sb + L::SEG + (g + 8) * RS + col * 2,
              pack_bf16(e1 * (bf16_lo(v1) - acc[2]), e1 * (bf16_hi(v1) - acc[3])));
      }
    }
    __syncwarp();   // the update below reads only this warp's columns of -diag(eta) G
    // W += K^T (-diag(eta) G), own columns
#pragma unroll
    for (int ct = 0; ct < L::CT; ++ct) {
      const int nt = warp + NWARP * ct;
      if (nt < L::NT) {
#pragma unroll
        for (int mt = 0; mt < L::MT; ++mt) {
          uint32_t a[4], b[2];
          frag_a_t(in + L::IN_K, RS, 16 * mt, 0, a);
          frag_b_t(sb + L::SEG, RS, 0, 8 * nt, b);
          mma(st[ct][mt], a, b);
        }
      }
    }
    put_state(wn, nullptr);
  }
  cp_async_wait_all();
  __syncthreads();   // checkpoints written above are read back below through cp.async

  // ---------------------------------------------------------------- sweep 2: adjoint, reversed
  auto prefetch = [&](uint32_t buf, int c) {
    const size_t row = s_tok + (size_t)c * BC;
    cp_rows(Rows16{}, buf + L::IN_Q, p.Q + row * D);
    cp_rows(Rows16{}, buf + L::IN_K, p.K + row * D);
    cp_rows(Rows16{}, buf + L::IN_V, p.V + row * D);
    cp_rows(Rows16{}, buf + L::IN_DO, p.dO + row * D);
    cp_rows(RowsD{}, buf + L::IN_W, ck + (size_t)c * D * D);
    cp_eta(buf + L::IN_ETA, c);
  };
  load_state(p.dW_out);
  put_state(sb + L::XB, nullptr);
#pragma unroll
  for (int s = 0; s < L::NBUF - 1; ++s) {
    if (s < n) prefetch(sb + s * L::IN_BYTES, n - 1 - s);
    cp_async_commit();
  }
  for (int i = 0; i < n; ++i) {
    const int c = n - 1 - i;
    const size_t row0 = s_tok + (size_t)c * BC;
    const uint32_t in = sb + (i % L::NBUF) * L::IN_BYTES;
    const uint32_t xb = sb + L::XB + (i & 1) * L::WBYTES;
    const uint32_t xn = sb + L::XB + ((i + 1) & 1) * L::WBYTES;
    cp_async_wait<L::NBUF - 2>();
    __syncthreads();
    if (i + L::NBUF - 1 < n)
      prefetch(sb + ((i + L::NBUF - 1) % L::NBUF) * L::IN_BYTES, c - (L::NBUF - 1));
    cp_async_commit();
    const float e_g = ldsf(in + L::IN_ETA + 4 * g), e_g8 = ldsf(in + L::IN_ETA + 4 * (g + 8));
    if (i > 0)   // dK of the previous chunk (c + 1), staged in its phase D
      copy_out<D, BC, THREADS>(sb + L::SOK, RS, p.dK + (row0 + BC) * D, threadIdx.x);

    // Phase A: G = K W - V, U = K X, dO W^T (column tiles); scores Q K^T (warps 0-1)
    float G[L::CT][4], U[L::CT][4], T1[L::CT][4];
#pragma unroll
    for (int ct = 0; ct < L::CT; ++ct) {
      const int nt = warp + NWARP * ct;
#pragma unroll
      for (int j = 0; j < 4; ++j) G[ct][j] = U[ct][j] = T1[ct][j] = 0.f;
      if (nt < L::NT) {
#pragma unroll
        for (int ks = 0; ks < L::KS; ++ks) {
          uint32_t a[4], b[2];
          frag_a(in + L::IN_K, RS, 0, 16 * ks, a);
          frag_b_t(in + L::IN_W, RS, 16 * ks, 8 * nt, b);
          mma(G[ct], a, b);
          frag_b_t(xb, RS, 16 * ks, 8 * nt, b);
          mma(U[ct], a, b);
          frag_a(in + L::IN_DO, RS, 0, 16 * ks, a);
          frag_b(in + L::IN_W, RS, 8 * nt, 16 * ks, b);
          mma(T1[ct], a, b);
        }
        const int col = 8 * nt + 2 * tq;
        const uint32_t v0 = ldsu32(in + L::IN_V + g * RS + col * 2);
        const uint32_t v1 = ldsu32(in + L::IN_V + (g + 8) * RS + col * 2);
        G[ct][0] -= bf16_lo(v0), G[ct][1] -= bf16_hi(v0);
        G[ct][2] -= bf16_lo(v1), G[ct][3] -= bf16_hi(v1);
        sts32(sb + L::SG + g * RS + col * 2, pack_bf16(G[ct][0], G[ct][1]));
        sts32(sb + L::SG + (g + 8) * RS + col * 2, pack_bf16(G[ct][2], G[ct][3]));
        sts32(sb + L::SEG + g * RS + col * 2, pack_bf16(e_g * G[ct][0], e_g * G[ct][1]));
        sts32(sb + L::SEG + (g + 8) * RS + col * 2, pack_bf16(e_g8 * G[ct][2], e_g8 * G[ct][3]));
        // -U_s . G_s over this tile's 8 columns (rows g and g + 8)
        float r0 = U[ct][0] * G[ct][0] + U[ct][1] * G[ct][1];
        float r1 = U[ct][2] * G[ct][2] + U[ct][3] * G[ct][3];
        r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
        r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
        r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
        r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
        if (tq == 0) {
          stsf(sb + L::SDE2 + nt * 64 + 4 * g, -r0);
          stsf(sb + L::SDE2 + nt * 64 + 4 * (g + 8), -r1);
        }
      }
    }
    if (warp < 2) {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < L::KS; ++ks) {
        uint32_t a[4], b[2];
        frag_a(in + L::IN_Q, RS, 0, 16 * ks, a);
        frag_b(in + L::IN_K, RS, 8 * warp, 16 * ks, b);
        mma(s, a, b);
      }
      const int col = 8 * warp + 2 * tq;
      stsf(sb + L::SS + (g * 20 + col) * 4, s[0]);
      stsf(sb + L::SS + (g * 20 + col + 1) * 4, s[1]);
      stsf(sb + L::SS + ((g + 8) * 20 + col) * 4, s[2]);
      stsf(sb + L::SS + ((g + 8) * 20 + col + 1) * 4, s[3]);
    }
    __syncthreads();

    // Phase B (warps 0-1, score columns 8w..8w+7): dA = -tril(dO G^T), dS, A, deta's first term
    if (warp < 2) {
      float pacc[4] = {0.f, 0.f, 0.f, 0.f}, pacc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < L::KS; ++ks) {
        uint32_t a[4], b[2];
        frag_a(in + L::IN_DO, RS, 0, 16 * ks, a);
        frag_b(sb + L::SG, RS, 8 * warp, 16 * ks, b);
        mma((ks & 1) ? pacc2 : pacc, a, b);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) pacc[j] += pacc2[j];
      float col_sum[2] = {0.f, 0.f};
      float dsv[4], av[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = g + (j >> 1) * 8, s = 8 * warp + 2 * tq + (j & 1);
        const bool on = t >= s;
        const float m = on ? -pacc[j] : 0.f;
        const float sv = ldsf(sb + L::SS + (t * 20 + s) * 4);
        const float es = ldsf(in + L::IN_ETA + 4 * s);
        dsv[j] = m * es;
        av[j] = on ? sv * es : 0.f;
        col_sum[j & 1] += m * sv;
      }
      const int col = 8 * warp + 2 * tq;
      sts32(sb + L::SDS + g * L::SRS + col * 2, pack_bf16(dsv[0], dsv[1]));
      sts32(sb + L::SDS + (g + 8) * L::SRS + col * 2, pack_bf16(dsv[2], dsv[3]));
      sts32(sb + L::SA + g * L::SRS + col * 2, pack_bf16(av[0], av[1]));
      sts32(sb + L::SA + (g + 8) * L::SRS + col * 2, pack_bf16(av[2], av[3]));
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        col_sum[j] += __shfl_xor_sync(0xffffffffu, col_sum[j], 4);
        col_sum[j] += __shfl_xor_sync(0xffffffffu, col_sum[j], 8);
        col_sum[j] += __shfl_xor_sync(0xffffffffu, col_sum[j], 16);
      }
      if (g == 0) {
        stsf(sb + L::SDE1 + 4 * col, col_sum[0]);
        stsf(sb + L::SDE1 + 4 * (col + 1), col_sum[1]);
      }
    }
    __syncthreads();

    // Phase C: dG = -A^T dO - diag(eta) U, dV = -dG, dQ = dO W^T + dS K (column tiles); deta
#pragma unroll
    for (int ct = 0; ct < L::CT; ++ct) {
      const int nt = warp + NWARP * ct;
      if (nt < L::NT) {
        float at[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t a[4], b[2];
        frag_a_t(sb + L::SA, L::SRS, 0, 0, a);
        frag_b_t(in + L::IN_DO, RS, 0, 8 * nt, b);
        mma(at, a, b);
        frag_a(sb + L::SDS, L::SRS, 0, 0, a);
        frag_b_t(in + L::IN_K, RS, 0, 8 * nt, b);
        mma(T1[ct], a, b);
        float dg[4];
        dg[0] = -at[0] - e_g * U[ct][0];
        dg[1] = -at[1] - e_g * U[ct][1];
        dg[2] = -at[2] - e_g8 * U[ct][2];
        dg[3] = -at[3] - e_g8 * U[ct][3];
        const int col = 8 * nt + 2 * tq;
        sts32(sb + L::SDG + g * RS + col * 2, pack_bf16(dg[0], dg[1]));
        sts32(sb + L::SDG + (g + 8) * RS + col * 2, pack_bf16(dg[2], dg[3]));
        sts32(sb + L::SOV + g * RS + col * 2, pack_bf16(-dg[0], -dg[1]));
        sts32(sb + L::SOV + (g + 8) * RS + col * 2, pack_bf16(-dg[2], -dg[3]));
        sts32(sb + L::SOQ + g * RS + col * 2, pack_bf16(T1[ct][0], T1[ct][1]));
        sts32(sb + L::SOQ + (g + 8) * RS + col * 2, pack_bf16(T1[ct][2], T1[ct][3]));
      }
    }
    if (warp == NWARP - 1 && lane < BC) {
      float de = ldsf(sb + L::SDE1 + 4 * lane);
#pragma unroll
      for (int nt = 0; nt < L::NT; ++nt) de += ldsf(sb + L::SDE2 + nt * 64 + 4 * lane);
      p.deta[row0 + lane] = de;
    }
    __syncthreads();

    // Phase D: dK = dS^T Q + dG W^T - diag(eta) G X^T (column tiles); X += Q^T dO + K^T dG
    copy_out<D, BC, THREADS>(sb + L::SOV, RS, p.dV + row0 * D, threadIdx.x);
    copy_out<D, BC, THREADS>(sb + L::SOQ, RS, p.dQ + row0 * D, threadIdx.x);
#pragma unroll
    for (int ct = 0; ct < L::CT; ++ct) {
      const int nt = warp + NWARP * ct;
      if (nt < L::NT) {
        float k1[4] = {0.f, 0.f, 0.f, 0.f}, k2[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t a[4], b[2];
        frag_a_t(sb + L::SDS, L::SRS, 0, 0, a);
        frag_b_t(in + L::IN_Q, RS, 0, 8 * nt, b);
        mma(k1, a, b);
#pragma unroll
        for (int ks = 0; ks < L::KS; ++ks) {
          frag_a(sb + L::SDG, RS, 0, 16 * ks, a);
          frag_b(in + L::IN_W, RS, 8 * nt, 16 * ks, b);
          mma(k1, a, b);
          frag_a(sb + L::SEG, RS, 0, 16 * ks, a);
          frag_b(xb, RS, 8 * nt, 16 * ks, b);
          mma(k2, a, b);
        }
        const int col = 8 * nt + 2 * tq;
        sts32(sb + L::SOK + g * RS + col * 2, pack_bf16(k1[0] - k2[0], k1[1] - k2[1]));
        sts32(sb + L::SOK + (g + 8) * RS + col * 2, pack_bf16(k1[2] - k2[2], k1[3] - k2[3]));
      }
    }
#pragma unroll
    for (int ct = 0; ct < L::CT; ++ct) {
      const int nt = warp + NWARP * ct;
      if (nt < L::NT) {
#pragma unroll
        for (int mt = 0; mt < L::MT; ++mt) {
          uint32_t a[4], b[2];
          frag_a_t(in + L::IN_K, RS, 16 * mt, 0, a);
          frag_b_t(sb + L::SDG, RS, 0, 8 * nt, b);
          mma(st[ct][mt], a, b);
          frag_a_t(in + L::IN_Q, RS, 16 * mt, 0, a);
          frag_b_t(in + L::IN_DO, RS, 0, 8 * nt, b);
          mma(st[ct][mt], a, b);
        }
      }
    }
    put_state(xn, nullptr);
  }
  __syncthreads();   // dK of chunk 0
  copy_out<D, BC, THREADS>(sb + L::SOK, RS, p.dK + s_tok * D, threadIdx.x);
  // dW0 (fp32)
  float* dw = p.dW0 + (size_t)blockIdx.x * D * D;
#pragma unroll
  for (int ct = 0; ct < L::CT; ++ct) {
    const int nt = warp + NWARP * ct;
    if (nt < L::NT) {
#pragma unroll
      for (int mt = 0; mt < L::MT; ++mt) {
        const int row = mt * 16 + g, col = nt * 8 + 2 * tq;
        *reinterpret_cast<float2*>(dw + row * D + col) = make_float2(st[ct][mt][0], st[ct][mt][1]);
        *reinterpret_cast<float2*>(dw + (row + 8) * D + col) =
            make_float2(st[ct][mt][2], st[ct][mt][3]);
      }
    }
  }
}

template <int D>
int launch_d(const DualBwdParams& p, int streams, const LaunchCtx& ctx) {
  constexpr int smem = BwdCfg<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(dual_bwd_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) {
    dual_bwd_kernel<D><<<streams, THREADS, smem, ctx.stream>>>(p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual bwd launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

// dt: 1 = bf16 (the public dtype code)
bool dual_bwd_supported(int d, int C, int dt) {
  return dt == 1 && C == BC && (d == 32 || d == 64 || d == 128);
}

size_t dual_bwd_workspace_bytes(int B, int H, int T, int d) {
  const size_t chunks = (size_t)B * H * (T / BC) * d * d * 2;   // one checkpoint per chunk
  return d == 64 ? std::max(chunks, dual_bwd_stage_workspace_bytes(B, H, T)) : chunks;
}

int launch_dual_bwd(const AssocBwdArgs& a, const LaunchCtx& ctx) {
  DualBwdParams p;
  p.Q = static_cast<const uint16_t*>(a.Q);
  p.K = static_cast<const uint16_t*>(a.K);
  p.V = static_cast<const uint16_t*>(a.V);
  p.dO = static_cast<const uint16_t*>(a.dO);
  p.eta = a.eta;
  p.eta_scalar = a.eta_scalar;
  p.W0 = a.S0;
  p.dW_out = a.dS_out;
  p.dQ = static_cast<uint16_t*>(a.dQ);
  p.dK = static_cast<uint16_t*>(a.dK);
  p.dV = static_cast<uint16_t*>(a.dV);
  p.deta = a.deta;
  p.dW0 = a.dS0;
  p.ckpt = static_cast<uint16_t*>(a.ws);
  p.T = a.T;
  p.have_ckpt = 0;
  const int streams = a.B * a.H;
  // d = 64: the stage form by default ("dual_bwd_form" 0); with 2 the chunk-start checkpoints
  // come from the stage kernel's state-only chain (one SM's four chain warps per stream, no block
  // barriers), which writes them faster than this kernel's own forward sweep (1)
  const int form = a.d == 64 ? tuning(kTuneDualBwdForm) : 1;
  if (form == 0) return launch_dual_bwd_stage(a, ctx);
  if (form == 2) {
    StateArgs f{a.K, a.K, a.V, a.eta, a.eta_scalar, a.S0, nullptr, nullptr, a.B, a.H, a.T, a.d,
                BC, 1, nullptr, 0};
    const int st = launch_dual_tc_checkpoints(f, p.ckpt, ctx);
    if (st != kOk) return st;
    p.have_ckpt = 1;
  }
  switch (a.d) {
    case 32: return launch_d<32>(p, streams, ctx);
    case 64: return launch_d<64>(p, streams, ctx);
    case 128: return launch_d<128>(p, streams, ctx);
    default: return kUnsupported;
  }
}

}  // namespace ttt
