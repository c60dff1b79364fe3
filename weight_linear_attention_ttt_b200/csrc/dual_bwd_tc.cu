// Backward of the TTT-Linear mini-batch dual form, bf16, d = 64, chunk C = 16: the state
// gradient's chain on warp MMAs in registers, every product that needs the forward states on
// tcgen05 tensor cores, one 128-token stage at a time.
//
// Forward per (batch, head) stream and chunk c ("RNN의 기억을 작은 모델로 바꾼다면: Test-Time
// Training 읽기", section "gradient를 효율적인 layer로 만드는 작업", the mini-batch update and its
// dual form): G = K W_c - V, E = diag(eta) G, O = Q W_c - tril(Q K^T) E, W_c+1 = W_c - K^T E.
// Outer-loop training differentiates through these updates. With X_c = dL/dW_c+1 and
// A' = tril(Q K^T) of the chunk (unscaled), the chunk adjoint is
//     R   = A'^T dO + K X_c,        dG = -diag(eta) R,        dV = -dG,      deta_s = -G_s . R_s
//     dQ  = dO W_c^T - tril(dO E^T) K
//     dK  = -triu(E dO^T)_chunk Q - E X_c^T + dG W_c^T
//     X_c-1 = X_c + Q^T dO + K^T dG
// (the per-chunk form is the one the fp64 reference differentiates statement by statement).
//
// Stage form. A stage holds 128 tokens (8 chunks) with start state W_s and, in the reverse
// order, the state gradient X_e after its last chunk. Inside the stage
//     W_c   = W_s - sum_{c' < c} K_c'^T E_c'
//     X_c   = X_e + sum_{c' > c} (Q_c'^T dO_c' + K_c'^T dG_c')
// so every W- or X-dependent term of the stage's 128 rows is a masked product over the stage:
//     dQ = dO W_s^T + P1 K                      P1[t][s] = -[s <= t] eta_s dO_t . G_s
//     dK = P1^T Q - diag(eta) G X_e^T + dG W_s^T + P2 K + P2^T K
//                                               P2[a][b] = -[chunk(b) < chunk(a)] eta_b dG_a . G_b
// (the token mask s <= t covers the chunk's own triangle and the earlier chunks of dO E^T alike;
// P2 carries dG W_c^T's corrections below the chunk diagonal and, transposed, E X_c^T's above it).
// Only R, dG and the state gradient itself are serial; they stay on the warps.
//
// Inputs the forward produced: G and -E of every token and the state at every stage start,
// written by the forward stage kernel's state-only chain (one launch before this one). With -E as
// the tensor operand the scores come out scaled and negated: P1 = mask(dO (-E)^T),
// P2 = mask(dG (-E)^T), and -diag(eta) G X_e^T = (-E) X_e^T accumulates into dK directly.
//
// Roles (320 threads):
//   * warp 0: TMA producer, a 2-slot ring of one stage each: Q, K, dO, -E [128][64] (128-byte
//     swizzle), W_s [64][64], the rates.
//   * warp 1: owns TMEM, issues every tcgen05.mma (elected lane): S1 = dO (-E)^T, dQ, the P1
//     and X_e parts of dK as soon as the stage's P1 is masked; S2 = dG (-E)^T and the rest of dK
//     once the chain has finished the stage.
//   * warps 2-5 (one TMEM lane quarter each): mask S1 into P1 and S2 into P2 (bf16, shared
//     memory, read K-major for P K and MN-major for P^T Q / P^T K), drain dQ and dK through a
//     shared tile to TMA stores, write deta.
//   * warps 6-9, the chain: each keeps X^T[16 columns, 64] as fp32 m16n8 accumulators (the state
//     gradient's columns are independent) and per chunk, from the last, forms A'^T = K Q^T,
//     R^T = dO^T A' + X^T K^T, dG^T, the chunk's deta partial sums, X^T += dG^T K + dO^T Q;
//     stores dG^T (the MN-major A operand of the stage's products), dV and, at each stage
//     start, bf16(X_e^T). The next chunk's fragments are loaded before this chunk's stores.
// TMEM columns: S1 [0, 128), S2 [128, 256), dQ [256, 320), dK [320, 384).
// Precision: X and every accumulation fp32; W_s, -E, X_e, dG and the masked scores are bf16
// tensor operands (relative error ~2^-9 per operand); deta uses the bf16 -E (or G) rows.
#include <algorithm>
#include <string>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int BD = 64;                 // head dim
constexpr int BC = 16;                 // chunk (the warp-MMA tile height)
constexpr int BR = 128;                // tokens per stage
constexpr int BKS = BD / 16;           // 16-wide k-steps over d
constexpr int TILE = BR * BD * 2;      // [128][64] bf16
constexpr int WTILE = BD * BD * 2;     // [64][64] bf16
// one ring slot
constexpr int SL_Q = 0, SL_K = TILE, SL_DO = 2 * TILE, SL_NE = 3 * TILE, SL_W = 4 * TILE;
constexpr int SL_ETA = SL_W + WTILE;   // 128 fp32 rates
constexpr int SL_DETA = SL_ETA + 512;  // [4 chain warps][128] fp32 deta partial sums
constexpr int SLOT = (SL_DETA + 4 * 512 + 1023) / 1024 * 1024;
constexpr int P_OFF = 2 * SLOT;        // P1 / P2 [128][128] bf16 (two [128][64] blocks); staging
constexpr int DG_OFF = P_OFF + 2 * TILE;   // dG^T of a stage, x2: [2 token blocks][64][64]
constexpr int DG_BYTES = TILE;
constexpr int XE_OFF = DG_OFF + 2 * DG_BYTES;   // bf16 X_e^T [64][64]
constexpr int BAR_OFF = XE_OFF + WTILE;
constexpr int SMEM = 1024 + BAR_OFF + 256;
constexpr int THREADS = 320;
constexpr float kTinyRate = 1e-20f;   // below it deta is formed from G, not from -E / eta
constexpr int PRODUCER = 0, MMA = 1, EPI0 = 2, CHAIN0 = 6;
constexpr uint32_t TM_S1 = 0, TM_S2 = 128, TM_DQ = 256, TM_DK = 320, TM_COLS = 512;
static_assert(SLOT % 1024 == 0 && P_OFF % 1024 == 0 && DG_OFF % 1024 == 0 &&
                  XE_OFF % 1024 == 0, "1024-byte aligned operand tiles");
static_assert(SMEM <= 227 * 1024, "shared memory");

struct DbtParams {
  const float* eta;     // [streams, T] or nullptr (eta_scalar)
  float eta_scalar;
  const float* dW_out;  // [streams, 64, 64] or nullptr
  const uint16_t* G;    // [streams, T, 64] bf16 residual rows of the forward
  float* dW0;
  float* deta;
  uint16_t* dV;
  int T;
  unsigned* err;
  uint64_t wait_ns;
};

__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t colbyte) {
  return swz<128>(row * 128 + colbyte);
}

__global__ void __launch_bounds__(THREADS, 1)
    dual_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmNE,
                       const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmdQ,
                       const __grid_constant__ CUtensorMap tmdK, const DbtParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + BAR_OFF;
  const uint32_t full = bar, empty = bar + 16;   // ring (x2)
  const uint32_t s1full = bar + 32;   // S1 accumulated (MMA commit)
  const uint32_t p1full = bar + 40;   // P1 written, S1 read (4 epilogue warps)
  const uint32_t dqfull = bar + 48;   // dQ and the P1 part of dK complete (MMA commit)
  const uint32_t dqfree = bar + 56;   // dQ read out of TMEM (4 epilogue warps)
  const uint32_t s2full = bar + 64;   // S2 accumulated (MMA commit)
  const uint32_t p2full = bar + 72;   // P2 written, S2 read (4 epilogue warps)
  const uint32_t dkfull = bar + 80;   // dK complete (MMA commit)
  const uint32_t dkfree = bar + 88;   // dK read out (4 epilogue warps)
  const uint32_t xeready = bar + 96;  // bf16 X_e^T stored (4 chain warps)
  const uint32_t xefree = bar + 104;  // (-E) X_e^T has read it (MMA commit)
  const uint32_t cdone = bar + 112;   // the chain finished a stage: dG^T and deta sums (x2)
  const uint32_t dgfree = bar + 128;  // the stage's products have read dG^T buffer b (x2)
  const uint32_t mdone = bar + 144;   // every MMA issued has completed
  const uint32_t tslot = bar + 160;

  const int stream = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int nst = (T + BR - 1) / BR;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 9);   // MMA commit, 4 chain warps, 4 epilogue warps
      mbar_init(cdone + 8 * s, 4);
      mbar_init(dgfree + 8 * s, 1);
    }
    mbar_init(s1full, 1);
    mbar_init(p1full, 4);
    mbar_init(dqfull, 1);
    mbar_init(dqfree, 4);
    mbar_init(s2full, 1);
    mbar_init(p2full, 4);
    mbar_init(dkfull, 1);
    mbar_init(dkfree, 4);
    mbar_init(xeready, 4);
    mbar_init(xefree, 1);
    mbar_init(mdone, 1);
    fence_mbar_init();
  }
  // Rates and dG^T start at zero: in a partial last stage (processed first) the absent tokens'
  // rates and dG rows are read by the masked products (multiplied by zero rows of G and K), so
  // they must hold finite values.
  for (int s = 0; s < 2; ++s)
    for (int i = threadIdx.x; i < 64; i += THREADS)
      sts128(sbase + s * SLOT + SL_ETA + 16 * i, make_uint4(0u, 0u, 0u, 0u));   // 512 bytes
  for (int i = threadIdx.x; i < 2 * DG_BYTES / 16; i += THREADS)
    sts128(sbase + DG_OFF + 16 * i, make_uint4(0u, 0u, 0u, 0u));
  fence_proxy_async_smem();
  if (warp == MMA) umma::tmem_alloc(tslot, TM_COLS);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + BAR_OFF + 160);

  if (warp == PRODUCER) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmdO);
      prefetch_tmap(&tmNE);
      prefetch_tmap(&tmW);
      int issued = 0;
      for (int i = 0; i < nst; ++i) {
        const int j = nst - 1 - i, sl = i & 1;
        if (i >= 2 && !mbar_wait(empty + 8 * sl, ((i >> 1) - 1) & 1, p.err, p.wait_ns)) break;
        const int rows = min(BR, T - j * BR);
        const uint32_t fb = full + 8 * sl;
        const uint32_t st = sbase + sl * SLOT;
        // a scalar rate is written into the slot, so every consumer reads the slot (the
        // arrival below releases these stores)
        if (!p.eta)
          for (int r = 0; r < BR; ++r) stsf(st + SL_ETA + 4 * r, p.eta_scalar);
        mbar_arrive_expect_tx(fb, 4 * TILE + WTILE + (p.eta ? rows * 4 : 0));
        tma_load_3d(st + SL_Q, &tmQ, fb, 0, j * BR, stream);
        tma_load_3d(st + SL_K, &tmK, fb, 0, j * BR, stream);
        tma_load_3d(st + SL_DO, &tmdO, fb, 0, j * BR, stream);
        tma_load_3d(st + SL_NE, &tmNE, fb, 0, j * BR, stream);
        tma_load_3d(st + SL_W, &tmW, fb, 0, 0, stream * nst + j);
        if (p.eta)
          bulk_load(st + SL_ETA, p.eta + (size_t)stream * T + (size_t)j * BR, rows * 4, fb);
        issued = i + 1;
      }
      // copies still in flight must land before the CTA may exit (normally all have)
      for (int i = max(0, issued - 2); i < issued; ++i)
        mbar_wait(full + 8 * (i & 1), (i >> 1) & 1, p.err, 1000000000ull);
    }
  } else if (warp == MMA) {
    // ------------------------------------------------------------------ tcgen05 issue warp
    // The whole warp runs the loop (warp-uniform waits); an elected lane issues.
    const uint32_t id_s1 = umma::idesc_bf16(128, 128, false, false);   // dO (-E)^T
    const uint32_t id_kk = umma::idesc_bf16(128, 64, false, false);    // dO W_s^T
    const uint32_t id_kn = umma::idesc_bf16(128, 64, false, true);     // P K, (-E) X_e^T
    const uint32_t id_nn = umma::idesc_bf16(128, 64, true, true);      // P^T Q, P^T K
    const uint32_t id_s2 = umma::idesc_bf16(128, 128, true, false);    // dG (-E)^T
    const uint32_t id_nk = umma::idesc_bf16(128, 64, true, false);     // dG W_s^T
    const uint32_t sP = sbase + P_OFF;
    auto slot = [&](int i) -> uint32_t { return sbase + (i & 1) * SLOT; };
    // S1 = dO (-E)^T of stage i
    auto issue_s1 = [&](int i) {
      const uint32_t st = slot(i);
#pragma unroll
      for (int ks = 0; ks < BKS; ++ks)
        umma::mma_ss_elect(tmem + TM_S1, umma::desc_kmajor(st + SL_DO + 32 * ks),
                           umma::desc_kmajor(st + SL_NE + 32 * ks), id_s1, ks > 0);
      umma::commit_elect(s1full);
    };
    // dQ = dO W_s^T + P1 K; dK = P1^T Q + (-E) X_e^T
    auto early = [&](int i) -> bool {
      const uint32_t st = slot(i);
      if (!mbar_wait_warp(p1full, i & 1, p.err, p.wait_ns)) return false;
      if (i >= 1 && !mbar_wait_warp(dqfree, (i - 1) & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
#pragma unroll
      for (int ks = 0; ks < BKS; ++ks)
        umma::mma_ss_elect(tmem + TM_DQ, umma::desc_kmajor(st + SL_DO + 32 * ks),
                           umma::desc_kmajor(st + SL_W + 32 * ks), id_kk, ks > 0);
#pragma unroll
      for (int ks = 0; ks < BR / 16; ++ks)
        umma::mma_ss_elect(tmem + TM_DQ, umma::desc_kmajor(sP + (ks >> 2) * TILE + 32 * (ks & 3)),
                           umma::desc_mnmajor(st + SL_K + 2048 * ks, TILE), id_kn, true);
      if (i >= 1 && !mbar_wait_warp(dkfree, (i - 1) & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
#pragma unroll
      for (int ks = 0; ks < BR / 16; ++ks)
        umma::mma_ss_elect(tmem + TM_DK, umma::desc_mnmajor(sP + 2048 * ks, TILE),
                           umma::desc_mnmajor(st + SL_Q + 2048 * ks, TILE), id_nn, ks > 0);
      umma::commit_elect(dqfull);   // P1 is no longer read
      if (!mbar_wait_warp(xeready, i & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
#pragma unroll
      for (int ks = 0; ks < BKS; ++ks)
        umma::mma_ss_elect(tmem + TM_DK, umma::desc_kmajor(st + SL_NE + 32 * ks),
                           umma::desc_mnmajor(sbase + XE_OFF + 2048 * ks, WTILE), id_kn, true);
      umma::commit_elect(xefree);
      return true;
    };
    // S2 = dG (-E)^T; dK += dG W_s^T + P2 K + P2^T K
    auto late = [&](int i) -> bool {
      const uint32_t st = slot(i);
      const int b = i & 1;
      const uint32_t sDG = sbase + DG_OFF + b * DG_BYTES;
      if (!mbar_wait_warp(cdone + 8 * b, (i >> 1) & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
#pragma unroll
      for (int ks = 0; ks < BKS; ++ks)
        umma::mma_ss_elect(tmem + TM_S2, umma::desc_mnmajor(sDG + 2048 * ks, DG_BYTES / 2),
                           umma::desc_kmajor(st + SL_NE + 32 * ks), id_s2, ks > 0);
      umma::commit_elect(s2full);
#pragma unroll
      for (int ks = 0; ks < BKS; ++ks)
        umma::mma_ss_elect(tmem + TM_DK, umma::desc_mnmajor(sDG + 2048 * ks, DG_BYTES / 2),
                           umma::desc_kmajor(st + SL_W + 32 * ks), id_nk, true);
      if (!mbar_wait_warp(p2full, i & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
#pragma unroll
      for (int ks = 0; ks < BR / 16; ++ks)
        umma::mma_ss_elect(tmem + TM_DK, umma::desc_kmajor(sP + (ks >> 2) * TILE + 32 * (ks & 3)),
                           umma::desc_mnmajor(st + SL_K + 2048 * ks, TILE), id_kn, true);
#pragma unroll
      for (int ks = 0; ks < BR / 16; ++ks)
        umma::mma_ss_elect(tmem + TM_DK, umma::desc_mnmajor(sP + 2048 * ks, TILE),
                           umma::desc_mnmajor(st + SL_K + 2048 * ks, TILE), id_nn, true);
      umma::commit_elect(dkfull);
      umma::commit_elect(empty + 8 * (i & 1));   // the slot's tiles are no longer read
      umma::commit_elect(dgfree + 8 * b);
      return true;
    };
    // Order per iteration: S1 of stage i as soon as its tiles land, then the late products of
    // stage i-1, then the early products of stage i. (Issuing the late products first overlaps
    // more of the pipeline with the chain and measured slower, 0.133 against 0.128 ms: the
    // chain's warp MMAs and shared-memory loads share the SM with the products.)
    bool ok = true;
    for (int i = 0; ok && i < nst; ++i) {
      if (!mbar_wait_warp(full + 8 * (i & 1), (i >> 1) & 1, p.err, p.wait_ns)) break;
      // S1 of the previous stage has been read (its P1 written)
      if (i >= 1 && !mbar_wait_warp(p1full, (i - 1) & 1, p.err, p.wait_ns)) break;
      umma::fence_after();
      issue_s1(i);
      if (i >= 1 && !late(i - 1)) break;
      ok = early(i);
      if (ok && i + 1 == nst) ok = late(i);
    }
    // every MMA this warp issued completes before TMEM is released
    umma::commit_elect(mdone);
    mbar_wait_warp(mdone, 0, p.err, 1000000000ull);
  } else if (warp < CHAIN0) {
    // ------------------------------------------------------------------ epilogue warps
    const int q = warp & 3;                    // TMEM lane quarter: rows 32q .. 32q+31
    const int r = 32 * q + lane;               // stage row: query token t of S1, key s of S2
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int etid = threadIdx.x - 32 * EPI0;  // 0..127
    const uint32_t sP = sbase + P_OFF;
    // Both masks keep a 32-column group [c0, c0+32) for every row of this warp when c0 < 32q,
    // for none when c0 > 32q, and row by row in the group c0 = 32q (keep(col) decides there):
    // the query mask s <= t of P1 and the chunk mask chunk(t) < chunk(s) of P2 alike.
    auto group_mode = [&](int c0) { return c0 < 32 * q ? 1 : (c0 == 32 * q ? 2 : 0); };
    // P[r][:] = S[r][col] where kept, else 0, from the fp32 scores in TMEM columns
    // col0 .. col0+127 (already scaled and negated by the -E operand), as bf16 into the two
    // [128][64] blocks of the P tile. Groups masked for every row are not loaded.
    auto mask_rows = [&](uint32_t col0, auto keep) {
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        const int m0 = group_mode(64 * kb), m1 = group_mode(64 * kb + 32);   // warp-uniform
        uint32_t v[2][32];
        if (m0 != 0) umma::ld32x32(tmem + tl + col0 + 64 * kb, v[0]);
        if (m1 != 0) umma::ld32x32(tmem + tl + col0 + 64 * kb + 32, v[1]);
        if (m0 != 0) {
          umma::wait_ld();
          umma::reg_fence(v[0]);
          umma::reg_fence(v[1]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int m = h ? m1 : m0;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int x0 = 32 * h + 8 * k4;   // column within the block
            uint4 out = make_uint4(0u, 0u, 0u, 0u);
            if (m != 0) {
              uint32_t w[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                float a0 = __uint_as_float(v[h][8 * k4 + 2 * u]);
                float a1 = __uint_as_float(v[h][8 * k4 + 2 * u + 1]);
                if (m == 2) {
                  if (!keep(64 * kb + x0 + 2 * u)) a0 = 0.f;
                  if (!keep(64 * kb + x0 + 2 * u + 1)) a1 = 0.f;
                }
                w[u] = pack_bf16(a0, a1);
              }
              out = make_uint4(w[0], w[1], w[2], w[3]);
            }
            sts128(sP + kb * TILE + swz128(r, 16 * (4 * h + k4)), out);
          }
        }
      }
      fence_proxy_async_smem();
      umma::fence_before();
      __syncwarp();
    };
    // 64 fp32 columns of TMEM row r -> bf16 -> the staging tile (P block 0) -> TMA store
    auto stage_out = [&](const uint32_t (&v)[64], const CUtensorMap* tmap, int j) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        sts128(sP + swz128(r, 16 * k),
               make_uint4(pack_bf16(__uint_as_float(v[8 * k]), __uint_as_float(v[8 * k + 1])),
                          pack_bf16(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3])),
                          pack_bf16(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5])),
                          pack_bf16(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7]))));
      fence_proxy_async_smem();
      bar_sync_named(1, 128);
      if (etid == 0) {
        tma_store_3d(tmap, sP, 0, j * BR, stream);
        bulk_commit();
      }
    };
    auto load64 = [&](uint32_t col, uint32_t (&v)[64]) {
      uint32_t a[32], b[32];
      umma::ld32x32(tmem + tl + col, a);
      umma::ld32x32(tmem + tl + col + 32, b);
      umma::wait_ld();
      umma::reg_fence(a);
      umma::reg_fence(b);
#pragma unroll
      for (int x = 0; x < 32; ++x) v[x] = a[x], v[32 + x] = b[x];
    };
    for (int i = 0; i < nst; ++i) {
      const int j = nst - 1 - i, b = i & 1;
      const uint32_t st = sbase + (i & 1) * SLOT;
      // P1 = [s <= t] (dO (-E)^T)[t][s]; the staging tile's last store must have read P
      bool got = mbar_wait_warp(s1full, i & 1, p.err, p.wait_ns);
      if (got && etid == 0) bulk_wait_read<0>();
      if (bar_or_named(1, 128, !got)) break;
      umma::fence_after();
      mask_rows(TM_S1, [&](int s) { return s <= r; });
      if (lane == 0) mbar_arrive(p1full);
      // dQ
      got = mbar_wait_warp(dqfull, i & 1, p.err, p.wait_ns);
      if (bar_or_named(1, 128, !got)) break;
      umma::fence_after();
      {
        uint32_t v[64];
        load64(TM_DQ, v);
        umma::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dqfree);
        stage_out(v, &tmdQ, j);
      }
      // P2 = [chunk(t) < chunk(s)] (dG (-E)^T)[s][t]
      got = mbar_wait_warp(s2full, i & 1, p.err, p.wait_ns);
      if (got) got = mbar_wait_warp(cdone + 8 * b, (i >> 1) & 1, p.err, p.wait_ns);
      if (got && etid == 0) bulk_wait_read<0>();
      if (bar_or_named(1, 128, !got)) break;
      umma::fence_after();
      mask_rows(TM_S2, [&](int t) { return (t >> 4) < (r >> 4); });
      if (lane == 0) mbar_arrive(p2full);
      // deta of the stage (the four chain warps' partial sums, in a fixed order)
      if (j * BR + r < T)
        p.deta[(size_t)stream * T + (size_t)j * BR + r] =
            ((ldsf(st + SL_DETA + 4 * r) + ldsf(st + SL_DETA + 512 + 4 * r)) +
             ldsf(st + SL_DETA + 1024 + 4 * r)) + ldsf(st + SL_DETA + 1536 + 4 * r);
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + 8 * (i & 1));
      // dK
      got = mbar_wait_warp(dkfull, i & 1, p.err, p.wait_ns);
      if (bar_or_named(1, 128, !got)) break;
      umma::fence_after();
      {
        uint32_t v[64];
        load64(TM_DK, v);
        umma::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dkfree);
        stage_out(v, &tmdK, j);
      }
    }
    if (etid == 0) bulk_wait<0>();
  } else {
    // ------------------------------------------------------------------ chain warps
    const int cw = warp - CHAIN0;
    const int g = lane >> 2, tq = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;   // ldmatrix / stmatrix: matrix, row
    const int colw = 16 * cw;                  // this warp's 16 columns of X (and of dG, dV)
    // Fragment offsets in the [128][64] tiles (128-byte swizzle), relative to a chunk's rows:
    // rows as the B operand of (.) x^T (K and Q), via ldmatrix.trans as the B operand of the
    // state update (K and Q), and via ldmatrix.trans this warp's 16 columns as an A operand (dO^T
    // and (-E)^T). (Transposing the row fragments in registers with movmatrix instead of the
    // second ldmatrix pass measured slower: 159 against 129 us per call.)
    uint32_t o_brow[BKS], o_btrn[BKS];
#pragma unroll
    for (int ks = 0; ks < BKS; ++ks) {
      o_brow[ks] = swz128(8 * (mi >> 1) + rr, 2 * (16 * ks + 8 * (mi & 1)));
      o_btrn[ks] = swz128(8 * (mi & 1) + rr, 2 * (16 * ks + 8 * (mi >> 1)));
    }
    const uint32_t o_at = swz128(8 * (mi >> 1) + rr, 2 * (colw + 8 * (mi & 1)));
    // stmatrix targets in the [64 rows][64] tiles of X_e^T and dG^T: row colw + 8 (mi & 1) + rr,
    // column offset 8 (mi >> 1) within a 16-wide step
    const int srow = colw + 8 * (mi & 1) + rr;
    const int scol = 8 * (mi >> 1);
    constexpr uint32_t CHUNK_BYTES = BC * 128;

    // X^T[colw .. colw+15, :] as m16n8 fp32 accumulators; tile jt holds columns 8jt .. 8jt+7
    // of X^T (rows of X).
    float xc[BD / 8][4];
    {
      const float* x0 = p.dW_out ? p.dW_out + (size_t)stream * BD * BD : nullptr;
#pragma unroll
      for (int jt = 0; jt < BD / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          xc[jt][e] = x0 ? x0[row * BD + colw + g] : 0.f;
          xc[jt][2 + e] = x0 ? x0[row * BD + colw + g + 8] : 0.f;
        }
    }
    bool ok = true;
    for (int i = 0; i < nst; ++i) {
      const int j = nst - 1 - i, b = i & 1;
      const uint32_t st = sbase + (i & 1) * SLOT;
      const uint32_t sQ = st + SL_Q, sK = st + SL_K, sdO = st + SL_DO;
      const uint32_t sEta = st + SL_ETA, sDeta = st + SL_DETA;
      const uint32_t sDG = sbase + DG_OFF + b * DG_BYTES;
      bool got = mbar_wait_warp(full + 8 * (i & 1), (i >> 1) & 1, p.err, p.wait_ns);
      if (got && i >= 1) got = mbar_wait_warp(xefree, (i - 1) & 1, p.err, p.wait_ns);
      if (!got) {
        ok = false;
        break;
      }
      // bf16(X_e^T): the B operand (MN-major) of the stage's (-E) X_e^T
#pragma unroll
      for (int ks = 0; ks < BKS; ++ks)
        stsm_x4(sbase + XE_OFF + swz128(srow, 2 * (16 * ks + scol)),
                pack_bf16(xc[2 * ks][0], xc[2 * ks][1]), pack_bf16(xc[2 * ks][2], xc[2 * ks][3]),
                pack_bf16(xc[2 * ks + 1][0], xc[2 * ks + 1][1]),
                pack_bf16(xc[2 * ks + 1][2], xc[2 * ks + 1][3]));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(xeready);
      // dG^T buffer b was last read by the products of stage i-2
      if (i >= 2 && !mbar_wait_warp(dgfree + 8 * b, ((i >> 1) - 1) & 1, p.err, p.wait_ns)) {
        ok = false;
        break;
      }
      const int chunks = min(BR, T - j * BR) / BC;
      uint16_t* dv = p.dV + ((size_t)stream * T + (size_t)j * BR) * BD;
      const uint16_t* gst = p.G + ((size_t)stream * T + (size_t)j * BR) * BD + colw + g;
      const uint32_t sNE = st + SL_NE;
      struct Ops {
        uint32_t kb[BKS][4], qb[BKS][4], kt[BKS][4], qt[BKS][4], dot[4], ne[4];
        float e0, e1, e8, e9;
      };
      auto load = [&](Ops& o, const int c) {
        const uint32_t cb = c * CHUNK_BYTES;
#pragma unroll
        for (int ks = 0; ks < BKS; ++ks) {
          ldsm_x4(sK + cb + o_brow[ks], o.kb[ks]);
          ldsm_x4(sQ + cb + o_brow[ks], o.qb[ks]);
        }
        ldsm_x4_t(sdO + cb + o_at, o.dot);
        ldsm_x4_t(sNE + cb + o_at, o.ne);
#pragma unroll
        for (int ks = 0; ks < BKS; ++ks) {
          ldsm_x4_t(sK + cb + o_btrn[ks], o.kt[ks]);
          ldsm_x4_t(sQ + cb + o_btrn[ks], o.qt[ks]);
        }
        o.e0 = ldsf(sEta + 4 * (16 * c + 2 * tq));
        o.e1 = ldsf(sEta + 4 * (16 * c + 2 * tq + 1));
        o.e8 = ldsf(sEta + 4 * (16 * c + 8 + 2 * tq));
        o.e9 = ldsf(sEta + 4 * (16 * c + 9 + 2 * tq));
      };
      // G[s][j] of chunk c at the R^T fragment's positions (j = colw + g (+8), s = 16c + 2tq
      // (+1) (+8)) as raw bf16 bits, for chunks with a rate too small to divide by
      auto load_g = [&](uint32_t (&gq)[8], const int c) {
        const uint16_t* gp = gst + (size_t)(16 * c + 2 * tq) * BD;
        gq[0] = __ldg(gp);
        gq[1] = __ldg(gp + BD);
        gq[2] = __ldg(gp + 8);
        gq[3] = __ldg(gp + BD + 8);
        gq[4] = __ldg(gp + 8 * BD);
        gq[5] = __ldg(gp + 9 * BD);
        gq[6] = __ldg(gp + 8 * BD + 8);
        gq[7] = __ldg(gp + 9 * BD + 8);
      };
      auto gval = [](uint32_t x) { return __uint_as_float(x << 16); };
      struct Res {
        uint32_t n[4];   // bf16 dG^T fragments
        float d[4];      // deta partial sums of s = 2tq, 2tq+1, 8+2tq, 9+2tq (lanes g = 0)
      };
      // slow_c: the stage holds a rate too small to divide by (see deta below)
      auto compute = [&](const Ops& o, const int c, Res& res, auto slow_c) {
        // A'^T = K Q^T (rows: keys s, columns: queries t), kept where s <= t. The K rows loaded
        // as B fragments are the A fragments of K in another register order.
        float at[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < BKS; ++ks) {
          mma16816(at[0], o.kb[ks][0], o.kb[ks][2], o.kb[ks][1], o.kb[ks][3], o.qb[ks][0],
                   o.qb[ks][1]);
          mma16816(at[1], o.kb[ks][0], o.kb[ks][2], o.kb[ks][1], o.kb[ks][3], o.qb[ks][2],
                   o.qb[ks][3]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int t = 8 * nt + 2 * tq;
          if (g > t) at[nt][0] = 0.f;
          if (g > t + 1) at[nt][1] = 0.f;
          if (g + 8 > t) at[nt][2] = 0.f;
          if (g + 8 > t + 1) at[nt][3] = 0.f;
        }
        // the A'^T accumulators are the B fragments of A' (k = query t, n = key s)
        const uint32_t ba0[2] = {pack_bf16(at[0][0], at[0][1]), pack_bf16(at[1][0], at[1][1])};
        const uint32_t ba1[2] = {pack_bf16(at[0][2], at[0][3]), pack_bf16(at[1][2], at[1][3])};
        // R^T = dO^T A' + X^T K^T (two accumulators halve the dependent chain)
        float ra[2][4] = {}, rb[2][4] = {};
        mma16816(ra[0], o.dot[0], o.dot[1], o.dot[2], o.dot[3], ba0[0], ba0[1]);
        mma16816(ra[1], o.dot[0], o.dot[1], o.dot[2], o.dot[3], ba1[0], ba1[1]);
#pragma unroll
        for (int ks = 0; ks < BKS; ++ks) {
          const uint32_t a0 = pack_bf16(xc[2 * ks][0], xc[2 * ks][1]);
          const uint32_t a1 = pack_bf16(xc[2 * ks][2], xc[2 * ks][3]);
          const uint32_t a2 = pack_bf16(xc[2 * ks + 1][0], xc[2 * ks + 1][1]);
          const uint32_t a3 = pack_bf16(xc[2 * ks + 1][2], xc[2 * ks + 1][3]);
          float (&acc)[2][4] = (ks & 1) ? rb : ra;
          mma16816(acc[0], a0, a1, a2, a3, o.kb[ks][0], o.kb[ks][1]);
          mma16816(acc[1], a0, a1, a2, a3, o.kb[ks][2], o.kb[ks][3]);
        }
        float R[2][4], dg[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const float ea0 = n ? o.e8 : o.e0, ea1 = n ? o.e9 : o.e1;
#pragma unroll
          for (int x = 0; x < 4; ++x) R[n][x] = ra[n][x] + rb[n][x];
          dg[n][0] = -ea0 * R[n][0];
          dg[n][1] = -ea1 * R[n][1];
          dg[n][2] = -ea0 * R[n][2];
          dg[n][3] = -ea1 * R[n][3];
        }
        res.n[0] = pack_bf16(dg[0][0], dg[0][1]);
        res.n[1] = pack_bf16(dg[0][2], dg[0][3]);
        res.n[2] = pack_bf16(dg[1][0], dg[1][1]);
        res.n[3] = pack_bf16(dg[1][2], dg[1][3]);
        // X^T += dG^T K + dO^T Q
#pragma unroll
        for (int jp = 0; jp < BKS; ++jp) {
          mma16816(xc[2 * jp], res.n[0], res.n[1], res.n[2], res.n[3], o.kt[jp][0], o.kt[jp][1]);
          mma16816(xc[2 * jp + 1], res.n[0], res.n[1], res.n[2], res.n[3], o.kt[jp][2],
                   o.kt[jp][3]);
          mma16816(xc[2 * jp], o.dot[0], o.dot[1], o.dot[2], o.dot[3], o.qt[jp][0], o.qt[jp][1]);
          mma16816(xc[2 * jp + 1], o.dot[0], o.dot[1], o.dot[2], o.dot[3], o.qt[jp][2],
                   o.qt[jp][3]);
        }
        // deta_s = -G_s . R_s over this warp's 16 columns (the epilogue adds the four warps'):
        // with the -E = -diag(eta) G fragments this is (-E_s . R_s) / eta_s. A stage holding a
        // rate too small to divide by takes G itself from global memory for those tokens.
        float d0 = bf16_lo(o.ne[0]) * R[0][0] + bf16_lo(o.ne[1]) * R[0][2];
        float d1 = bf16_hi(o.ne[0]) * R[0][1] + bf16_hi(o.ne[1]) * R[0][3];
        float d2 = bf16_lo(o.ne[2]) * R[1][0] + bf16_lo(o.ne[3]) * R[1][2];
        float d3 = bf16_hi(o.ne[2]) * R[1][1] + bf16_hi(o.ne[3]) * R[1][3];
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
          d0 += __shfl_xor_sync(0xffffffffu, d0, m);
          d1 += __shfl_xor_sync(0xffffffffu, d1, m);
          d2 += __shfl_xor_sync(0xffffffffu, d2, m);
          d3 += __shfl_xor_sync(0xffffffffu, d3, m);
        }
        res.d[0] = __fdividef(d0, o.e0);
        res.d[1] = __fdividef(d1, o.e1);
        res.d[2] = __fdividef(d2, o.e8);
        res.d[3] = __fdividef(d3, o.e9);
        if constexpr (decltype(slow_c)::value) {
          uint32_t gq[8];
          load_g(gq, c);
          float g0 = gval(gq[0]) * R[0][0] + gval(gq[2]) * R[0][2];
          float g1 = gval(gq[1]) * R[0][1] + gval(gq[3]) * R[0][3];
          float g2 = gval(gq[4]) * R[1][0] + gval(gq[6]) * R[1][2];
          float g3 = gval(gq[5]) * R[1][1] + gval(gq[7]) * R[1][3];
#pragma unroll
          for (int m = 4; m < 32; m <<= 1) {
            g0 += __shfl_xor_sync(0xffffffffu, g0, m);
            g1 += __shfl_xor_sync(0xffffffffu, g1, m);
            g2 += __shfl_xor_sync(0xffffffffu, g2, m);
            g3 += __shfl_xor_sync(0xffffffffu, g3, m);
          }
          if (fabsf(o.e0) < kTinyRate) res.d[0] = -g0;
          if (fabsf(o.e1) < kTinyRate) res.d[1] = -g1;
          if (fabsf(o.e8) < kTinyRate) res.d[2] = -g2;
          if (fabsf(o.e9) < kTinyRate) res.d[3] = -g3;
        }
      };
      auto store = [&](const Res& res, const int c) {
        // dG^T of chunk c: tokens 16c .. 16c+15 of the stage's [2][64][64] buffer
        stsm_x4(sDG + (c >> 2) * (DG_BYTES / 2) + swz128(srow, 2 * (16 * (c & 3) + scol)),
                res.n[0], res.n[1], res.n[2], res.n[3]);
        if (g == 0) {
          const uint32_t dd = sDeta + cw * 512 + 4 * 16 * c;
          stsf(dd + 4 * (2 * tq), res.d[0]);
          stsf(dd + 4 * (2 * tq + 1), res.d[1]);
          stsf(dd + 4 * (8 + 2 * tq), res.d[2]);
          stsf(dd + 4 * (9 + 2 * tq), res.d[3]);
        }
        // dV = -dG: each 8x8 block transposed in registers into dV rows
        uint16_t* d = dv + (size_t)(16 * c + g) * BD + colw + 2 * tq;
        *reinterpret_cast<uint32_t*>(d) = movm_t(res.n[0]) ^ 0x80008000u;
        *reinterpret_cast<uint32_t*>(d + 8) = movm_t(res.n[1]) ^ 0x80008000u;
        *reinterpret_cast<uint32_t*>(d + 8 * BD) = movm_t(res.n[2]) ^ 0x80008000u;
        *reinterpret_cast<uint32_t*>(d + 8 * BD + 8) = movm_t(res.n[3]) ^ 0x80008000u;
      };
      // a rate too small to divide by anywhere in the stage (absent tokens' rates are zero and
      // are never divided by: their chunks are not processed)
      bool slow = false;
#pragma unroll
      for (int x = 0; x < 4; ++x)
        slow |= 4 * lane + x < chunks * BC && fabsf(ldsf(sEta + 4 * (4 * lane + x))) < kTinyRate;
      slow = __any_sync(0xffffffffu, slow);
      if (chunks == BR / BC && !slow) {
        // software pipeline: chunk c's products, then chunk c-1's fragments, then chunk c's
        // stores
        Ops o[2];
        load(o[1], BR / BC - 1);
#pragma unroll
        for (int c = BR / BC - 1; c >= 0; --c) {
          Res res;
          compute(o[c & 1], c, res, std::false_type{});
          if (c >= 1) load(o[(c - 1) & 1], c - 1);
          store(res, c);
        }
      } else {
#pragma unroll 1
        for (int c = chunks - 1; c >= 0; --c) {
          Ops o;
          load(o, c);
          Res res;
          if (slow)
            compute(o, c, res, std::true_type{});
          else
            compute(o, c, res, std::false_type{});
          store(res, c);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(cdone + 8 * b);
        mbar_arrive(empty + 8 * (i & 1));
      }
    }
    if (ok) {
      float* x0 = p.dW0 + (size_t)stream * BD * BD;
#pragma unroll
      for (int jt = 0; jt < BD / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          x0[row * BD + colw + g] = xc[jt][e];
          x0[row * BD + colw + g + 8] = xc[jt][2 + e];
        }
    }
  }
  umma::fence_before();
  __syncthreads();
  if (warp == MMA) umma::tmem_dealloc(tmem, TM_COLS);
}

}  // namespace

size_t dual_bwd_stage_workspace_bytes(int B, int H, int T) {
  const size_t bh = (size_t)B * H;
  return 2 * bh * T * BD * 2 + bh * ((T + BR - 1) / BR) * BD * BD * 2;   // -E, G, W_s
}

int launch_dual_bwd_stage(const AssocBwdArgs& a, const LaunchCtx& ctx) {
  if (!(a.d == BD && a.C == BC)) {
    *ctx.msg = "dual bwd (stage form): d = 64, C = 16 only";
    return kUnsupported;
  }
  if (a.ws_bytes < dual_bwd_stage_workspace_bytes(a.B, a.H, a.T)) {
    *ctx.msg = "dual bwd (stage form): workspace too small";
    return kWorkspace;
  }
  const int BH = a.B * a.H, T = a.T, nst = (T + BR - 1) / BR;
  uint16_t* NE = static_cast<uint16_t*>(a.ws);
  uint16_t* G = NE + (size_t)BH * T * BD;
  uint16_t* Ws = G + (size_t)BH * T * BD;
  // the forward's residuals and stage-start states: the stage kernel's state-only chain
  StateArgs f{a.K, a.K, a.V, a.eta, a.eta_scalar, a.S0, nullptr, nullptr, a.B, a.H, a.T, a.d,
              BC, 1, nullptr, 0};
  int st = launch_dual_tc_stage_checkpoints(f, Ws, G, NE, ctx);
  if (st != kOk) return st;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  const uint64_t dims[3] = {(uint64_t)BD, (uint64_t)T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)BD * 2, (uint64_t)T * BD * 2};
  const uint32_t box[3] = {(uint32_t)BD, (uint32_t)BR, 1};
  const uint64_t wdims[3] = {(uint64_t)BD, (uint64_t)BD, (uint64_t)BH * nst};
  const uint64_t wstrides[2] = {(uint64_t)BD * 2, (uint64_t)BD * BD * 2};
  const uint32_t wbox[3] = {(uint32_t)BD, (uint32_t)BD, 1};
  CUtensorMap tq, tk, tdo, tne, tw, tdq, tdk;
  if (!make_tmap_3d(&tq, a.Q, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tk, a.K, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tdo, a.dO, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tne, NE, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tw, Ws, bf, wdims, wstrides, wbox, sw, ctx.msg) ||
      !make_tmap_3d(&tdq, a.dQ, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tdk, a.dK, bf, dims, strides, box, sw, ctx.msg))
    return kCuda;
  cudaError_t e = cudaFuncSetAttribute(dual_bwd_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  const int limit = tuning(kTuneWaitLimitNs);
  DbtParams p{a.eta, a.eta_scalar, a.dS_out, G, a.dS0, a.deta, static_cast<uint16_t*>(a.dV), T,
              ctx.err, limit > 0 ? (uint64_t)limit : 4000000000ull};
  dual_bwd_tc_kernel<<<BH, THREADS, SMEM, ctx.stream>>>(tq, tk, tdo, tne, tw, tdq, tdk, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual bwd (stage form) launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace ttt
