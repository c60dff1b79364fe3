// TTT-Linear mini-batch dual form, bf16 inputs, d = 64, chunk C = 16, 32 or 64, with the state
// resident in TMEM and the serial chain reduced to 16 x 16 Gram-block updates.
//
// Computes, per (batch, head) stream and chunk c (source: "RNN의 기억을 작은 모델로 바꾼다면:
// Test-Time Training 읽기", section "gradient를 효율적인 layer로 만드는 작업" for the mini-batch
// update and its dual form; section "읽는 동안 문제를 하나 더 푼다" for reading the updated model):
//     G_c = K_c W - V_c,   E_c = diag(eta_c) G_c
//     O_c = Q_c W - tril(Q_c K_c^T) E_c
//     W   = W - K_c^T E_c
//
// Stage form. A pipeline stage holds R = 128 tokens, split into 16-token sub-chunks u = 0 .. 7.
// With W_s the state at the stage's start, the state at the start of sub-chunk u is
// W_s - sum_{u' before u} K_u'^T E_u', so the residual of sub-chunk u is
//     G_u = (K_u W_s - V_u) - sum_{u'} (K_u K_u'^T) E_u'     (u' in earlier chunks of the stage)
// and E_u = diag(eta_u) G_u. Only the 16 x 16 blocks of the stage's key Gram matrix
// A = K K^T couple the sub-chunks: the serial chain is a blocked forward substitution with one
// 16 x 16 x 16 product per later sub-chunk (right-looking: as soon as E_u is known it is folded
// into every later residual, the next sub-chunk's first). Everything else is a 128-row product
// per stage on the 5th-generation tensor core:
//     X^T   = W_s^T K^T                  (M = 64 columns of W, N = 128 tokens, K = 64)
//     A     = K K^T                      (M = N = 128 tokens, K = 64)
//     S     = Q K^T                      (M = N = 128 tokens, K = 64)
//     O     = Q W_s - tril(S) E          (M = 128 tokens, N = 64, K = 64 and 128)
//     W^T  += (-E^T) K                   (M = 64, N = 64, K = 128; the state accumulates in TMEM)
// With C = 16 CM, the CM sub-chunks of one chunk all take their residual at the chunk's start
// (one gradient step per chunk), so only blocks between different chunks enter the chain.
//
// Roles (one CTA per stream, 10 warps):
//   * chain warps 0 .. 3: warp w owns columns 16w .. 16w+15 of W. Per stage it reads its rows of
//     X^T from TMEM as mma.sync accumulator fragments (the M = 64 accumulator puts rows
//     16w .. 16w+15 in lanes 32w .. 32w+15, the warp's own subpartition), subtracts V^T, and runs
//     the substitution on mma.sync: E_u^T = eta (.) R_u^T, then R_u'^T += (-E_u^T) A_{u,u'} for
//     later u'. It stores -E^T (bf16) for the tensor-core products, and after the stage's state
//     update reads W^T back from TMEM to store bf16(W_{s+1}^T), the operand of the next stage.
//   * warp 4: TMA producer (3-stage ring of Q/K/V tiles [128 tokens][64] and the rates).
//   * warp 5: owns TMEM and issues every tcgen05.mma from an elected lane.
//   * warps 6 .. 9 (one per TMEM lane quarter): write the Gram blocks the chain needs as bf16
//     16 x 16 tiles into shared memory, mask S into the bf16 P (TMEM to TMEM), and drain O
//     through a shared tile to TMA stores.
// The critical path of a stage is the chain, the state update, the state read-back and X^T of
// the next stage; the other products are issued while a chain runs. Each 128-row product reads
// its operands from shared memory at about 128 bytes per cycle, the bound of the whole SM's
// shared-memory traffic, so they start only once the chain is past its first sub-chunks.
// TMEM columns: S [0, 128), A and X^T (time-shared) [128, 256), P [256, 320),
// O (x2) [320, 448), W^T [448, 512).
// Precision: W is fp32 in TMEM throughout. The residuals use bf16(W_s), bf16 keys, bf16 Gram
// blocks and bf16 E with fp32 accumulation; the outputs use bf16(W_s), bf16 scores and bf16 E.
#include <algorithm>
#include <string>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int GD = 64;              // head dim
constexpr int GR = 128;             // tokens per stage
constexpr int GU = GR / 16;         // 16-token sub-chunks per stage
constexpr int GNSTAGE = 3;
constexpr int GTILE = GR * GD * 2;  // one [128][64] bf16 tile, 128-byte swizzle
constexpr int GSTAGE_BYTES = 3 * GTILE + 1024;   // Q, K, V, rates (512 B, padded)
constexpr int GE_SUB = GD * 128;    // [64 columns][64 tokens] bf16 sub-tile of -E^T
constexpr int GE_BYTES = 2 * GE_SUB;
constexpr int GW_BYTES = GD * 128;  // bf16 W_s^T [64][64]
constexpr int GNBLK = GU * (GU - 1) / 2;   // Gram blocks (u, u') with u < u'
constexpr int GA_BYTES = GNBLK * 512;
constexpr int GO_BYTES = GR * GD * 2;   // bf16 output tile [128][64], 128-byte swizzle
constexpr int GE_OFF = GNSTAGE * GSTAGE_BYTES;
constexpr int GW_OFF = GE_OFF + GE_BYTES;
constexpr int GO_OFF = GW_OFF + GW_BYTES;
constexpr int GA_OFF = GO_OFF + GO_BYTES;
constexpr int GBAR_OFF = GA_OFF + 2 * GA_BYTES;
constexpr int GSMEM = 1024 + GBAR_OFF + 256;
constexpr int GTHREADS = 320;
constexpr int GPRODUCER = 4, GMMA = 5, GEPI0 = 6;
// The chain's progress mark (a sub-chunk of the stage) after which the products off its path
// are issued: 0 and 2 measured within 1% of each other on the 125M- and 1.3B-layer shapes, 4
// about 5% slower (the products then overlap the next state update).
constexpr int GMID = 2;
constexpr uint32_t GTM_S = 0, GTM_A = 128, GTM_P = 256, GTM_O = 320, GTM_W = 448;
constexpr uint32_t GTM_COLS = 512;
static_assert(GSMEM <= 227 * 1024, "shared memory");
static_assert(GE_OFF % 1024 == 0 && GW_OFF % 1024 == 0 && GO_OFF % 1024 == 0 &&
                  GA_OFF % 1024 == 0,
              "alignment");

struct GramParams {
  const float* eta;
  float eta_scalar;
  const float* W0;
  float* Wout;
  int T;
  unsigned* err;
  uint64_t wait_ns;
};

// Byte offset inside a TMA-swizzled tile with 128-byte rows.
__device__ __forceinline__ uint32_t gswz(uint32_t row, uint32_t colbyte) {
  return swz<128>(row * 128 + colbyte);
}
// Gram block (u, v), u < v: a 16 x 16 bf16 tile, row = token of sub-chunk v, column = token of
// sub-chunk u, 32 bytes per row; the two 16-byte halves of rows 4..7 and 12..15 are swapped so
// that an 8-row ldmatrix touches every bank once.
__device__ __forceinline__ uint32_t gblk(int u, int v) { return 512u * (v * (v - 1) / 2 + u); }
__device__ __forceinline__ uint32_t gblk_row(int r, int half) {
  return 32u * r + 16u * (half ^ ((r >> 2) & 1));
}
// bf16(W^T) of the 16 rows a chain warp owns, as m16n8 fragments wc[jt] (columns 8jt .. 8jt+7
// of W^T), into the [64][64] K-major operand tile.
__device__ __forceinline__ void store_wt(uint32_t sW, int srow, int scol, const float (&wc)[8][4]) {
#pragma unroll
  for (int ks = 0; ks < GD / 16; ++ks)
    stsm_x4(sW + gswz(srow, 2 * (16 * ks + scol)), pack_bf16(wc[2 * ks][0], wc[2 * ks][1]),
            pack_bf16(wc[2 * ks][2], wc[2 * ks][3]),
            pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]),
            pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]));
}

template <int CM>
__global__ void __launch_bounds__(GTHREADS, 1)
    dual_gram_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmO, const GramParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + GBAR_OFF;
  const uint32_t full = bar, empty = bar + 8 * GNSTAGE;     // stage ring
  const uint32_t adone = bar + 48;    // A of a stage computed (MMA commit)
  const uint32_t gready = bar + 56;   // A written as bf16 blocks (4 epilogue warps)
  const uint32_t sdone = bar + 64;    // S of a stage computed (MMA commit)
  const uint32_t pready = bar + 72;   // S masked into P (4 epilogue warps)
  const uint32_t xdone = bar + 80;    // X^T computed (MMA commit)
  const uint32_t xfree = bar + 88;    // X^T read by the chain (4 chain warps)
  const uint32_t eready = bar + 96;   // -E^T of the stage stored (4 chain warps)
  const uint32_t wdone = bar + 104;   // state update of the stage complete (MMA commit)
  const uint32_t wready = bar + 112;  // bf16 W_s^T stored (4 chain warps)
  const uint32_t odone = bar + 120;   // O of the stage complete (MMA commit)
  const uint32_t ofree = bar + 128;   // O read out (x2 by TMEM buffer, 4 epilogue warps)
  const uint32_t cmid = bar + 144;    // the chain is past sub-chunk GMID of a stage (4 warps)
  const uint32_t mdone = bar + 152;   // every MMA issued has completed (MMA commit)
  const uint32_t tslot = bar + 160;

  const int stream = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int nst = (T + GR - 1) / GR;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GNSTAGE; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    mbar_init(adone, 1);
    mbar_init(gready, 4);
    mbar_init(sdone, 1);
    mbar_init(pready, 4);
    mbar_init(xdone, 1);
    mbar_init(xfree, 4);
    mbar_init(eready, 4);
    mbar_init(wdone, 1);
    mbar_init(wready, 4);
    mbar_init(odone, 1);
    mbar_init(ofree, 4);
    mbar_init(ofree + 8, 4);
    mbar_init(cmid, 4);
    mbar_init(mdone, 1);
    fence_mbar_init();
  }
  if (warp == GMMA) umma::tmem_alloc(tslot, GTM_COLS);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + GBAR_OFF + 160);

  const uint32_t id_sa = umma::idesc_bf16(128, 128, false, false);  // Q K^T and K K^T
  const uint32_t id_x = umma::idesc_bf16(64, 128, false, false);    // W_s^T K^T
  const uint32_t id_w = umma::idesc_bf16(64, 64, false, true);      // (-E^T) K
  const uint32_t id_o = umma::idesc_bf16(128, 64, false, false);    // Q W_s and P (-E)
  const uint32_t sE = sbase + GE_OFF, sW = sbase + GW_OFF;
  auto stage_q = [&](int j) { return sbase + (j % GNSTAGE) * GSTAGE_BYTES; };

  if (warp == GPRODUCER) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int j = 0; j < nst; ++j) {
        const int s = j % GNSTAGE;
        if (j >= GNSTAGE &&
            !mbar_wait(empty + 8 * s, ((j / GNSTAGE) - 1) & 1, p.err, p.wait_ns))
          break;
        const int rows = min(GR, T - j * GR);
        const uint32_t fb = full + 8 * s;
        const uint32_t st = sbase + s * GSTAGE_BYTES;
        if (!p.eta)
          for (int i = 0; i < GR; ++i) stsf(st + 3 * GTILE + 4 * i, p.eta_scalar);
        mbar_arrive_expect_tx(fb, 3 * GTILE + (p.eta ? rows * 4 : 0));
        tma_load_3d(st, &tmQ, fb, 0, j * GR, stream);
        tma_load_3d(st + GTILE, &tmK, fb, 0, j * GR, stream);
        tma_load_3d(st + 2 * GTILE, &tmV, fb, 0, j * GR, stream);
        if (p.eta)
          bulk_load(st + 3 * GTILE, p.eta + (size_t)stream * T + (size_t)j * GR, rows * 4, fb);
        issued = j + 1;
        // every CTA starts at once: the first stage lands sooner when the ring's other stages
        // are requested after it
        if (j == 0 && !mbar_wait(fb, 0, p.err, p.wait_ns)) break;
      }
      // copies still in flight must land before the CTA may exit (normally all have)
      for (int j = max(0, issued - GNSTAGE); j < issued; ++j)
        mbar_wait(full + 8 * (j % GNSTAGE), (j / GNSTAGE) & 1, p.err, 1000000000ull);
    }
  } else if (warp == GMMA) {
    // ------------------------------------------------------------------ tcgen05 issue warp
    // The whole warp runs the schedule (warp-uniform waits); an elected lane issues, in this
    // order per stage j: the state update of j, S of j+1 (it runs while the chain reads the new
    // state back), X^T of j+1 (the next stage starts when it lands), the output product of j,
    // then -- once the chain of j+1 is past its progress mark -- A of j+2 and Q W_s of j+1,
    // which run while that chain does. The output product of j completes before the chain of
    // j+1 rewrites -E^T (the chain waits for it), and every reader of bf16(W_j^T) is issued
    // before the state update of j, whose completion lets the chain rewrite that tile.
    auto issue_a = [&](int j) -> bool {   // A = K K^T, into the A columns once X^T of j-1 is read
      if (!mbar_wait_warp(full + 8 * (j % GNSTAGE), (j / GNSTAGE) & 1, p.err, p.wait_ns))
        return false;
      umma::fence_after();
      const uint32_t sK = stage_q(j) + GTILE;
#pragma unroll
      for (int ks = 0; ks < GD / 16; ++ks)
        umma::mma_ss_elect(tmem + GTM_A, umma::desc_kmajor(sK + 32 * ks),
                           umma::desc_kmajor(sK + 32 * ks), id_sa, ks > 0);
      umma::commit_elect(adone);
      return true;
    };
    auto issue_s = [&](int j) -> bool {   // S = Q K^T once S of j-1 has been masked
      if (j >= 1 && !mbar_wait_warp(pready, (j - 1) & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
      const uint32_t sQ = stage_q(j), sK = sQ + GTILE;
#pragma unroll
      for (int ks = 0; ks < GD / 16; ++ks)
        umma::mma_ss_elect(tmem + GTM_S, umma::desc_kmajor(sQ + 32 * ks),
                           umma::desc_kmajor(sK + 32 * ks), id_sa, ks > 0);
      umma::commit_elect(sdone);
      return true;
    };
    auto issue_x = [&](int j) -> bool {   // X^T = W_j^T K_j^T once A of j has been read out
      if (!mbar_wait_warp(wready, j & 1, p.err, p.wait_ns)) return false;
      if (!mbar_wait_warp(gready, j & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
      const uint32_t sK = stage_q(j) + GTILE;
#pragma unroll
      for (int ks = 0; ks < GD / 16; ++ks)
        umma::mma_ss_elect(tmem + GTM_A, umma::desc_kmajor(sW + 32 * ks),
                           umma::desc_kmajor(sK + 32 * ks), id_x, ks > 0);
      umma::commit_elect(xdone);
      return true;
    };
    auto issue_o1 = [&](int j) -> bool {  // O = Q W_s into O buffer j&1, drained for stage j-2
      if (j >= 2 && !mbar_wait_warp(ofree + 8 * (j & 1), ((j - 2) >> 1) & 1, p.err, p.wait_ns))
        return false;
      umma::fence_after();
      const uint32_t sQ = stage_q(j);
#pragma unroll
      for (int ks = 0; ks < GD / 16; ++ks)
        umma::mma_ss_elect(tmem + GTM_O + 64 * (j & 1), umma::desc_kmajor(sQ + 32 * ks),
                           umma::desc_kmajor(sW + 32 * ks), id_o, ks > 0);
      return true;
    };
    auto issue_w = [&](int j) -> bool {   // W^T += (-E^T) K_j
      if (!mbar_wait_warp(eready, j & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
      const uint32_t sK = stage_q(j) + GTILE;
#pragma unroll
      for (int ks = 0; ks < GR / 16; ++ks)
        umma::mma_ss_elect(tmem + GTM_W,
                           umma::desc_kmajor(sE + (ks >> 2) * GE_SUB + 32 * (ks & 3)),
                           umma::desc_mnmajor(sK + 2048 * ks, GTILE), id_w, true);
      umma::commit_elect(wdone);
      return true;
    };
    auto issue_o2 = [&](int j) -> bool {  // O += P (-E) once S of j has been masked
      if (!mbar_wait_warp(pready, j & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
#pragma unroll
      for (int ks = 0; ks < GR / 16; ++ks)
        umma::mma_ts_elect(tmem + GTM_O + 64 * (j & 1), tmem + GTM_P + 8 * ks,
                           umma::desc_kmajor(sE + (ks >> 2) * GE_SUB + 32 * (ks & 3)), id_o,
                           true);
      umma::commit_elect(odone);
      umma::commit_elect(empty + 8 * (j % GNSTAGE));   // the stage's tiles are no longer read
      return true;
    };
    bool ok = nst > 0;
    if (ok) ok = issue_a(0) && issue_s(0) && issue_x(0) && issue_o1(0);
    if (ok && nst > 1) ok = mbar_wait_warp(xfree, 0, p.err, p.wait_ns) && issue_a(1);
    for (int j = 0; ok && j < nst; ++j) {
      if (!issue_w(j)) break;
      // S of j+1 runs while the chain reads the new state back
      if (j + 1 < nst && !(issue_s(j + 1) && issue_x(j + 1))) break;
      if (!issue_o2(j)) break;
      if (j + 2 < nst &&
          !(mbar_wait_warp(cmid, (j + 1) & 1, p.err, p.wait_ns) &&
            mbar_wait_warp(xfree, (j + 1) & 1, p.err, p.wait_ns) && issue_a(j + 2)))
        break;
      if (j + 1 < nst && !issue_o1(j + 1)) break;
    }
    // every MMA this warp issued completes before TMEM is released
    umma::commit_elect(mdone);
    mbar_wait_warp(mdone, 0, p.err, 1000000000ull);
  } else if (warp >= GEPI0) {
    // ------------------------------------------------------------------ epilogue warps
    const int q = warp & 3;                  // TMEM lane quarter: rows 32q .. 32q+31
    const int t = 32 * q + lane;             // token row within the stage
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int vrow = t >> 4, r16 = t & 15;   // sub-chunk of the row, row inside it
    // Stage j: masked scores P[t][s] = S[t][s] for s <= t, else 0 (bf16 pairs, TMEM to TMEM),
    // and the Gram blocks (u, vrow), u < vrow, as bf16 tiles for the chain.
    // The quarter's rows need key groups 0 .. q of S (32 keys each; group q holds the
    // diagonal) and Gram column pairs 0 .. q (32 columns = sub-chunks 2p, 2p+1). TMEM loads are
    // issued two groups at a time, the next pair in flight while the previous one is packed.
    // Words of P for keys 64 pp + 32 g + (0 .. 31), g = 0, 1, from the TMEM group loaded into v
    // (groups past the diagonal may hold anything: every key there is masked).
    // Words of P for keys 64 pp + 32 g + (0 .. 31), g = 0, 1, from the TMEM group loaded into v:
    // below the quarter's diagonal group the scores pass unmasked, above it they are zero, and
    // in the diagonal group key s is kept for s <= t.
    auto pack_scores = [&](const uint32_t (&v)[32], int pp, int g, uint32_t (&w)[32]) {
      const int grp = 2 * pp + g;
      if (grp < q) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[16 * g + i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
      } else if (grp > q) {
#pragma unroll
        for (int i = 0; i < 16; ++i) w[16 * g + i] = 0u;
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int k0 = 2 * i;   // key offsets inside the group: k0, k0 + 1 (kept if <= lane)
          w[16 * g + i] = pack_bf16(k0 <= lane ? __uint_as_float(v[2 * i]) : 0.f,
                                    k0 + 1 <= lane ? __uint_as_float(v[2 * i + 1]) : 0.f);
        }
      }
    };
    // Gram blocks (u, vrow) for u = 2 pr, 2 pr + 1 from the TMEM column pair pr loaded into v.
    auto store_blocks = [&](const uint32_t (&v)[32], int pr, uint32_t sA) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int u = 2 * pr + h;
        if (u < vrow) {
          const uint32_t blk = sA + gblk(u, vrow);
          auto f = [&](int i) { return __uint_as_float(v[16 * h + i]); };
          sts128(blk + gblk_row(r16, 0), make_uint4(pack_bf16(f(0), f(1)), pack_bf16(f(2), f(3)),
                                                    pack_bf16(f(4), f(5)), pack_bf16(f(6), f(7))));
          sts128(blk + gblk_row(r16, 1),
                 make_uint4(pack_bf16(f(8), f(9)), pack_bf16(f(10), f(11)),
                            pack_bf16(f(12), f(13)), pack_bf16(f(14), f(15))));
        }
      }
    };
    // Gram blocks of stage j: column pairs 0, 1, then 2, 3 (the second pair in flight while the
    // first is written out).
    auto gram = [&](int j) -> bool {
      if (!mbar_wait_warp(adone, j & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
      const uint32_t sA = sbase + GA_OFF + GA_BYTES * (j & 1);
      uint32_t a0[32], a1[32], c0[32], c1[32];
      // (every quarter loads all four pairs: conditionally written load registers make the
      // compiler spill; the blocks a quarter does not own are skipped when storing)
      umma::ld32x32(tmem + tl + GTM_A, a0);
      umma::ld32x32(tmem + tl + GTM_A + 32, a1);
      umma::wait_ld();
      umma::reg_fence(a0);
      umma::reg_fence(a1);
      umma::ld32x32(tmem + tl + GTM_A + 64, c0);
      umma::ld32x32(tmem + tl + GTM_A + 96, c1);
      store_blocks(a0, 0, sA);
      store_blocks(a1, 1, sA);
      umma::wait_ld();
      umma::reg_fence(c0);
      umma::reg_fence(c1);
      store_blocks(c0, 2, sA);
      store_blocks(c1, 3, sA);
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(gready);
      return true;
    };
    // Masked scores of stage j into P (called once the output product of stage j-1, the last
    // reader of P, has completed): keys 0 .. 63, then keys 64 .. 127, which are all masked in
    // the first two quarters (their zeros are written on the first stage only).
    auto mask = [&](int j) -> bool {
      if (!mbar_wait_warp(sdone, j & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        if (pp == 1 && q < 2 && j > 0) break;
        uint32_t a0[32], a1[32], w[32];
        umma::ld32x32(tmem + tl + GTM_S + 64 * pp, a0);
        umma::ld32x32(tmem + tl + GTM_S + 64 * pp + 32, a1);
        umma::wait_ld();
        umma::reg_fence(a0);
        umma::reg_fence(a1);
        pack_scores(a0, pp, 0, w);
        pack_scores(a1, pp, 1, w);
        umma::st32x32(tmem + tl + GTM_P + 32 * pp, w);
      }
      umma::wait_st();
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pready);
      return true;
    };
    // Output of stage j: O accumulator -> bf16 -> shared tile -> one TMA store (a row per
    // thread written straight to global memory would touch 32 lines per store instruction and
    // hold up the chain's shared-memory loads behind it).
    const int etid = threadIdx.x - 32 * GEPI0;   // 0..127
    const uint32_t sO = sbase + GO_OFF;
    auto drain = [&](int j) -> bool {
      const bool got = mbar_wait_warp(odone, j & 1, p.err, p.wait_ns);
      // the previous store has finished reading the staging tile before anyone rewrites it
      if (got && etid == 0) bulk_wait_read<0>();
      if (bar_or_named(1, 128, !got)) return false;
      umma::fence_after();
      uint32_t v[64];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        umma::ld32x32(tmem + tl + GTM_O + 64 * (j & 1) + 32 * h, r);
        umma::wait_ld();
        umma::reg_fence(r);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[32 * h + i] = r[i];
      }
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ofree + 8 * (j & 1));
      auto f = [&](int i) { return __uint_as_float(v[i]); };
#pragma unroll
      for (int k = 0; k < GD / 8; ++k)
        sts128(sO + gswz(t, 16 * k),
               make_uint4(pack_bf16(f(8 * k), f(8 * k + 1)), pack_bf16(f(8 * k + 2), f(8 * k + 3)),
                          pack_bf16(f(8 * k + 4), f(8 * k + 5)),
                          pack_bf16(f(8 * k + 6), f(8 * k + 7))));
      fence_proxy_async_smem();
      bar_sync_named(1, 128);
      if (etid == 0) {
        tma_store_3d(&tmO, sO, 0, j * GR, stream);
        bulk_commit();
      }
      return true;
    };
    // Per stage j: the masked scores of j (the output product of j-1 was drained just before),
    // the Gram blocks of j+1 (wanted by X^T of j+1), then, once the output product of j has
    // completed, its drain.
    bool ok = nst > 0 && gram(0);
    for (int j = 0; ok && j < nst; ++j) {
      ok = mask(j);
      if (ok && j + 1 < nst) ok = gram(j + 1);
      if (ok) ok = drain(j);
    }
    if (etid == 0) bulk_wait<0>();
  } else {
    // ------------------------------------------------------------------ chain warps
    const int g = lane >> 2, tq = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;    // ldmatrix / stmatrix: matrix, row
    const int colw = 16 * warp;                 // first column of W this warp owns
    const uint32_t tlw = (uint32_t)(32 * warp) << 16;
    const int srow = colw + 8 * (mi & 1) + rr;  // stmatrix rows of the [64][...] operand tiles
    const int scol = 8 * (mi >> 1);
    const uint32_t o_vt = gswz(8 * (mi >> 1) + rr, 2 * (colw + 8 * (mi & 1)));
    const uint32_t o_g = gblk_row(8 * (mi >> 1) + rr, mi & 1);
    constexpr uint32_t SUB_BYTES = 16 * 128;    // 16 token rows of a [128][64] tile

    // W^T rows colw .. colw+15 as m16n8 fragments: wc[jt] holds columns 8jt .. 8jt+7 of W^T.
    auto store_wout = [&](const float (&wc)[GD / 8][4]) {
      float* wo = p.Wout + (size_t)stream * GD * GD;
#pragma unroll
      for (int jt = 0; jt < GD / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          wo[row * GD + colw + g] = wc[jt][e];
          wo[row * GD + colw + g + 8] = wc[jt][2 + e];
        }
    };
    {
      float wc[GD / 8][4];
      const float* w0 = p.W0 ? p.W0 + (size_t)stream * GD * GD : nullptr;
#pragma unroll
      for (int jt = 0; jt < GD / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          wc[jt][e] = w0 ? w0[row * GD + colw + g] : 0.f;
          wc[jt][2 + e] = w0 ? w0[row * GD + colw + g + 8] : 0.f;
        }
      uint32_t wr[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) wr[i] = __float_as_uint(wc[i >> 2][i & 3]);
      umma::st16x256b_x8(tmem + tlw + GTM_W, wr);
      umma::wait_st();
      store_wt(sW, srow, scol, wc);
      fence_proxy_async_smem();
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(wready);
      if (nst == 0) store_wout(wc);
    }
    for (int j = 0; j < nst; ++j) {
      const int s = j % GNSTAGE, b = j & 1;
      // warp-uniform waits (the stmatrix stores below need every lane); a wait that runs out
      // leaves W_out unwritten
      bool got = mbar_wait_warp(full + 8 * s, (j / GNSTAGE) & 1, p.err, p.wait_ns);
      if (got) got = mbar_wait_warp(xdone, j & 1, p.err, p.wait_ns);
      if (got) got = mbar_wait_warp(gready, j & 1, p.err, p.wait_ns);
      // the output product of the previous stage has read the -E^T tile this stage rewrites
      if (got && j >= 1) got = mbar_wait_warp(odone, (j - 1) & 1, p.err, p.wait_ns);
      if (!got) break;
      umma::fence_after();
      float R[2 * GU][4];
      {
        uint32_t xr[64];
        umma::ld16x256b_x16(tmem + tlw + GTM_A, xr);
        umma::wait_ld();
        umma::reg_fence_n(xr);
#pragma unroll
        for (int i = 0; i < 64; ++i) R[i >> 2][i & 3] = __uint_as_float(xr[i]);
      }
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(xfree);

      const uint32_t sV = sbase + s * GSTAGE_BYTES + 2 * GTILE;
      const uint32_t sEta = sV + GTILE;
      const uint32_t sA = sbase + GA_OFF + GA_BYTES * b;
      const int rows = min(GR, T - j * GR);
      // Operands of sub-chunk u: V^T fragments, rates (zero past the stream's end) and the Gram
      // blocks (u, v) of the later chunks' sub-chunks; loaded one sub-chunk ahead.
      struct Sub {
        uint32_t vt[4];
        float e[4];
        uint32_t gb[GU][4];
      };
      auto load_sub = [&](Sub& o, const int u) {
        ldsm_x4_t(sV + u * SUB_BYTES + o_vt, o.vt);
        const int t0 = 16 * u + 2 * tq;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tk = t0 + (i & 1) + 8 * (i >> 1);
          o.e[i] = tk < rows ? ldsf(sEta + 4 * tk) : 0.f;
        }
#pragma unroll
        for (int v = (u / CM + 1) * CM; v < GU; ++v) ldsm_x4(sA + gblk(u, v) + o_g, o.gb[v]);
      };
      Sub cur, nxt;
      load_sub(cur, 0);
#pragma unroll
      for (int u = 0; u < GU; ++u) {
        if (u + 1 < GU) load_sub(nxt, u + 1);
        float E[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const float ea0 = cur.e[2 * n], ea1 = cur.e[2 * n + 1];
          E[n][0] = (R[2 * u + n][0] - bf16_lo(cur.vt[2 * n])) * ea0;
          E[n][1] = (R[2 * u + n][1] - bf16_hi(cur.vt[2 * n])) * ea1;
          E[n][2] = (R[2 * u + n][2] - bf16_lo(cur.vt[2 * n + 1])) * ea0;
          E[n][3] = (R[2 * u + n][3] - bf16_hi(cur.vt[2 * n + 1])) * ea1;
        }
        // -E^T of sub-chunk u as the A operand of the updates below
        const uint32_t n0 = pack_bf16(E[0][0], E[0][1]) ^ 0x80008000u;
        const uint32_t n1 = pack_bf16(E[0][2], E[0][3]) ^ 0x80008000u;
        const uint32_t n2 = pack_bf16(E[1][0], E[1][1]) ^ 0x80008000u;
        const uint32_t n3 = pack_bf16(E[1][2], E[1][3]) ^ 0x80008000u;
        // fold E_u into the residuals of the later chunks' sub-chunks, the nearest first
#pragma unroll
        for (int v = (u / CM + 1) * CM; v < GU; ++v) {
          mma16816(R[2 * v], n0, n1, n2, n3, cur.gb[v][0], cur.gb[v][1]);
          mma16816(R[2 * v + 1], n0, n1, n2, n3, cur.gb[v][2], cur.gb[v][3]);
        }
        stsm_x4(sE + (u >> 2) * GE_SUB + gswz(srow, 2 * (16 * (u & 3) + scol)), n0, n1, n2, n3);
        if (u == GMID) {
          __syncwarp();
          if (lane == 0) mbar_arrive(cmid);
        }
        if (u + 1 < GU) cur = nxt;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(eready);

      // the state after the stage: bf16(W^T) for the next stage's products (every product
      // that read the previous tile was issued before the state update)
      if (!mbar_wait_warp(wdone, j & 1, p.err, p.wait_ns)) break;
      umma::fence_after();
      float wc[GD / 8][4];
      {
        uint32_t wr[32];
        umma::ld16x256b_x8(tmem + tlw + GTM_W, wr);
        umma::wait_ld();
        umma::reg_fence_n(wr);
#pragma unroll
        for (int i = 0; i < 32; ++i) wc[i >> 2][i & 3] = __uint_as_float(wr[i]);
      }
      if (j + 1 < nst) {
        store_wt(sW, srow, scol, wc);
        fence_proxy_async_smem();
        umma::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(wready);
      } else {
        store_wout(wc);
      }
    }
  }
  umma::fence_before();
  __syncthreads();
  if (warp == GMMA) umma::tmem_dealloc(tmem, GTM_COLS);
}

template <int CM>
int launch_gram(const StateArgs& a, const LaunchCtx& ctx) {
  const int BH = a.B * a.H;
  CUtensorMap tq, tk, tv, to;
  const uint64_t dims[3] = {(uint64_t)GD, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)GD * 2, (uint64_t)a.T * GD * 2};
  const uint32_t box[3] = {(uint32_t)GD, (uint32_t)GR, 1};
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_tmap_3d(&tq, a.Q, bf, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg) ||
      !make_tmap_3d(&tk, a.K, bf, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg) ||
      !make_tmap_3d(&tv, a.V, bf, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg) ||
      !make_tmap_3d(&to, a.O, bf, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg))
    return kCuda;
  auto kern = dual_gram_kernel<CM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GSMEM);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  const int limit = tuning(kTuneWaitLimitNs);
  GramParams p{a.eta, a.eta_scalar, a.S0, a.S_out, a.T, ctx.err,
               limit > 0 ? (uint64_t)limit : 4000000000ull};
  kern<<<BH, GTHREADS, GSMEM, ctx.stream>>>(tq, tk, tv, to, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual_gram launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

bool dual_gram_supported(int d, int C, int dt) {
  return dt == 1 && d == GD && (C == 16 || C == 32 || C == 64);
}

int launch_dual_gram(const StateArgs& a, const LaunchCtx& ctx) {
  switch (a.C) {
    case 16: return launch_gram<1>(a, ctx);
    case 32: return launch_gram<2>(a, ctx);
    case 64: return launch_gram<4>(a, ctx);
  }
  *ctx.msg = "dual_gram: chunk must be 16, 32 or 64";
  return kUnsupported;
}

}  // namespace ttt
