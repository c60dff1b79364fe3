// TTT-Linear mini-batch dual form, bf16 inputs, d = 64, chunk C = 16, 32 or 64: the state in
// registers, every 128-token stage evaluated as a blocked substitution over the stage's key Gram
// blocks, so that one 16 x 16 product per sub-chunk is all that sits on the serial chain.
//
// Computes, per (batch, head) stream and chunk c (source: "RNN의 기억을 작은 모델로 바꾼다면:
// Test-Time Training 읽기", section "gradient를 효율적인 layer로 만드는 작업" for the mini-batch
// update and its dual form; section "읽는 동안 문제를 하나 더 푼다" for reading the updated model):
//     G_c = K_c W - V_c,   E_c = diag(eta_c) G_c
//     O_c = Q_c W - tril(Q_c K_c^T) E_c
//     W   = W - K_c^T E_c
//
// Stage form. A stage holds 128 tokens, eight 16-token sub-chunks u. With W_s the state at the
// stage's start, the residual of sub-chunk u is
//     G_u = (K_u W_s - V_u) - sum_{u'} (K_u K_u'^T) E_u'       (u' in earlier chunks)
// (the state at u's chunk start is W_s minus the earlier sub-chunks' updates). The chain warps
// hold W^T in fp32 registers, columns split over the warps. Per sub-chunk u, on mma.sync:
//   * X_u^T = W_s^T K_u^T           (8 products; W_s is fixed for the stage, so this is off the
//                                    chain and runs one sub-chunk ahead)
//   * E_u^T = eta (.) (X_u^T + D_u^T - V_u^T), where D_u holds the earlier sub-chunks' Gram
//     corrections; then D_v^T += (-E_u^T) A_{u,v} for the later chunks' sub-chunks v (two
//     products each; the next sub-chunk's first, the only product on the chain)
//   * W^T += (-E_u^T) K_u            (8 products into the fp32 state, off the chain)
// The 5th-generation tensor core computes what depends on the data alone, a stage ahead of the
// chain: A = K K^T (whose 16 x 16 blocks the epilogue writes as bf16 tiles for the chain),
// S = Q K^T, and the outputs O = Q W_s - tril(S) E once the chain has stored W_s and -E.
// No tensor-core round trip sits on the chain.
//
// Roles (one CTA per stream, 10 warps):
//   * chain warps 0 .. 3: warp w owns columns 16w .. 16w+15 of W (rows of W^T, as fp32 m16n8
//     accumulators for the whole sequence); at the end of a stage it stores bf16(W^T) for the
//     next stage's output product and -E^T of every sub-chunk for this stage's.
//   * warp 4: TMA producer (3-stage ring of Q/K/V tiles [128 tokens][64] and the rates).
//   * warp 5: owns TMEM and issues every tcgen05.mma from an elected lane.
//   * warps 6 .. 9 (one per TMEM lane quarter): write the Gram blocks as bf16 16 x 16 tiles into
//     shared memory, mask S into the bf16 P (TMEM to TMEM), and drain O through a shared tile to
//     TMA stores.
// TMEM columns: S [0, 128), A [128, 256), P [256, 320), O (x2) [320, 448).
// Precision: W is fp32 throughout; the residuals use bf16(W_s), bf16 keys, bf16 Gram blocks and
// bf16 E with fp32 accumulation, the state update bf16 E and keys; the outputs use bf16(W_s),
// bf16 scores and bf16 E.
#include <algorithm>
#include <string>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int RD = 64;              // head dim
constexpr int RR = 128;             // tokens per stage
constexpr int RU = RR / 16;         // 16-token sub-chunks per stage
constexpr int RKS = RD / 16;        // 16-wide k-steps over d
constexpr int RNSTAGE = 3;
constexpr int RTILE = RR * RD * 2;  // one [128][64] bf16 tile, 128-byte swizzle
constexpr int RSTAGE_BYTES = 3 * RTILE + 1024;   // Q, K, V, rates (512 B, padded)
constexpr int RE_SUB = RD * 128;    // [64 columns][64 tokens] bf16 sub-tile of -E^T
constexpr int RE_BYTES = 2 * RE_SUB;
constexpr int RW_BYTES = RD * 128;  // bf16 W_s^T [64][64] (x2: stages alternate)
constexpr int RO_BYTES = RR * RD * 2;
constexpr int RNBLK = RU * (RU - 1) / 2;   // Gram blocks (u, v) with u < v
constexpr int RA_BYTES = RNBLK * 512;
constexpr int RE_OFF = RNSTAGE * RSTAGE_BYTES;
constexpr int RW_OFF = RE_OFF + RE_BYTES;
constexpr int RO_OFF = RW_OFF + 2 * RW_BYTES;
constexpr int RA_OFF = RO_OFF + RO_BYTES;
constexpr int RBAR_OFF = RA_OFF + 2 * RA_BYTES;
constexpr int RSMEM = 1024 + RBAR_OFF + 256;
constexpr int RTHREADS = 320;
constexpr int RPRODUCER = 4, RMMA = 5, REPI0 = 6;
constexpr uint32_t RTM_S = 0, RTM_A = 128, RTM_P = 256, RTM_O = 320;
constexpr uint32_t RTM_COLS = 512;
static_assert(RSMEM <= 227 * 1024, "shared memory");
static_assert(RE_OFF % 1024 == 0 && RW_OFF % 1024 == 0 && RO_OFF % 1024 == 0 &&
                  RA_OFF % 1024 == 0,
              "alignment");

struct RgramParams {
  const float* eta;
  float eta_scalar;
  const float* W0;
  float* Wout;
  int T;
  unsigned* err;
  uint64_t wait_ns;
};

// Byte offset inside a TMA-swizzled tile with 128-byte rows.
__device__ __forceinline__ uint32_t rswz(uint32_t row, uint32_t colbyte) {
  return swz<128>(row * 128 + colbyte);
}
// Gram block (u, v), u < v: a 16 x 16 bf16 tile, row = token of sub-chunk v, column = token of
// sub-chunk u, 32 bytes per row; the two 16-byte halves of rows 4..7 and 12..15 are swapped so
// that an 8-row ldmatrix touches every bank once.
__device__ __forceinline__ uint32_t rblk(int u, int v) { return 512u * (v * (v - 1) / 2 + u); }
__device__ __forceinline__ uint32_t rblk_row(int r, int half) {
  return 32u * r + 16u * (half ^ ((r >> 2) & 1));
}

template <int CM>
__global__ void __launch_bounds__(RTHREADS, 1)
    dual_rgram_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmO, const RgramParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + RBAR_OFF;
  const uint32_t full = bar, empty = bar + 8 * RNSTAGE;     // stage ring
  const uint32_t adone = bar + 48;    // A of a stage computed (MMA commit)
  const uint32_t gready = bar + 56;   // A written as bf16 blocks (4 epilogue warps)
  const uint32_t sdone = bar + 64;    // S of a stage computed (MMA commit)
  const uint32_t pready = bar + 72;   // S masked into P (4 epilogue warps)
  const uint32_t eready = bar + 80;   // -E^T of the stage stored (4 chain warps)
  const uint32_t wready = bar + 88;   // bf16 W_s^T of a stage stored (4 chain warps)
  const uint32_t o1done = bar + 96;   // Q W_s complete (x2 by W_s^T buffer, MMA commit)
  const uint32_t odone = bar + 112;   // O of the stage complete (MMA commit)
  const uint32_t ofree = bar + 120;   // O read out (x2 by TMEM buffer, 4 epilogue warps)
  const uint32_t mdone = bar + 136;   // every MMA issued has completed (MMA commit)
  const uint32_t tslot = bar + 144;

  const int stream = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int nst = (T + RR - 1) / RR;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RNSTAGE; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    mbar_init(adone, 1);
    mbar_init(gready, 4);
    mbar_init(sdone, 1);
    mbar_init(pready, 4);
    mbar_init(eready, 4);
    mbar_init(wready, 4);
    mbar_init(o1done, 1);
    mbar_init(o1done + 8, 1);
    mbar_init(odone, 1);
    mbar_init(ofree, 4);
    mbar_init(ofree + 8, 4);
    mbar_init(mdone, 1);
    fence_mbar_init();
  }
  if (warp == RMMA) umma::tmem_alloc(tslot, RTM_COLS);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + RBAR_OFF + 144);

  const uint32_t id_sa = umma::idesc_bf16(128, 128, false, false);  // Q K^T and K K^T
  const uint32_t id_o = umma::idesc_bf16(128, 64, false, false);    // Q W_s and P (-E)
  const uint32_t sE = sbase + RE_OFF;
  auto stage_q = [&](int j) { return sbase + (j % RNSTAGE) * RSTAGE_BYTES; };
  auto stage_w = [&](int j) { return sbase + RW_OFF + RW_BYTES * (j & 1); };

  if (warp == RPRODUCER) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int j = 0; j < nst; ++j) {
        const int s = j % RNSTAGE;
        if (j >= RNSTAGE &&
            !mbar_wait(empty + 8 * s, ((j / RNSTAGE) - 1) & 1, p.err, p.wait_ns))
          break;
        const int rows = min(RR, T - j * RR);
        const uint32_t fb = full + 8 * s;
        const uint32_t st = sbase + s * RSTAGE_BYTES;
        if (!p.eta)
          for (int i = 0; i < RR; ++i) stsf(st + 3 * RTILE + 4 * i, p.eta_scalar);
        mbar_arrive_expect_tx(fb, 3 * RTILE + (p.eta ? rows * 4 : 0));
        tma_load_3d(st, &tmQ, fb, 0, j * RR, stream);
        tma_load_3d(st + RTILE, &tmK, fb, 0, j * RR, stream);
        tma_load_3d(st + 2 * RTILE, &tmV, fb, 0, j * RR, stream);
        if (p.eta)
          bulk_load(st + 3 * RTILE, p.eta + (size_t)stream * T + (size_t)j * RR, rows * 4, fb);
        issued = j + 1;
      }
      // copies still in flight must land before the CTA may exit (normally all have)
      for (int j = max(0, issued - RNSTAGE); j < issued; ++j)
        mbar_wait(full + 8 * (j % RNSTAGE), (j / RNSTAGE) & 1, p.err, 1000000000ull);
    }
  } else if (warp == RMMA) {
    // ------------------------------------------------------------------ tcgen05 issue warp
    // The whole warp runs the schedule (warp-uniform waits); an elected lane issues. Per stage
    // j: A of j+1 (once A of j has been written out as blocks), S of j+1 (once S of j has been
    // masked), the output product of j (once the chain has stored -E^T of j) and Q W_s of j+1
    // (once the chain has stored bf16(W_(j+1)^T) and O buffer (j+1)&1 has been read out). None
    // of these is on the chain: A of j+1 is ready long before the chain of j+1 starts.
    auto issue_a = [&](int j) -> bool {   // A = K K^T into the A columns
      if (!mbar_wait_warp(full + 8 * (j % RNSTAGE), (j / RNSTAGE) & 1, p.err, p.wait_ns))
        return false;
      if (j >= 1 && !mbar_wait_warp(gready, (j - 1) & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
      const uint32_t sK = stage_q(j) + RTILE;
#pragma unroll
      for (int ks = 0; ks < RKS; ++ks)
        umma::mma_ss_elect(tmem + RTM_A, umma::desc_kmajor(sK + 32 * ks),
                           umma::desc_kmajor(sK + 32 * ks), id_sa, ks > 0);
      umma::commit_elect(adone);
      return true;
    };
    auto issue_s = [&](int j) -> bool {   // S = Q K^T (stage j landed: issue_a(j) waited)
      if (j >= 1 && !mbar_wait_warp(pready, (j - 1) & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
      const uint32_t sQ = stage_q(j), sK = sQ + RTILE;
#pragma unroll
      for (int ks = 0; ks < RKS; ++ks)
        umma::mma_ss_elect(tmem + RTM_S, umma::desc_kmajor(sQ + 32 * ks),
                           umma::desc_kmajor(sK + 32 * ks), id_sa, ks > 0);
      umma::commit_elect(sdone);
      return true;
    };
    auto issue_o1 = [&](int j) -> bool {  // O = Q W_s into O buffer j&1
      if (!mbar_wait_warp(wready, j & 1, p.err, p.wait_ns)) return false;
      if (j >= 2 && !mbar_wait_warp(ofree + 8 * (j & 1), ((j - 2) >> 1) & 1, p.err, p.wait_ns))
        return false;
      umma::fence_after();
      const uint32_t sQ = stage_q(j), sW = stage_w(j);
#pragma unroll
      for (int ks = 0; ks < RKS; ++ks)
        umma::mma_ss_elect(tmem + RTM_O + 64 * (j & 1), umma::desc_kmajor(sQ + 32 * ks),
                           umma::desc_kmajor(sW + 32 * ks), id_o, ks > 0);
      umma::commit_elect(o1done + 8 * (j & 1));   // the chain may rewrite this W_s^T tile
      return true;
    };
    auto issue_o2 = [&](int j) -> bool {  // O += P (-E)
      if (!mbar_wait_warp(eready, j & 1, p.err, p.wait_ns)) return false;
      if (!mbar_wait_warp(pready, j & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
#pragma unroll
      for (int ks = 0; ks < RR / 16; ++ks)
        umma::mma_ts_elect(tmem + RTM_O + 64 * (j & 1), tmem + RTM_P + 8 * ks,
                           umma::desc_kmajor(sE + (ks >> 2) * RE_SUB + 32 * (ks & 3)), id_o,
                           true);
      umma::commit_elect(odone);
      umma::commit_elect(empty + 8 * (j % RNSTAGE));   // the stage's tiles are no longer read
      return true;
    };
    bool ok = nst > 0 && issue_a(0) && issue_s(0) && issue_o1(0);
    for (int j = 0; ok && j < nst; ++j) {
      if (j + 1 < nst && !(issue_a(j + 1) && issue_s(j + 1))) break;
      if (!issue_o2(j)) break;
      if (j + 1 < nst && !issue_o1(j + 1)) break;
    }
    // every MMA this warp issued completes before TMEM is released
    umma::commit_elect(mdone);
    mbar_wait_warp(mdone, 0, p.err, 1000000000ull);
  } else if (warp >= REPI0) {
    // ------------------------------------------------------------------ epilogue warps
    const int q = warp & 3;                  // TMEM lane quarter: rows 32q .. 32q+31
    const int t = 32 * q + lane;             // token row within the stage
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int vrow = t >> 4, r16 = t & 15;   // sub-chunk of the row, row inside it
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
          const uint32_t blk = sA + rblk(u, vrow);
          auto f = [&](int i) { return __uint_as_float(v[16 * h + i]); };
          sts128(blk + rblk_row(r16, 0), make_uint4(pack_bf16(f(0), f(1)), pack_bf16(f(2), f(3)),
                                                    pack_bf16(f(4), f(5)), pack_bf16(f(6), f(7))));
          sts128(blk + rblk_row(r16, 1),
                 make_uint4(pack_bf16(f(8), f(9)), pack_bf16(f(10), f(11)),
                            pack_bf16(f(12), f(13)), pack_bf16(f(14), f(15))));
        }
      }
    };
    // Gram blocks of stage j (every quarter loads all four column pairs: conditionally written
    // load registers make the compiler spill; blocks a quarter does not own are skipped)
    auto gram = [&](int j) -> bool {
      if (!mbar_wait_warp(adone, j & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
      const uint32_t sA = sbase + RA_OFF + RA_BYTES * (j & 1);
      uint32_t a0[32], a1[32], c0[32], c1[32];
      umma::ld32x32(tmem + tl + RTM_A, a0);
      umma::ld32x32(tmem + tl + RTM_A + 32, a1);
      umma::wait_ld();
      umma::reg_fence(a0);
      umma::reg_fence(a1);
      umma::ld32x32(tmem + tl + RTM_A + 64, c0);
      umma::ld32x32(tmem + tl + RTM_A + 96, c1);
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
        umma::ld32x32(tmem + tl + RTM_S + 64 * pp, a0);
        umma::ld32x32(tmem + tl + RTM_S + 64 * pp + 32, a1);
        umma::wait_ld();
        umma::reg_fence(a0);
        umma::reg_fence(a1);
        pack_scores(a0, pp, 0, w);
        pack_scores(a1, pp, 1, w);
        umma::st32x32(tmem + tl + RTM_P + 32 * pp, w);
      }
      umma::wait_st();
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pready);
      return true;
    };
    // Output of stage j: O accumulator -> bf16 -> shared tile -> one TMA store.
    const int etid = threadIdx.x - 32 * REPI0;   // 0..127
    const uint32_t sO = sbase + RO_OFF;
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
        umma::ld32x32(tmem + tl + RTM_O + 64 * (j & 1) + 32 * h, r);
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
      for (int k = 0; k < RD / 8; ++k)
        sts128(sO + rswz(t, 16 * k),
               make_uint4(pack_bf16(f(8 * k), f(8 * k + 1)), pack_bf16(f(8 * k + 2), f(8 * k + 3)),
                          pack_bf16(f(8 * k + 4), f(8 * k + 5)),
                          pack_bf16(f(8 * k + 6), f(8 * k + 7))));
      fence_proxy_async_smem();
      bar_sync_named(1, 128);
      if (etid == 0) {
        tma_store_3d(&tmO, sO, 0, j * RR, stream);
        bulk_commit();
      }
      return true;
    };
    // Per stage j: the masked scores of j (the output product of j-1 was drained just before),
    // the Gram blocks of j+1, then, once the output product of j has completed, its drain.
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
    const int srow = colw + 8 * (mi & 1) + rr;  // stmatrix rows of the [64][...] operand tiles
    const int scol = 8 * (mi >> 1);
    auto off = [&](int row, int col) -> uint32_t { return rswz(row, 2 * col); };
    // In a 16-token sub-chunk of the K tile: K rows as the B operand of W^T K^T, K via
    // ldmatrix.trans as the B operand of E^T K; V^T in accumulator order.
    uint32_t o_brow[RKS], o_btrn[RKS];
#pragma unroll
    for (int ks = 0; ks < RKS; ++ks) {
      o_brow[ks] = off(8 * (mi >> 1) + rr, 16 * ks + 8 * (mi & 1));
      o_btrn[ks] = off(8 * (mi & 1) + rr, 16 * ks + 8 * (mi >> 1));
    }
    const uint32_t o_vt = off(8 * (mi >> 1) + rr, colw + 8 * (mi & 1));
    const uint32_t o_g = rblk_row(8 * (mi >> 1) + rr, mi & 1);
    constexpr uint32_t SUB_BYTES = 16 * 128;    // 16 token rows of a [128][64] tile

    // W^T rows colw .. colw+15 as m16n8 fp32 fragments: wc[jt] holds columns 8jt .. 8jt+7.
    float wc[RD / 8][4];
    {
      const float* w0 = p.W0 ? p.W0 + (size_t)stream * RD * RD : nullptr;
#pragma unroll
      for (int jt = 0; jt < RD / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          wc[jt][e] = w0 ? w0[row * RD + colw + g] : 0.f;
          wc[jt][2 + e] = w0 ? w0[row * RD + colw + g + 8] : 0.f;
        }
    }
    // bf16(W^T) of this warp's rows into the [64][64] K-major operand tile
    auto store_wt = [&](uint32_t sW) {
#pragma unroll
      for (int ks = 0; ks < RKS; ++ks)
        stsm_x4(sW + rswz(srow, 2 * (16 * ks + scol)), pack_bf16(wc[2 * ks][0], wc[2 * ks][1]),
                pack_bf16(wc[2 * ks][2], wc[2 * ks][3]),
                pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]),
                pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]));
    };
    store_wt(stage_w(0));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(wready);
    bool ok = true;
    for (int j = 0; j < nst; ++j) {
      const int s = j % RNSTAGE;
      // warp-uniform waits (the stmatrix stores below need every lane): the stage's tiles, its
      // Gram blocks, and the output product of j-1, which read the -E^T tile this stage rewrites
      bool got = mbar_wait_warp(full + 8 * s, (j / RNSTAGE) & 1, p.err, p.wait_ns);
      if (got) got = mbar_wait_warp(gready, j & 1, p.err, p.wait_ns);
      if (got && j >= 1) got = mbar_wait_warp(odone, (j - 1) & 1, p.err, p.wait_ns);
      if (!got) {
        ok = false;
        break;
      }
      const uint32_t sK = sbase + s * RSTAGE_BYTES + RTILE;
      const uint32_t sV = sK + RTILE;
      const uint32_t sEta = sV + RTILE;
      const uint32_t sA = sbase + RA_OFF + RA_BYTES * (j & 1);
      const int rows = min(RR, T - j * RR);
      // bf16(W_s^T) as the A operand of X^T = W_s^T K^T for the whole stage
      uint32_t wa[RKS][4];
#pragma unroll
      for (int ks = 0; ks < RKS; ++ks) {
        wa[ks][0] = pack_bf16(wc[2 * ks][0], wc[2 * ks][1]);
        wa[ks][1] = pack_bf16(wc[2 * ks][2], wc[2 * ks][3]);
        wa[ks][2] = pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]);
        wa[ks][3] = pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]);
      }
      // X_u^T = W_s^T K_u^T (two 8-token tiles, even and odd k-steps in separate accumulators)
      auto x_of = [&](const int u, float (&x)[2][4]) {
        float xa[2][4] = {}, xb[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < RKS; ++ks) {
          uint32_t kb[4];
          ldsm_x4(sK + u * SUB_BYTES + o_brow[ks], kb);
          float (&acc)[2][4] = (ks & 1) ? xb : xa;
          mma16816(acc[0], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], kb[0], kb[1]);
          mma16816(acc[1], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], kb[2], kb[3]);
        }
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) x[n][e] = xa[n][e] + xb[n][e];
      };
      // corrections of the later sub-chunks' residuals by the earlier sub-chunks' E
      float D[RU][2][4];
#pragma unroll
      for (int v = 0; v < RU; ++v)
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) D[v][n][e] = 0.f;
      float X[2][4];
      x_of(0, X);
#pragma unroll
      for (int u = 0; u < RU; ++u) {
        // operands of sub-chunk u: V^T fragments and rates (zero past the stream's end)
        uint32_t vt[4];
        ldsm_x4_t(sV + u * SUB_BYTES + o_vt, vt);
        float ev[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tk = 16 * u + 2 * tq + (i & 1) + 8 * (i >> 1);
          ev[i] = tk < rows ? ldsf(sEta + 4 * tk) : 0.f;
        }
        // the next sub-chunk's X runs beside this one's substitution step
        float Xn[2][4];
        if (u + 1 < RU) x_of(u + 1, Xn);
        float E[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const float ea0 = ev[2 * n], ea1 = ev[2 * n + 1];
          E[n][0] = (X[n][0] + D[u][n][0] - bf16_lo(vt[2 * n])) * ea0;
          E[n][1] = (X[n][1] + D[u][n][1] - bf16_hi(vt[2 * n])) * ea1;
          E[n][2] = (X[n][2] + D[u][n][2] - bf16_lo(vt[2 * n + 1])) * ea0;
          E[n][3] = (X[n][3] + D[u][n][3] - bf16_hi(vt[2 * n + 1])) * ea1;
        }
        // -E_u^T as an A operand
        const uint32_t n0 = pack_bf16(E[0][0], E[0][1]) ^ 0x80008000u;
        const uint32_t n1 = pack_bf16(E[0][2], E[0][3]) ^ 0x80008000u;
        const uint32_t n2 = pack_bf16(E[1][0], E[1][1]) ^ 0x80008000u;
        const uint32_t n3 = pack_bf16(E[1][2], E[1][3]) ^ 0x80008000u;
        // fold E_u into the later chunks' sub-chunks, the nearest first (the chain's product)
#pragma unroll
        for (int v = (u / CM + 1) * CM; v < RU; ++v) {
          uint32_t gb[4];
          ldsm_x4(sA + rblk(u, v) + o_g, gb);
          mma16816(D[v][0], n0, n1, n2, n3, gb[0], gb[1]);
          mma16816(D[v][1], n0, n1, n2, n3, gb[2], gb[3]);
        }
        stsm_x4(sE + (u >> 2) * RE_SUB + rswz(srow, 2 * (16 * (u & 3) + scol)), n0, n1, n2, n3);
        // W^T += (-E_u^T) K_u into the fp32 state (the next stage's W_s)
#pragma unroll
        for (int jp = 0; jp < RKS; ++jp) {
          uint32_t kt[4];
          ldsm_x4_t(sK + u * SUB_BYTES + o_btrn[jp], kt);
          mma16816(wc[2 * jp], n0, n1, n2, n3, kt[0], kt[1]);
          mma16816(wc[2 * jp + 1], n0, n1, n2, n3, kt[2], kt[3]);
        }
        if (u + 1 < RU) {
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) X[n][e] = Xn[n][e];
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(eready);
      if (j + 1 < nst) {
        // bf16(W_(j+1)^T) into the tile that Q W_s of stage j-1 read (one barrier per tile, so
        // its phases cannot run ahead of this wait)
        if (j >= 1 &&
            !mbar_wait_warp(o1done + 8 * ((j + 1) & 1), ((j - 1) >> 1) & 1, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        store_wt(stage_w(j + 1));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(wready);
      }
    }
    if (ok) {
      float* wo = p.Wout + (size_t)stream * RD * RD;
#pragma unroll
      for (int jt = 0; jt < RD / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          wo[row * RD + colw + g] = wc[jt][e];
          wo[row * RD + colw + g + 8] = wc[jt][2 + e];
        }
    }
  }
  umma::fence_before();
  __syncthreads();
  if (warp == RMMA) umma::tmem_dealloc(tmem, RTM_COLS);
}

template <int CM>
int launch_rgram(const StateArgs& a, const LaunchCtx& ctx) {
  const int BH = a.B * a.H;
  CUtensorMap tq, tk, tv, to;
  const uint64_t dims[3] = {(uint64_t)RD, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)RD * 2, (uint64_t)a.T * RD * 2};
  const uint32_t box[3] = {(uint32_t)RD, (uint32_t)RR, 1};
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_tmap_3d(&tq, a.Q, bf, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg) ||
      !make_tmap_3d(&tk, a.K, bf, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg) ||
      !make_tmap_3d(&tv, a.V, bf, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg) ||
      !make_tmap_3d(&to, a.O, bf, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg))
    return kCuda;
  auto kern = dual_rgram_kernel<CM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, RSMEM);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  const int limit = tuning(kTuneWaitLimitNs);
  RgramParams p{a.eta, a.eta_scalar, a.S0, a.S_out, a.T, ctx.err,
                limit > 0 ? (uint64_t)limit : 4000000000ull};
  kern<<<BH, RTHREADS, RSMEM, ctx.stream>>>(tq, tk, tv, to, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual_rgram launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

int launch_dual_rgram(const StateArgs& a, const LaunchCtx& ctx) {
  switch (a.C) {
    case 16: return launch_rgram<1>(a, ctx);
    case 32: return launch_rgram<2>(a, ctx);
    case 64: return launch_rgram<4>(a, ctx);
  }
  *ctx.msg = "dual_rgram: chunk must be 16, 32 or 64";
  return kUnsupported;
}

}  // namespace ttt
