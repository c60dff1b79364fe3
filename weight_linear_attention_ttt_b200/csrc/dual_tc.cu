// TTT-Linear mini-batch dual form, bf16 inputs, d = 64, chunk C = 16, 32 or 64: the serial chain
// on warp MMAs in registers, the outputs on tcgen05 tensor cores with TMEM accumulators.
//
// Computes, per (batch, head) stream and chunk c (source: "RNN의 기억을 작은 모델로 바꾼다면:
// Test-Time Training 읽기", section "gradient를 효율적인 layer로 만드는 작업" for the mini-batch
// update and its dual form; section "읽는 동안 문제를 하나 더 푼다" for reading the updated model):
//     G   = K_c W - V_c,   E = diag(eta_c) G
//     O_c = Q_c W - tril(Q_c K_c^T) E
//     W   = W - K_c^T E
//
// Outputs per stage. A pipeline stage holds R = 128 tokens (128 / C chunks). Inside it the state at
// the start of chunk c is W_c = W_s - sum_{c' < c} K_c'^T E_c' (W_s: the state at the stage's
// start), so
//     O_c = Q_c W_s - sum_{c' < c} (Q_c K_c'^T) E_c' - tril(Q_c K_c^T) E_c,
// and stacked over the stage this is one causal product with the plain token mask (key s <= query
// t covers both the earlier chunks and the inclusive diagonal of the own chunk):
//     O_stage = Q W_s - tril(Q K^T) E_stage          (128 x COLS, K = 64 and K = 128)
// Only E depends on the chain; the 128-row products are what the 5th-generation tensor core is
// built for, and they run asynchronously to the warps that carry the chain.
//
// The mask does not depend on C: only the chain does (a chunk of C = 16 CM tokens takes the CM
// residuals of its 16-token sub-chunks at the chunk-start W, then applies their CM updates).
//
// Roles (NC chain warps, COLS = 16 NC output columns of the stream per CTA):
//   * chain warps 0 .. NC-1: each keeps W^T[16 columns, 64] as fp32 m16n8 accumulators for the
//     whole sequence and runs, per chunk, P^T = W^T K_c^T -> E^T -> W^T -= E^T K_c on mma.sync
//     (the packed accumulators are the next A operand: no register transposes). At each stage
//     start it stores bf16(W^T) (the B operand of Q W_s), after each chunk -E^T (the B operand
//     of the masked product) into shared memory with stmatrix.
//   * warp NC: TMA producer (3-stage ring of Q/K/V tiles [128 tokens][64] and the rates).
//   * warp NC+1: owns TMEM and issues every tcgen05.mma from an elected lane: S = Q K^T when a
//     stage lands, O = Q W_s when the chain has stored W_s, O += P (-E) when it has stored E.
//   * warps NC+2 .. NC+5 (one per TMEM lane quarter): turn S into the masked bf16 P (TMEM to
//     TMEM, the A operand of the last product), then drain O through a shared tile to TMA
//     stores.
// TMEM columns: S (x2) [0, 256), P (x2, bf16 pairs) [256, 384), O (x2) [384, 384 + 2 COLS).
// Precision: W is fp32 throughout; the chain rounds bf16(W) and E once per chunk; the outputs
// use bf16(W_s), bf16 scores and bf16 E with fp32 accumulation (relative error ~2^-9 per operand).
#include <algorithm>
#include <string>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int TD = 64;             // head dim
constexpr int TC = 16;             // sub-chunk (the warp-MMA tile height)
constexpr int TR = 128;            // tokens per stage
constexpr int TCPS = TR / TC;      // sub-chunks per stage
constexpr int TKS = TD / 16;       // 16-wide k-steps over d
constexpr int NSTAGE = 3;
constexpr int TILE = TR * TD * 2;  // one [128][64] bf16 tile, 128-byte swizzle
constexpr int STAGE_BYTES = 3 * TILE + 1024;   // Q, K, V, rates (512 B, padded)
constexpr uint32_t TM_S = 0, TM_P = 256, TM_O = 384;

template <int NC, int WC>
struct TcCfg {
  static constexpr int COLS = WC * NC;            // output columns per CTA
  static constexpr int NG = TD / COLS;            // CTAs per stream
  static constexpr int ORB = COLS * 2;            // bytes per row of the O tile
  static constexpr int ESUB = COLS * 128;         // one [COLS][64 tokens] sub-tile of E
  static constexpr int E_BYTES = 2 * ESUB;        // E^T of a stage: [COLS][128 tokens]
  static constexpr int W_BYTES = COLS * 128;      // bf16 W_s^T: [COLS][64]
  static constexpr int O_BYTES = TR * ORB;        // output tile [128][COLS]
  static constexpr int E_OFF = NSTAGE * STAGE_BYTES;
  static constexpr int W_OFF = E_OFF + 2 * E_BYTES;
  static constexpr int O_OFF = W_OFF + 2 * W_BYTES;
  static constexpr int BAR_OFF = O_OFF + O_BYTES;
  static constexpr int SMEM = 1024 + BAR_OFF + 256;
  static constexpr int THREADS = 32 * (NC + 6);
  static constexpr int PRODUCER = NC, MMA = NC + 1, EPI0 = NC + 2;
  static constexpr uint32_t TM_COLS = 512;
  static_assert(TM_O + 2 * COLS <= TM_COLS, "TMEM columns");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(ESUB % 1024 == 0 && W_BYTES % 1024 == 0 && O_BYTES % 1024 == 0, "alignment");
};

struct TcParams {
  const float* eta;
  float eta_scalar;
  const float* W0;
  float* Wout;
  int T;
  unsigned* err;
  uint64_t wait_ns;   // limit of every pipeline wait; copies in flight get a fixed second
};

// Transpose of an 8x8 bf16 tile held as one register per lane in MMA-fragment order.
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void stsm_x2(uint32_t addr, uint32_t r0, uint32_t r1) {
  asm volatile("stmatrix.sync.aligned.m8n8.x2.shared.b16 [%0], {%1, %2};" ::"r"(addr), "r"(r0),
               "r"(r1)
               : "memory");
}
// Byte offset inside a TMA-swizzled tile with RB-byte rows (RB = 32, 64 or 128).
template <int RB>
__device__ __forceinline__ uint32_t swz_rows(uint32_t row, uint32_t colbyte) {
  return swz<RB>(row * RB + colbyte);
}

// SO (state only): the chain alone, for callers that need the final state and no outputs (the
// segment maps of the sequence-parallel form): no Q loads, no tcgen05 products, no O stores.
// CK (with SO, 16-column chains, C = 16), the dual-form backward's inputs:
//   1: every chunk's starting state leaves as a bf16 d x d checkpoint through tmC: each chain
//      warp stages its 16 columns with stmatrix.trans and TMA-stores them;
//   2: every stage's starting state W_s leaves the same way (one per 128 tokens), and of every
//      token the residual G = K W_c - V through tmO and -E = -diag(eta) G through tmQ, as bf16
//      [T][d] rows (each chain warp collects its 16 columns of the stage in two [128][16] tiles,
//      stored once per stage; tmQ and the ring's Q tiles are unused by the state-only chain).
template <int NC, int CM, int WC, bool SO, int CK = 0>
__global__ void __launch_bounds__(TcCfg<NC, WC>::THREADS, 1)
    dual_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const __grid_constant__ CUtensorMap tmC, const TcParams p) {
  static_assert(!CK || (SO && WC == 16 && CM == 1), "checkpoints: state-only 16-column chains");
  using Cfg = TcCfg<NC, WC>;
  constexpr int COLS = Cfg::COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + Cfg::BAR_OFF;
  const uint32_t full = bar, empty = bar + 8 * NSTAGE;      // stage ring
  const uint32_t sfull = bar + 48;    // S accumulator written (x2, MMA commit)
  const uint32_t pfull = bar + 64;    // P written (x2, 4 epilogue warps)
  const uint32_t wready = bar + 80;   // bf16 W_s stored (x2, NC chain warps)
  const uint32_t eready = bar + 96;   // -E of the stage stored (x2, NC chain warps)
  const uint32_t ofull = bar + 112;   // O accumulator complete (x2, MMA commit)
  const uint32_t ofree = bar + 128;   // O accumulator read out (x2, 4 epilogue warps)
  const uint32_t mdone = bar + 144;   // every MMA issued has completed (MMA commit)
  const uint32_t tslot = bar + 160;

  const int stream = blockIdx.x / Cfg::NG;
  const int col_cta = (blockIdx.x % Cfg::NG) * COLS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int nst = (T + TR - 1) / TR;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, SO ? NC : NC + 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sfull + 8 * b, 1);
      mbar_init(pfull + 8 * b, 4);
      mbar_init(wready + 8 * b, NC);
      mbar_init(eready + 8 * b, NC);
      mbar_init(ofull + 8 * b, 1);
      mbar_init(ofree + 8 * b, 4);
    }
    mbar_init(mdone, 1);
    fence_mbar_init();
  }
  // E buffers start at zero: in a partial last stage the absent chunks' columns of E are read
  // by the masked product (multiplied by zero scores), so they must hold finite values.
  for (int i = threadIdx.x; i < 2 * Cfg::E_BYTES / 16; i += Cfg::THREADS)
    sts128(sbase + Cfg::E_OFF + 16 * i, make_uint4(0u, 0u, 0u, 0u));
  fence_proxy_async_smem();
  if (warp == Cfg::MMA) umma::tmem_alloc(tslot, Cfg::TM_COLS);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Cfg::BAR_OFF + 160);

  if (warp == Cfg::PRODUCER) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int j = 0; j < nst; ++j) {
        const int s = j % NSTAGE;
        if (j >= NSTAGE &&
            !mbar_wait(empty + 8 * s, ((j / NSTAGE) - 1) & 1, p.err, p.wait_ns))
          break;
        const int rows = min(TR, T - j * TR);
        const uint32_t fb = full + 8 * s;
        const uint32_t st = sbase + s * STAGE_BYTES;
        // a scalar rate is written into the stage's rate slot, so the chain warps read the
        // slot unconditionally (the arrival below releases these stores)
        if (!p.eta)
          for (int i = 0; i < TR; ++i) stsf(st + 3 * TILE + 4 * i, p.eta_scalar);
        mbar_arrive_expect_tx(fb, (SO ? 2 : 3) * TILE + (p.eta ? rows * 4 : 0));
        if (!SO) tma_load_3d(st, &tmQ, fb, 0, j * TR, stream);
        tma_load_3d(st + TILE, &tmK, fb, 0, j * TR, stream);
        tma_load_3d(st + 2 * TILE, &tmV, fb, 0, j * TR, stream);
        if (p.eta)
          bulk_load(st + 3 * TILE, p.eta + (size_t)stream * T + (size_t)j * TR, rows * 4, fb);
        issued = j + 1;
      }
      // copies still in flight must land before the CTA may exit (normally all have)
      for (int j = max(0, issued - NSTAGE); j < issued; ++j)
        mbar_wait(full + 8 * (j % NSTAGE), (j / NSTAGE) & 1, p.err, 1000000000ull);
    }
  } else if (SO && warp >= Cfg::MMA) {
    // state only: no products and no outputs
  } else if (warp == Cfg::MMA) {
    // ------------------------------------------------------------------ tcgen05 issue warp
    // The whole warp runs the loop (warp-uniform waits); an elected lane issues.
    const uint32_t id_s = umma::idesc_bf16(128, 128, false, false);   // Q K^T
    const uint32_t id_o = umma::idesc_bf16(128, COLS, false, false);  // Q W_s and P (-E)
    auto issue_s = [&](int j) -> bool {
      const int s = j % NSTAGE, b = j & 1;
      if (!mbar_wait_warp(full + 8 * s, (j / NSTAGE) & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
      const uint32_t sQ = sbase + s * STAGE_BYTES, sK = sQ + TILE;
#pragma unroll
      for (int ks = 0; ks < TKS; ++ks)
        umma::mma_ss_elect(tmem + TM_S + 128 * b, umma::desc_kmajor(sQ + 32 * ks),
                           umma::desc_kmajor(sK + 32 * ks), id_s, ks > 0);
      umma::commit_elect(sfull + 8 * b);
      return true;
    };
    bool ok = nst > 0 ? issue_s(0) : true;
    for (int j = 0; ok && j < nst; ++j) {
      const int s = j % NSTAGE, b = j & 1;
      const uint32_t sQ = sbase + s * STAGE_BYTES;
      const uint32_t dO = tmem + TM_O + COLS * b;
      // O = Q W_s once the chain has stored W_s and the epilogue has read out O(j-2)
      if (!mbar_wait_warp(wready + 8 * b, (j >> 1) & 1, p.err, p.wait_ns)) break;
      if (j >= 2 && !mbar_wait_warp(ofree + 8 * b, ((j >> 1) - 1) & 1, p.err, p.wait_ns)) break;
      umma::fence_after();
      const uint32_t sW = sbase + Cfg::W_OFF + Cfg::W_BYTES * b;
#pragma unroll
      for (int ks = 0; ks < TKS; ++ks)
        umma::mma_ss_elect(dO, umma::desc_kmajor(sQ + 32 * ks), umma::desc_kmajor(sW + 32 * ks),
                           id_o, ks > 0);
      // O += P (-E) once the scores are masked and the chain has stored the stage's -E
      if (!mbar_wait_warp(pfull + 8 * b, (j >> 1) & 1, p.err, p.wait_ns)) break;
      if (!mbar_wait_warp(eready + 8 * b, (j >> 1) & 1, p.err, p.wait_ns)) break;
      umma::fence_after();
      const uint32_t sE = sbase + Cfg::E_OFF + Cfg::E_BYTES * b;
#pragma unroll
      for (int ks = 0; ks < TR / 16; ++ks)
        umma::mma_ts_elect(dO, tmem + TM_P + 64 * b + 8 * ks,
                           umma::desc_kmajor(sE + (ks >> 2) * Cfg::ESUB + 32 * (ks & 3)), id_o,
                           true);
      umma::commit_elect(ofull + 8 * b);
      umma::commit_elect(empty + 8 * s);   // Q and K of the stage are no longer read
      // scores of the next stage (score buffer (j+1)&1 was read by the masking of stage j-1,
      // which completed before the wait on pfull above in the previous iteration)
      if (j + 1 < nst) ok = issue_s(j + 1);
    }
    // every MMA this warp issued completes before TMEM is released
    umma::commit_elect(mdone);
    mbar_wait_warp(mdone, 0, p.err, 1000000000ull);
  } else if (warp >= Cfg::EPI0) {
    // ------------------------------------------------------------------ epilogue warps
    const int q = warp & 3;                       // TMEM lane quarter: rows 32q .. 32q+31
    const int t = 32 * q + lane;                  // token row within the stage
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int etid = threadIdx.x - 32 * Cfg::EPI0;   // 0..127
    const uint32_t sO = sbase + Cfg::O_OFF;
    // Masked scores of stage j: P[t][s] = S[t][s] for s <= t, else 0, as bf16 pairs.
    auto mask = [&](int j) -> bool {
      const int b = j & 1;
      if (!mbar_wait_warp(sfull + 8 * b, (j >> 1) & 1, p.err, p.wait_ns)) return false;
      umma::fence_after();
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {        // key tokens 64 pp .. 64 pp + 63
        uint32_t v[32] = {}, w[32];
        if (2 * pp <= q) {
          umma::ld32x32(tmem + tl + TM_S + 128 * b + 64 * pp, v);
          umma::wait_ld();
          umma::reg_fence(v);
        }
        uint32_t v2[32] = {};
        if (2 * pp + 1 <= q) {
          umma::ld32x32(tmem + tl + TM_S + 128 * b + 64 * pp + 32, v2);
          umma::wait_ld();
          umma::reg_fence(v2);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int s0 = 64 * pp + 2 * i, s1 = s0 + 1;   // key tokens of word i
          const uint32_t x0 = i < 16 ? v[2 * i] : v2[2 * i - 32];
          const uint32_t x1 = i < 16 ? v[2 * i + 1] : v2[2 * i - 31];
          const bool k0 = s0 <= t, k1 = s1 <= t;
          w[i] = pack_bf16(k0 ? __uint_as_float(x0) : 0.f, k1 ? __uint_as_float(x1) : 0.f);
        }
        umma::st32x32(tmem + tl + TM_P + 64 * b + 32 * pp, w);
      }
      umma::wait_st();
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull + 8 * b);
      return true;
    };
    // Output of stage j: O accumulator -> bf16 -> shared tile -> TMA store.
    auto drain = [&](int j) -> bool {
      const int b = j & 1;
      const bool got = mbar_wait_warp(ofull + 8 * b, (j >> 1) & 1, p.err, p.wait_ns);
      // the previous store has finished reading the shared tile before anyone rewrites it
      if (got && etid == 0) bulk_wait_read<0>();
      if (bar_or_named(1, 128, !got)) return false;
      umma::fence_after();
      uint32_t v[COLS];
      if constexpr (COLS >= 32) {
#pragma unroll
        for (int h = 0; h < COLS / 32; ++h) {
          uint32_t r[32];
          umma::ld32x32(tmem + tl + TM_O + COLS * b + 32 * h, r);
          umma::wait_ld();
          umma::reg_fence(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[32 * h + i] = r[i];
        }
      } else {
        uint32_t r[16];
        umma::ld32x16(tmem + tl + TM_O + COLS * b, r);
        umma::wait_ld();
        umma::reg_fence_n(r);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = r[i];
      }
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ofree + 8 * b);
#pragma unroll
      for (int k = 0; k < COLS / 8; ++k)
        sts128(sO + swz_rows<Cfg::ORB>(t, 16 * k),
               make_uint4(pack_bf16(__uint_as_float(v[8 * k]), __uint_as_float(v[8 * k + 1])),
                          pack_bf16(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3])),
                          pack_bf16(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5])),
                          pack_bf16(__uint_as_float(v[8 * k + 6]),
                                    __uint_as_float(v[8 * k + 7]))));
      fence_proxy_async_smem();
      bar_sync_named(1, 128);
      if (etid == 0) {
        tma_store_3d(&tmO, sO, col_cta, j * TR, stream);
        bulk_commit();
      }
      return true;
    };
    for (int j = 0; j < nst; ++j) {
      // P buffer j&1 was last read by the product of stage j-2, drained (ofull) just before
      const bool ok = mask(j);
      if (bar_or_named(1, 128, !ok)) break;
      if (j >= 1 && !drain(j - 1)) break;
      if (j + 1 == nst) drain(j);
    }
    if (etid == 0) bulk_wait<0>();
  } else if constexpr (WC == 8) {
    // ------------------------------------------------------------------ chain warps, 8 columns
    // Each warp keeps W[:, 8 columns] (d x 8) as four m16n8 fp32 accumulators; bf16(W) and E
    // reach the B operand of the next products through movmatrix transposes. Two such warps
    // share each SM sub-partition, so two chains interleave.
    static_assert(CM == 1, "the 8-column chain takes 16-token chunks");
    const int g = lane >> 2, tq = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;
    const int colw = 8 * warp;
    const int colg = col_cta + colw;
    auto off = [&](int row, int col) -> uint32_t { return swz_rows<128>(row, 2 * col); };
    // K rows as the A operand (matrices (r0-7, lo) (r8-15, lo) (r0-7, hi) (r8-15, hi)); K^T as
    // the A operand of the update via ldmatrix.trans; V in accumulator order
    uint32_t o_arow[TKS], o_atrn[TKS];
#pragma unroll
    for (int ks = 0; ks < TKS; ++ks) {
      o_arow[ks] = off(8 * (mi & 1) + rr, 16 * ks + 8 * (mi >> 1));
      o_atrn[ks] = off(8 * (mi >> 1) + rr, 16 * ks + 8 * (mi & 1));
    }
    const uint32_t o_v0 = off(g, colg + 2 * tq), o_v1 = off(g + 8, colg + 2 * tq);
    constexpr uint32_t CHUNK_BYTES = 16 * 128;
    // stmatrix rows: W column colw + rr of the [COLS][...] tiles
    const int srow = colw + rr;
    float wc[TKS][4];   // W[16 mt + g (+8)][colg + 2 tq (+1)]
    {
      const float* w0 = p.W0 ? p.W0 + (size_t)stream * TD * TD : nullptr;
#pragma unroll
      for (int mt = 0; mt < TKS; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float2 v = make_float2(0.f, 0.f);
          if (w0)
            v = *reinterpret_cast<const float2*>(w0 + (16 * mt + 8 * h + g) * TD + colg + 2 * tq);
          wc[mt][2 * h] = v.x;
          wc[mt][2 * h + 1] = v.y;
        }
    }
    struct Ops8 {
      uint32_t ka[TKS][4], kt[TKS][4], v0, v1;
      float eg, eg8;
    };
    bool ok = true;
    for (int j = 0; j < nst; ++j) {
      const int s = j % NSTAGE, b = j & 1;
      bool got = mbar_wait_warp(full + 8 * s, (j / NSTAGE) & 1, p.err, p.wait_ns);
      if (!SO && got && j >= 2)
        got = mbar_wait_warp(ofull + 8 * b, ((j >> 1) - 1) & 1, p.err, p.wait_ns);
      if (!got) {
        ok = false;
        break;
      }
      const uint32_t sK = sbase + s * STAGE_BYTES + TILE;
      const uint32_t sV = sK + TILE;
      const uint32_t sEta = sV + TILE;
      const uint32_t sE = sbase + Cfg::E_OFF + Cfg::E_BYTES * b;
      const uint32_t sW = sbase + Cfg::W_OFF + Cfg::W_BYTES * b;
      const int chunks = min(TR, T - j * TR) / TC;
      // bf16(W_s)^T rows for the stage's Q W_s product: the B fragments of two k-steps per
      // stmatrix (matrix m: k = 32 pp + 8 m)
      if constexpr (!SO) {
#pragma unroll
        for (int pp = 0; pp < TKS / 2; ++pp) {
          const uint32_t w00 = movm_t(pack_bf16(wc[2 * pp][0], wc[2 * pp][1]));
          const uint32_t w01 = movm_t(pack_bf16(wc[2 * pp][2], wc[2 * pp][3]));
          const uint32_t w10 = movm_t(pack_bf16(wc[2 * pp + 1][0], wc[2 * pp + 1][1]));
          const uint32_t w11 = movm_t(pack_bf16(wc[2 * pp + 1][2], wc[2 * pp + 1][3]));
          stsm_x4(sW + swz_rows<128>(srow, 2 * (32 * pp + 8 * mi)), w00, w01, w10, w11);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(wready + 8 * b);
      }

      auto load = [&](Ops8& o, const int c) {
        const uint32_t cb = c * CHUNK_BYTES;
#pragma unroll
        for (int ks = 0; ks < TKS; ++ks) {
          ldsm_x4(sK + cb + o_arow[ks], o.ka[ks]);
          ldsm_x4_t(sK + cb + o_atrn[ks], o.kt[ks]);
        }
        o.v0 = ldsu32(sV + cb + o_v0);
        o.v1 = ldsu32(sV + cb + o_v1);
        o.eg = ldsf(sEta + 4 * (16 * c + g));
        o.eg8 = ldsf(sEta + 4 * (16 * c + g + 8));
      };
      // bf16(W) -> P = K W -> E -> W -= K^T E; -E^T is stored for the outputs
      auto chain = [&](const Ops8& o, const int c) {
        uint32_t wb[TKS][2];
#pragma unroll
        for (int ks = 0; ks < TKS; ++ks) {
          wb[ks][0] = movm_t(pack_bf16(wc[ks][0], wc[ks][1]));
          wb[ks][1] = movm_t(pack_bf16(wc[ks][2], wc[ks][3]));
        }
        float pa[4] = {}, pb[4] = {};
#pragma unroll
        for (int ks = 0; ks < TKS; ++ks) {
          if (ks & 1)
            mma16816(pb, o.ka[ks][0], o.ka[ks][1], o.ka[ks][2], o.ka[ks][3], wb[ks][0], wb[ks][1]);
          else
            mma16816(pa, o.ka[ks][0], o.ka[ks][1], o.ka[ks][2], o.ka[ks][3], wb[ks][0], wb[ks][1]);
        }
        const float e0 = (pa[0] + pb[0] - bf16_lo(o.v0)) * o.eg;
        const float e1 = (pa[1] + pb[1] - bf16_hi(o.v0)) * o.eg;
        const float e2 = (pa[2] + pb[2] - bf16_lo(o.v1)) * o.eg8;
        const float e3 = (pa[3] + pb[3] - bf16_hi(o.v1)) * o.eg8;
        const uint32_t n0 = movm_t(pack_bf16(e0, e1)) ^ 0x80008000u;   // -E, tokens 0-7
        const uint32_t n1 = movm_t(pack_bf16(e2, e3)) ^ 0x80008000u;   // -E, tokens 8-15
#pragma unroll
        for (int mt = 0; mt < TKS; ++mt)
          mma16816(wc[mt], o.kt[mt][0], o.kt[mt][1], o.kt[mt][2], o.kt[mt][3], n0, n1);
        // -E^T of chunk c (lanes 0-7 address matrix 0, tokens 16c..; lanes 8-15 matrix 1)
        if constexpr (!SO)
          stsm_x2(sE + (c >> 2) * Cfg::ESUB +
                      swz_rows<128>(srow, 2 * (16 * (c & 3) + 8 * (mi & 1))),
                  n0, n1);
      };
      if (chunks == TCPS) {
        Ops8 ops[2];
        load(ops[0], 0);
#pragma unroll
        for (int c = 0; c < TCPS; ++c) {
          if (c + 1 < TCPS) load(ops[(c + 1) & 1], c + 1);
          chain(ops[c & 1], c);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < chunks; ++c) {
          Ops8 o;
          load(o, c);
          chain(o, c);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (!SO) mbar_arrive(eready + 8 * b);
        mbar_arrive(empty + 8 * s);
      }
    }
    if (ok && p.Wout) {
      float* wo = p.Wout + (size_t)stream * TD * TD;
#pragma unroll
      for (int mt = 0; mt < TKS; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          *reinterpret_cast<float2*>(wo + (16 * mt + 8 * h + g) * TD + colg + 2 * tq) =
              make_float2(wc[mt][2 * h], wc[mt][2 * h + 1]);
    }
  } else {
    // ------------------------------------------------------------------ chain warps, 16 columns
    const int g = lane >> 2, tq = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;    // ldmatrix / stmatrix: matrix, row
    const int colw = 16 * warp;                 // first column of this warp inside the CTA's
    const int colg = col_cta + colw;            // ... and in the stream's W
    auto off = [&](int row, int col) -> uint32_t { return swz_rows<128>(row, 2 * col); };
    // K rows as the B operand of W^T K^T, K via ldmatrix.trans as the B operand of the update,
    // V^T in accumulator order.
    uint32_t o_brow[TKS], o_btrn[TKS];
#pragma unroll
    for (int ks = 0; ks < TKS; ++ks) {
      o_brow[ks] = off(8 * (mi >> 1) + rr, 16 * ks + 8 * (mi & 1));
      o_btrn[ks] = off(8 * (mi & 1) + rr, 16 * ks + 8 * (mi >> 1));
    }
    const uint32_t o_vt = off(8 * (mi >> 1) + rr, colg + 8 * (mi & 1));
    // stmatrix targets: row 16 warp + 8 (mi & 1) + rr of the [COLS][64] tiles of W_s^T and of
    // -E^T, k offset 8 (mi >> 1) within a 16-wide step
    const int srow = colw + 8 * (mi & 1) + rr;
    const int scol = 8 * (mi >> 1);
    constexpr uint32_t CHUNK_BYTES = 16 * 128;   // 16 token rows of a [128][64] tile

    // The state as m16n8 fp32 accumulators: W^T[colg .. colg+15, :]; tile jt holds columns
    // 8jt .. 8jt+7 of W^T (rows of W).
    float wc[TD / 8][4];
    {
      const float* w0 = p.W0 ? p.W0 + (size_t)stream * TD * TD : nullptr;
#pragma unroll
      for (int jt = 0; jt < TD / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          wc[jt][e] = w0 ? w0[row * TD + colg + g] : 0.f;
          wc[jt][2 + e] = w0 ? w0[row * TD + colg + g + 8] : 0.f;
        }
    }
    struct Ops {
      uint32_t kb[TKS][4], kt[TKS][4], vt[4];
      float e0, e1, e8, e9;
    };
    bool ok = true;
    for (int j = 0; j < nst; ++j) {
      const int s = j % NSTAGE, b = j & 1;
      // warp-uniform waits: the stmatrix stores below need every lane
      bool got = mbar_wait_warp(full + 8 * s, (j / NSTAGE) & 1, p.err, p.wait_ns);
      // E and W_s buffers b were last read by the products of stage j-2
      if (!SO && got && j >= 2)
        got = mbar_wait_warp(ofull + 8 * b, ((j >> 1) - 1) & 1, p.err, p.wait_ns);
      if (!got) {
        ok = false;
        break;
      }
      const uint32_t sK = sbase + s * STAGE_BYTES + TILE;
      const uint32_t sV = sK + TILE;
      const uint32_t sEta = sV + TILE;
      const uint32_t sE = sbase + Cfg::E_OFF + Cfg::E_BYTES * b;
      const uint32_t sW = sbase + Cfg::W_OFF + Cfg::W_BYTES * b;
      const int chunks = min(TR, T - j * TR) / TC;

      if constexpr (CK == 2) {
        // W_s as W rows (stmatrix.trans of the bf16 W^T fragments), one TMA store per stage
        const uint32_t wtile = sbase + Cfg::W_OFF + warp * 2048;
        if (lane == 0) bulk_wait_read<1>();   // the previous stage's W_s store has read it
        __syncwarp();
#pragma unroll
        for (int ks = 0; ks < TKS; ++ks)
          stsm_x4_t(wtile + (16 * ks + (lane & 7) + 8 * (lane >> 4)) * 32 + ((lane >> 3) & 1) * 16,
                    pack_bf16(wc[2 * ks][0], wc[2 * ks][1]), pack_bf16(wc[2 * ks][2], wc[2 * ks][3]),
                    pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]),
                    pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmC, wtile, colg, 0, stream * nst + j);
          bulk_commit();
          // pending: G, -E of stage j-2 (their tiles are rewritten below), W_s of j-1, G, -E of
          // j-1, W_s of j
          bulk_wait_read<3>();
        }
        __syncwarp();
      }
      // bf16(W_s^T) for the stage's Q W_s product
      if constexpr (!SO) {
#pragma unroll
        for (int ks = 0; ks < TKS; ++ks)
          stsm_x4(sW + swz_rows<128>(srow, 2 * (16 * ks + scol)),
                  pack_bf16(wc[2 * ks][0], wc[2 * ks][1]), pack_bf16(wc[2 * ks][2], wc[2 * ks][3]),
                  pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]),
                  pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(wready + 8 * b);
      }

      auto load = [&](Ops& o, const int c) {
        const uint32_t cb = c * CHUNK_BYTES;
#pragma unroll
        for (int ks = 0; ks < TKS; ++ks) {
          ldsm_x4(sK + cb + o_brow[ks], o.kb[ks]);
          ldsm_x4_t(sK + cb + o_btrn[ks], o.kt[ks]);
        }
        ldsm_x4_t(sV + cb + o_vt, o.vt);
        o.e0 = ldsf(sEta + 4 * (16 * c + 2 * tq));
        o.e1 = ldsf(sEta + 4 * (16 * c + 2 * tq + 1));
        o.e8 = ldsf(sEta + 4 * (16 * c + 8 + 2 * tq));
        o.e9 = ldsf(sEta + 4 * (16 * c + 9 + 2 * tq));
      };
      // bf16(W^T) -> P^T = W^T K^T -> E^T -> W^T -= E^T K; -E^T is stored for the outputs
      auto chain = [&](const Ops& o, const int c) {
        uint32_t wa[TKS][4];
#pragma unroll
        for (int ks = 0; ks < TKS; ++ks) {
          wa[ks][0] = pack_bf16(wc[2 * ks][0], wc[2 * ks][1]);
          wa[ks][1] = pack_bf16(wc[2 * ks][2], wc[2 * ks][3]);
          wa[ks][2] = pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]);
          wa[ks][3] = pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]);
        }
        if constexpr (CK == 1) {
          // checkpoint W_c: wa holds this warp's 16 columns of bf16(W) as W^T fragments;
          // stmatrix.trans writes them as W rows into a [64 rows][16 columns] tile (32-byte rows,
          // double-buffered by chunk parity), which one TMA store sends to the checkpoint
          const int gc = j * TCPS + c;
          const uint32_t ctile = sbase + Cfg::E_OFF + warp * 4096 + (gc & 1) * 2048;
          if (lane == 0) bulk_wait_read<1>();   // the store of chunk gc-2 has read this tile
          __syncwarp();
#pragma unroll
          for (int ks = 0; ks < TKS; ++ks)
            stsm_x4_t(ctile + (16 * ks + (lane & 7) + 8 * (lane >> 4)) * 32 + ((lane >> 3) & 1) * 16,
                      wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmC, ctile, colg, 0, stream * (T / TC) + gc);
            bulk_commit();
          }
        }
        float pa[2][4] = {}, pb[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < TKS; ++ks) {
          float (&acc)[2][4] = (ks & 1) ? pb : pa;
          mma16816(acc[0], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], o.kb[ks][0], o.kb[ks][1]);
          mma16816(acc[1], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], o.kb[ks][2], o.kb[ks][3]);
        }
        float E[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          E[n][0] = pa[n][0] + pb[n][0] - bf16_lo(o.vt[2 * n]);   // G^T
          E[n][1] = pa[n][1] + pb[n][1] - bf16_hi(o.vt[2 * n]);
          E[n][2] = pa[n][2] + pb[n][2] - bf16_lo(o.vt[2 * n + 1]);
          E[n][3] = pa[n][3] + pb[n][3] - bf16_hi(o.vt[2 * n + 1]);
        }
        if constexpr (CK == 2) {
          // G rows of chunk c: the G^T fragments, transposed by stmatrix.trans, into rows
          // 16c .. 16c+15 of this warp's [128 tokens][16 columns] tile of the stage
          stsm_x4_t(sbase + Cfg::E_OFF + warp * 8192 + (j & 1) * 4096 +
                        (16 * c + (lane & 7) + 8 * (lane >> 4)) * 32 + ((lane >> 3) & 1) * 16,
                    pack_bf16(E[0][0], E[0][1]), pack_bf16(E[0][2], E[0][3]),
                    pack_bf16(E[1][0], E[1][1]), pack_bf16(E[1][2], E[1][3]));
        }
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const float ea0 = n ? o.e8 : o.e0, ea1 = n ? o.e9 : o.e1;
          E[n][0] *= ea0;
          E[n][1] *= ea1;
          E[n][2] *= ea0;
          E[n][3] *= ea1;
        }
        const uint32_t n0 = pack_bf16(E[0][0], E[0][1]) ^ 0x80008000u;
        const uint32_t n1 = pack_bf16(E[0][2], E[0][3]) ^ 0x80008000u;
        const uint32_t n2 = pack_bf16(E[1][0], E[1][1]) ^ 0x80008000u;
        const uint32_t n3 = pack_bf16(E[1][2], E[1][3]) ^ 0x80008000u;
        if constexpr (CK == 2) {   // -E rows of chunk c, into the stage's second tile
          stsm_x4_t(sbase + (j & 1) * STAGE_BYTES + warp * 4096 +
                        (16 * c + (lane & 7) + 8 * (lane >> 4)) * 32 + ((lane >> 3) & 1) * 16,
                    n0, n1, n2, n3);
        }
#pragma unroll
        for (int jp = 0; jp < TKS; ++jp) {
          mma16816(wc[2 * jp], n0, n1, n2, n3, o.kt[jp][0], o.kt[jp][1]);
          mma16816(wc[2 * jp + 1], n0, n1, n2, n3, o.kt[jp][2], o.kt[jp][3]);
        }
        // -E^T of chunk c: tokens 16c .. 16c+15 of the stage's [COLS][128] buffer
        if constexpr (!SO)
          stsm_x4(sE + (c >> 2) * Cfg::ESUB + swz_rows<128>(srow, 2 * (16 * (c & 3) + scol)),
                  n0, n1, n2, n3);
      };
      if constexpr (CM == 1) {
        if (chunks == TCPS) {
          Ops ops[2];
          load(ops[0], 0);
#pragma unroll
          for (int c = 0; c < TCPS; ++c) {
            if (c + 1 < TCPS) load(ops[(c + 1) & 1], c + 1);
            chain(ops[c & 1], c);
          }
        } else {
#pragma unroll 1
          for (int c = 0; c < chunks; ++c) {
            Ops o;
            load(o, c);
            chain(o, c);
          }
        }
      } else {
        // C = 16 CM: every sub-chunk's residual is taken at the chunk-start W (one gradient
        // step per chunk), then the CM updates are applied.
        auto chain_chunk = [&](const int cc) {
          uint32_t wa[TKS][4];
#pragma unroll
          for (int ks = 0; ks < TKS; ++ks) {
            wa[ks][0] = pack_bf16(wc[2 * ks][0], wc[2 * ks][1]);
            wa[ks][1] = pack_bf16(wc[2 * ks][2], wc[2 * ks][3]);
            wa[ks][2] = pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]);
            wa[ks][3] = pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]);
          }
          uint32_t ne[CM][4];
#pragma unroll
          for (int m = 0; m < CM; ++m) {
            const int c = CM * cc + m;   // 16-token sub-chunk within the stage
            const uint32_t cb = c * CHUNK_BYTES;
            uint32_t kb[TKS][4], vt[4];
#pragma unroll
            for (int ks = 0; ks < TKS; ++ks) ldsm_x4(sK + cb + o_brow[ks], kb[ks]);
            ldsm_x4_t(sV + cb + o_vt, vt);
            const float e0 = ldsf(sEta + 4 * (16 * c + 2 * tq));
            const float e1 = ldsf(sEta + 4 * (16 * c + 2 * tq + 1));
            const float e8 = ldsf(sEta + 4 * (16 * c + 8 + 2 * tq));
            const float e9 = ldsf(sEta + 4 * (16 * c + 9 + 2 * tq));
            float pa[2][4] = {}, pb[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < TKS; ++ks) {
              float (&acc)[2][4] = (ks & 1) ? pb : pa;
              mma16816(acc[0], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], kb[ks][0], kb[ks][1]);
              mma16816(acc[1], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], kb[ks][2], kb[ks][3]);
            }
            float E[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n) {
              const float ea0 = n ? e8 : e0, ea1 = n ? e9 : e1;
              E[n][0] = (pa[n][0] + pb[n][0] - bf16_lo(vt[2 * n])) * ea0;
              E[n][1] = (pa[n][1] + pb[n][1] - bf16_hi(vt[2 * n])) * ea1;
              E[n][2] = (pa[n][2] + pb[n][2] - bf16_lo(vt[2 * n + 1])) * ea0;
              E[n][3] = (pa[n][3] + pb[n][3] - bf16_hi(vt[2 * n + 1])) * ea1;
            }
            ne[m][0] = pack_bf16(E[0][0], E[0][1]) ^ 0x80008000u;
            ne[m][1] = pack_bf16(E[0][2], E[0][3]) ^ 0x80008000u;
            ne[m][2] = pack_bf16(E[1][0], E[1][1]) ^ 0x80008000u;
            ne[m][3] = pack_bf16(E[1][2], E[1][3]) ^ 0x80008000u;
            if constexpr (!SO)
              stsm_x4(sE + (c >> 2) * Cfg::ESUB +
                          swz_rows<128>(srow, 2 * (16 * (c & 3) + scol)),
                      ne[m][0], ne[m][1], ne[m][2], ne[m][3]);
          }
#pragma unroll
          for (int m = 0; m < CM; ++m) {
            const uint32_t cb = (CM * cc + m) * CHUNK_BYTES;
            uint32_t kt[TKS][4];
#pragma unroll
            for (int ks = 0; ks < TKS; ++ks) ldsm_x4_t(sK + cb + o_btrn[ks], kt[ks]);
#pragma unroll
            for (int jp = 0; jp < TKS; ++jp) {
              mma16816(wc[2 * jp], ne[m][0], ne[m][1], ne[m][2], ne[m][3], kt[jp][0], kt[jp][1]);
              mma16816(wc[2 * jp + 1], ne[m][0], ne[m][1], ne[m][2], ne[m][3], kt[jp][2],
                       kt[jp][3]);
            }
          }
        };
        if (chunks == TCPS) {
#pragma unroll
          for (int cc = 0; cc < TCPS / CM; ++cc) chain_chunk(cc);
        } else {
#pragma unroll 1
          for (int cc = 0; cc < chunks / CM; ++cc) chain_chunk(cc);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (!SO) mbar_arrive(eready + 8 * b);
        mbar_arrive(empty + 8 * s);   // K, V and the rates of the stage are consumed
        if constexpr (CK == 2) {      // the stage's G and -E rows of this warp's 16 columns
          tma_store_3d(&tmO, sbase + Cfg::E_OFF + warp * 8192 + (j & 1) * 4096, colg, j * TR,
                       stream);
          tma_store_3d(&tmQ, sbase + (j & 1) * STAGE_BYTES + warp * 4096, colg, j * TR, stream);
          bulk_commit();
        }
      }
    }
    if (ok && p.Wout) {
      float* wo = p.Wout + (size_t)stream * TD * TD;
#pragma unroll
      for (int jt = 0; jt < TD / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          wo[row * TD + colg + g] = wc[jt][e];
          wo[row * TD + colg + g + 8] = wc[jt][2 + e];
        }
    }
    if constexpr (CK) {
      if (lane == 0) bulk_wait<0>();   // the checkpoint stores have completed
    }
  }
  umma::fence_before();
  __syncthreads();
  if (warp == Cfg::MMA) umma::tmem_dealloc(tmem, Cfg::TM_COLS);
}

template <int NC, int CM, int WC, bool SO, int CK = 0>
int launch_tc(const StateArgs& a, const LaunchCtx& ctx, uint16_t* ckpt = nullptr,
              uint16_t* gbuf = nullptr, uint16_t* nebuf = nullptr) {
  using Cfg = TcCfg<NC, WC>;
  const int BH = a.B * a.H;
  CUtensorMap tq, tk, tv, to;
  const uint64_t dims[3] = {(uint64_t)TD, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)TD * 2, (uint64_t)a.T * TD * 2};
  const uint32_t box_in[3] = {(uint32_t)TD, (uint32_t)TR, 1};
  const uint32_t box_out[3] = {(uint32_t)Cfg::COLS, (uint32_t)TR, 1};
  const auto osw = Cfg::ORB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                   : (Cfg::ORB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                     : CU_TENSOR_MAP_SWIZZLE_32B);
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_tmap_3d(&tq, a.Q, bf, dims, strides, box_in, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg) ||
      !make_tmap_3d(&tk, a.K, bf, dims, strides, box_in, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg) ||
      !make_tmap_3d(&tv, a.V, bf, dims, strides, box_in, CU_TENSOR_MAP_SWIZZLE_128B, ctx.msg) ||
      !make_tmap_3d(&to, SO ? a.K : a.O, bf, dims, strides, box_out, osw, ctx.msg))
    return kCuda;
  if (CK == 2) {   // the rows of G and -E, 16-column boxes of a stage (tmO, tmQ unused)
    const uint32_t gbox[3] = {16, (uint32_t)TR, 1};
    if (!make_tmap_3d(&to, gbuf, bf, dims, strides, gbox, CU_TENSOR_MAP_SWIZZLE_NONE, ctx.msg) ||
        !make_tmap_3d(&tq, nebuf, bf, dims, strides, gbox, CU_TENSOR_MAP_SWIZZLE_NONE, ctx.msg))
      return kCuda;
  }
  CUtensorMap tc = tk;   // checkpoint map (CK only)
  if (CK) {
    const int n = CK == 1 ? a.T / TC : (a.T + TR - 1) / TR;
    const uint64_t cdims[3] = {(uint64_t)TD, (uint64_t)TD, (uint64_t)BH * n};
    const uint64_t cstrides[2] = {(uint64_t)TD * 2, (uint64_t)TD * TD * 2};
    const uint32_t cbox[3] = {16, (uint32_t)TD, 1};
    if (!make_tmap_3d(&tc, ckpt, bf, cdims, cstrides, cbox, CU_TENSOR_MAP_SWIZZLE_NONE, ctx.msg))
      return kCuda;
  }
  auto kern = dual_tc_kernel<NC, CM, WC, SO, CK>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  const int limit = tuning(kTuneWaitLimitNs);
  TcParams p{a.eta, a.eta_scalar, a.S0, a.S_out, a.T, ctx.err,
             limit > 0 ? (uint64_t)limit : 4000000000ull};
  kern<<<BH * Cfg::NG, Cfg::THREADS, Cfg::SMEM, ctx.stream>>>(tq, tk, tv, to, tc, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual_tc launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

template <int CM, int WC>
int launch_split(const StateArgs& a, int split, const LaunchCtx& ctx) {
  constexpr int N1 = 64 / WC;   // chain warps with one CTA per stream
  switch (split) {
    case 1: return a.O ? launch_tc<N1, CM, WC, false>(a, ctx) : launch_tc<N1, CM, WC, true>(a, ctx);
    case 2:
      return a.O ? launch_tc<N1 / 2, CM, WC, false>(a, ctx)
                 : launch_tc<N1 / 2, CM, WC, true>(a, ctx);
    case 4:
      return a.O ? launch_tc<N1 / 4, CM, WC, false>(a, ctx)
                 : launch_tc<N1 / 4, CM, WC, true>(a, ctx);
  }
  *ctx.msg = "dual_tc: column split must be 1, 2 or 4";
  return kUnsupported;
}

}  // namespace

// CTAs per stream: 1, 2 or 4 (64, 32 or 16 output columns each). A CTA holds one stream's
// column slice for the whole sequence and one CTA fits per SM; a stream is split over more SMs
// (fewer chain warps per SM, shorter per-chunk issue) only while every CTA still fits in one wave.
int dual_tc_split(int streams, int sms) {
  if (4 * streams <= sms) return 4;
  if (2 * streams <= sms) return 2;
  return 1;
}

bool dual_tc_supported(int d, int C, int dt) {
  return dt == 1 && d == TD && (C == 16 || C == 32 || C == 64);
}

int launch_dual_tc_checkpoints(const StateArgs& a, uint16_t* ckpt, const LaunchCtx& ctx) {
  if (!(dual_tc_supported(a.d, a.C, a.dt) && a.C == TC)) {
    *ctx.msg = "dual_tc checkpoints: bf16, d = 64, C = 16 only";
    return kUnsupported;
  }
  StateArgs s = a;
  s.O = nullptr;
  return launch_tc<4, 1, 16, true, 1>(s, ctx, ckpt);
}

int launch_dual_tc_stage_checkpoints(const StateArgs& a, uint16_t* Ws, uint16_t* G,
                                     uint16_t* NE, const LaunchCtx& ctx) {
  if (!(dual_tc_supported(a.d, a.C, a.dt) && a.C == TC)) {
    *ctx.msg = "dual_tc stage checkpoints: bf16, d = 64, C = 16 only";
    return kUnsupported;
  }
  StateArgs s = a;
  s.O = nullptr;
  return launch_tc<4, 1, 16, true, 2>(s, ctx, Ws, G, NE);
}

int launch_dual_tc(const StateArgs& a, int split, const LaunchCtx& ctx) {
  // Columns per chain warp for 16-token chunks: 16 with one CTA per stream (4 chain warps, one
  // per SM sub-partition; 42.6 against 52.7 us with 8 columns on the 125M-layer shape), 8 when
  // a stream is split over CTAs (444 against 477 us on the 1.3B-layer shape, 3.20 against
  // 3.56 ms on 4 streams of 262144 tokens). The tuning choice overrides.
  const int wcols = tuning(kTuneDualWarpCols);
  const bool eight = wcols ? wcols == 8 : split >= 2;
  switch (a.C) {
    case 16:
      return eight ? launch_split<1, 8>(a, split, ctx) : launch_split<1, 16>(a, split, ctx);
    case 32: return launch_split<2, 16>(a, split, ctx);
    case 64: return launch_split<4, 16>(a, split, ctx);
  }
  *ctx.msg = "dual_tc: chunk must be 16, 32 or 64";
  return kUnsupported;
}

}  // namespace ttt
