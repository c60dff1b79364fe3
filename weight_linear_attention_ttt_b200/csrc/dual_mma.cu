// TTT-Linear mini-batch dual form, bf16 inputs, chunk C = 16: tensor-core path.
//
// Computes, per (batch, head) stream and chunk c (source: "Learning to (Learn at Test Time)"
// reading, section on mini-batch TTT and the dual form; per-token rule section for reading the
// updated model):
//     G   = K_c W - V_c
//     O_c = Q_c W - tril(Q_c K_c^T) diag(eta_c) G
//     W   = W - K_c^T diag(eta_c) G
//
// Design. The chunk loop is a serial chain through W, and a 16-token chunk is too little work to
// hide latency, so the kernel is organised around that chain. It serves d = 32 and d = 128, and
// d = 64 when a caller selects it with ttt_set_tuning("dual_kernel", 1) (the default for d = 64
// is the stage-form kernel of dual_tc.cu, which moves the output products to tcgen05).
//   * The state never leaves registers. Columns of W are independent (the update mixes rows
//     only), so each compute warp owns WC output columns and keeps them as m16n8 fp32 MMA
//     accumulators for the whole sequence. Two forms:
//       - WC = 8 (d = 32 and d = 128): W[:, cols] (d x 8); per chunk
//             P    = K_c W[:, cols]            A = K_c (ldmatrix), B = bf16(W) (movmatrix.trans
//                                              of the accumulators: no shared-memory round trip)
//             E    = diag(eta) (P - V_c[:, cols])
//             W[:, cols] -= K_c^T E           A = K_c^T (ldmatrix.trans), B = E (movmatrix.trans)
//             O_c[:, cols] = Q_c W[:, cols] - mask(Q_c K_c^T) E
//         with the causal scores formed once per stage (one 16x8 piece per warp) and shared
//         through shared memory in MMA-fragment order.
//       - WC = 16 (d = 64): W^T[16 cols, :]; the packed accumulators are directly the A operand
//         of the next chunk's W^T K_c^T, so the chain needs no register transposes, and each
//         warp forms the causal scores itself from the Q and K fragments it holds.
//     Only P -> E -> update sits on the chain; the output products hang off it.
//   * Q/K/V tiles arrive by TMA (3-D tensor maps over [B*H, T, d], 128-byte swizzle) into a
//     multi-stage mbarrier ring filled by one producer warp; outputs leave through a
//     double-buffered shared tile and TMA stores (rows past T are clipped by the tensor map).
// Precision: W is fp32 throughout; its operand copy, E and the scores are rounded to bf16 once
// per chunk for the tensor cores (relative error ~2^-9 per operand, fp32 accumulation).
#include <algorithm>
#include <string>

#include "internal.h"
#include "ptx.cuh"

namespace ttt {
namespace {

template <int D, int NW, int CPS_ = 4, int WC_ = 8>
struct DualCfg {
  static constexpr int WC = WC_;                   // output columns per compute warp (8 or 16)
  static constexpr int C = 16;
  static constexpr int CPS = CPS_;                 // chunks per pipeline stage
  static constexpr int R = C * CPS;                // token rows per stage
  static constexpr int SUB = D >= 64 ? 64 : D;     // columns per swizzled sub-tile
  static constexpr int RB = SUB * 2;               // bytes per sub-tile row
  static constexpr int NSUB = D / SUB;
  static constexpr int SUB_BYTES = R * RB;
  static constexpr int TILE_BYTES = NSUB * SUB_BYTES;
  static constexpr int COLS = WC * NW;             // output columns per CTA
  static constexpr int NG = D / COLS;              // CTAs per stream
  static constexpr int OSUB = COLS >= 64 ? 64 : COLS;
  static constexpr int ORB = OSUB * 2;
  static constexpr int NOSUB = COLS / OSUB;
  static constexpr int OSUB_BYTES = R * ORB;
  static constexpr int OTILE_BYTES = NOSUB * OSUB_BYTES;
  static constexpr int ETA_BYTES = R * 4 <= 1024 ? 1024 : 2048;  // R floats, padded
  static constexpr int STAGE_BYTES = 3 * TILE_BYTES + ETA_BYTES;
  static constexpr int L_BYTES = CPS * 32 * 16;    // shared scores: [chunk][lane][4 x bf16x2]
  static constexpr int BUDGET = 200 * 1024;
  static constexpr int NSTAGE_FIT = (BUDGET - 2 * OTILE_BYTES - L_BYTES) / STAGE_BYTES;
  static constexpr int NSTAGE = NSTAGE_FIT > 8 ? 8 : NSTAGE_FIT;
  static constexpr int OUT_OFF = NSTAGE * STAGE_BYTES;
  static constexpr int L_OFF = OUT_OFF + 2 * OTILE_BYTES;
  static constexpr int BAR_OFF = L_OFF + L_BYTES;
  static constexpr int SMEM = 1024 + BAR_OFF + 16 * NSTAGE;
  static constexpr int THREADS = 32 * (NW + 1);
  static constexpr int KS = D / 16;                // 16-wide k-steps (and m-tiles) over d
  static_assert(NSTAGE >= 2, "pipeline depth");
  static_assert(R * 4 <= ETA_BYTES, "eta slot");
  static_assert(D % COLS == 0, "column split");
  static_assert(COLS >= 16, "TMA store box of at least 32 bytes");
};

struct DualParams {
  const float* eta;
  float eta_scalar;
  const float* W0;
  float* Wout;
  int T;
  unsigned* err;
};

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Named barrier that also ORs a predicate over the participating threads, so that a failed
// (timed-out) wait in any compute warp makes every compute warp leave the loop together.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}
// Transpose of an 8x8 bf16 tile held as one register per lane in MMA-fragment order.
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float ld_shared_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void ld_shared_v4(uint32_t a, uint32_t (&v)[4]) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(a));
}
__device__ __forceinline__ void st_shared_v2(uint32_t a, uint32_t x, uint32_t y) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void stsm_x2(uint32_t addr, uint32_t r0, uint32_t r1) {
  asm volatile("stmatrix.sync.aligned.m8n8.x2.shared.b16 [%0], {%1, %2};" ::"r"(addr), "r"(r0),
               "r"(r1)
               : "memory");
}

template <int D, int NW, int CPS, int WC>
__global__ void __launch_bounds__(DualCfg<D, NW, CPS, WC>::THREADS, 1)
    dual_mma_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmO, const DualParams p) {
  using Cfg = DualCfg<D, NW, CPS, WC>;
  constexpr int R = Cfg::R, KS = Cfg::KS, NSTAGE = Cfg::NSTAGE, RB = Cfg::RB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t full_bar = sbase + Cfg::BAR_OFF;
  const uint32_t empty_bar = full_bar + 8 * NSTAGE;

  const int stream = blockIdx.x / Cfg::NG;
  const int col_cta = (blockIdx.x % Cfg::NG) * Cfg::COLS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int nstg = (T + R - 1) / R;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(full_bar + 8 * s, 1);
      mbar_init(empty_bar + 8 * s, NW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ---------------------------------------------------------------- producer (one lane)
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int j = 0; j < nstg; ++j) {
        const int s = j % NSTAGE;
        if (j >= NSTAGE && !mbar_wait(empty_bar + 8 * s, ((j / NSTAGE) - 1) & 1, p.err)) break;
        const int rows = min(R, T - j * R);
        const uint32_t bytes = 3 * Cfg::TILE_BYTES + (p.eta ? rows * 4 : 0);
        const uint32_t fb = full_bar + 8 * s;
        const uint32_t st = sbase + s * Cfg::STAGE_BYTES;
        // a scalar rate is written into the stage's rate slot, so the compute warps read the
        // slot unconditionally (the arrival below releases these stores)
        if (!p.eta)
          for (int i = 0; i < R; ++i) stsf(st + 3 * Cfg::TILE_BYTES + 4 * i, p.eta_scalar);
        mbar_arrive_expect_tx(fb, bytes);
#pragma unroll
        for (int sub = 0; sub < Cfg::NSUB; ++sub) {
          tma_load_3d(st + sub * Cfg::SUB_BYTES, &tmQ, fb, sub * Cfg::SUB, j * R, stream);
          tma_load_3d(st + Cfg::TILE_BYTES + sub * Cfg::SUB_BYTES, &tmK, fb, sub * Cfg::SUB,
                      j * R, stream);
          tma_load_3d(st + 2 * Cfg::TILE_BYTES + sub * Cfg::SUB_BYTES, &tmV, fb, sub * Cfg::SUB,
                      j * R, stream);
        }
        if (p.eta)
          bulk_load(st + 3 * Cfg::TILE_BYTES, p.eta + (size_t)stream * T + (size_t)j * R,
                    rows * 4, fb);
        issued = j + 1;
      }
      // Copies still in flight must land before the CTA may exit (normally all have).
      for (int j = max(0, issued - NSTAGE); j < issued; ++j)
        mbar_wait(full_bar + 8 * (j % NSTAGE), (j / NSTAGE) & 1, p.err, 1000000000ull);
    }
    return;
  }

  // ------------------------------------------------------------------ compute warps
  const int g = lane >> 2, tq = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;   // ldmatrix: which 8x8 matrix / which row
  const int colw = WC * warp;                // first column of this warp inside the CTA's
  const int colg = col_cta + colw;           // ... and in the stream's W

  // Lane-constant parts of the swizzled shared-memory addresses. A chunk starts at row 16c,
  // a multiple of 8, so the XOR pattern of every access is the same for all chunks and the
  // address of chunk c is this offset plus 16c rows.
  auto off = [&](int row, int col) -> uint32_t {
    return (col / Cfg::SUB) * Cfg::SUB_BYTES + swz<RB>(row * RB + (col % Cfg::SUB) * 2);
  };
  uint32_t o_arow[KS], o_atrn[KS];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    // rows of K/Q as the A operand (M = tokens, K = d): matrices (r0-7,lo) (r8-15,lo)
    // (r0-7,hi) (r8-15,hi) give the four A registers in order.
    o_arow[ks] = off(8 * (mi & 1) + rr, 16 * ks + 8 * (mi >> 1));
    // K^T as the A operand (M = d, K = tokens) via ldmatrix.trans: matrices
    // (t0-7, d lo) (t0-7, d hi) (t8-15, d lo) (t8-15, d hi).
    o_atrn[ks] = off(8 * (mi >> 1) + rr, 16 * ks + 8 * (mi & 1));
  }
  const uint32_t o_v0 = off(g, colg + 2 * tq), o_v1 = off(g + 8, colg + 2 * tq);
  const uint32_t o_st = (colw / Cfg::OSUB) * Cfg::OSUB_BYTES +
                        swz<Cfg::ORB>((8 * (mi & 1) + rr) * Cfg::ORB + (colw % Cfg::OSUB) * 2);
  constexpr uint32_t CHUNK_ROWS_BYTES = 16 * RB;  // 16 rows of a sub-tile
  constexpr uint32_t CHUNK_ROWS_OBYTES = 16 * Cfg::ORB;
  const uint32_t sL = sbase + Cfg::L_OFF;

  // The state as m16n8 fp32 accumulators.
  //   WC = 8:  W[:, colg .. colg+7];    tile mt holds rows 16mt .. 16mt+15 of W.
  //   WC = 16: W^T[colg .. colg+15, :]; tile j holds columns 8j .. 8j+7 of W^T (rows of W).
  float wc[WC == 8 ? KS : D / 8][4];
  {
    const float* w0 = p.W0 ? p.W0 + (size_t)stream * D * D : nullptr;
    if constexpr (WC == 8) {
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float2 v = make_float2(0.f, 0.f);
          if (w0) v = *reinterpret_cast<const float2*>(w0 + (16 * mt + 8 * h + g) * D + colg +
                                                       2 * tq);
          wc[mt][2 * h] = v.x;
          wc[mt][2 * h + 1] = v.y;
        }
    } else {
#pragma unroll
      for (int jt = 0; jt < D / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          wc[jt][e] = w0 ? w0[row * D + colg + g] : 0.f;
          wc[jt][2 + e] = w0 ? w0[row * D + colg + g + 8] : 0.f;
        }
    }
  }
  // WC = 16 operand addresses: K rows as the B operand of W^T K^T, K via ldmatrix.trans as the
  // B operand of the update, V^T in accumulator order, and the 16-column output tile.
  uint32_t o_brow[KS], o_btrn[KS];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    o_brow[ks] = off(8 * (mi >> 1) + rr, 16 * ks + 8 * (mi & 1));
    o_btrn[ks] = off(8 * (mi & 1) + rr, 16 * ks + 8 * (mi >> 1));
  }
  const uint32_t o_vt = off(8 * (mi >> 1) + rr, colg + 8 * (mi & 1));
  const uint32_t o_st16 =
      (colw / Cfg::OSUB) * Cfg::OSUB_BYTES +
      swz<Cfg::ORB>((8 * (mi & 1) + rr) * Cfg::ORB + ((colw + 8 * (mi >> 1)) % Cfg::OSUB) * 2);

  bool ok = true;
  for (int j = 0; j < nstg; ++j) {
    const int s = j % NSTAGE;
    const bool got = mbar_wait(full_bar + 8 * s, (j / NSTAGE) & 1, p.err);
    const uint32_t sQ = sbase + s * Cfg::STAGE_BYTES;
    const uint32_t sK = sQ + Cfg::TILE_BYTES;
    const uint32_t sV = sK + Cfg::TILE_BYTES;
    const uint32_t sEta = sQ + 3 * Cfg::TILE_BYTES;
    const uint32_t sO = sbase + Cfg::OUT_OFF + (j & 1) * Cfg::OTILE_BYTES;
    const int chunks = got ? min(R, T - j * R) / 16 : 0;

    // ---- causal scores of this stage: piece (chunk cc, score columns 8jj..8jj+7) per warp,
    //      stored negated and masked as the A fragments of -mask(Q_c K_c^T).
    for (int pc = warp; pc < (WC == 8 ? 2 * chunks : 0); pc += NW) {
      const int cc = pc >> 1, jj = pc & 1;
      float lc[4] = {};
#pragma unroll
      for (int kp = 0; kp < (KS + 1) / 2; ++kp) {
        // B = K^T (K = d, N = score columns): rows 8jj.. of K, matrices (k lo) (k hi) of two
        // consecutive k-steps.
        uint32_t kb[4], qa[4];
        ldsm_x4(sK + cc * CHUNK_ROWS_BYTES + off(8 * jj + rr, 32 * kp + 8 * mi), kb);
        ldsm_x4(sQ + cc * CHUNK_ROWS_BYTES + o_arow[2 * kp], qa);
        mma16816(lc, qa[0], qa[1], qa[2], qa[3], kb[0], kb[1]);
        if (2 * kp + 1 < KS) {
          ldsm_x4(sQ + cc * CHUNK_ROWS_BYTES + o_arow[2 * kp + 1], qa);
          mma16816(lc, qa[0], qa[1], qa[2], qa[3], kb[2], kb[3]);
        }
      }
      // keep s <= t: s = 8jj + 2tq + e, t = g (+8)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (8 * jj + 2 * tq + (i & 1) > g + 8 * (i >> 1)) lc[i] = 0.f;
      st_shared_v2(sL + cc * 512 + lane * 16 + jj * 8, pack_bf16(-lc[0], -lc[1]),
                   pack_bf16(-lc[2], -lc[3]));
    }
    if constexpr (WC == 8) {
    named_bar_sync(1, 32 * NW);

    // Per chunk: operand loads, the chain, then the outputs. A warp issues in order and shared
    // stores may alias later shared loads, so in a full stage the loads of chunk c+1 are placed
    // in program order between chunk c's chain and its outputs: they then overlap chunk c's
    // output products. A partial last stage runs the plain rolled loop.
    struct Ops {
      uint32_t ka[KS][4], kt[KS][4], qa[KS][4], la[4], v0, v1;
      float eg, eg8;
    };
    auto load = [&](Ops& o, const int c) {
      const uint32_t cb = c * CHUNK_ROWS_BYTES;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        ldsm_x4(sK + cb + o_arow[ks], o.ka[ks]);
        ldsm_x4_t(sK + cb + o_atrn[ks], o.kt[ks]);
      }
      o.v0 = ld_shared_u32(sV + cb + o_v0);
      o.v1 = ld_shared_u32(sV + cb + o_v1);
      o.eg = ld_shared_f32(sEta + 4 * (16 * c + g));
      o.eg8 = ld_shared_f32(sEta + 4 * (16 * c + g + 8));
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) ldsm_x4(sQ + cb + o_arow[ks], o.qa[ks]);
      ld_shared_v4(sL + c * 512 + lane * 16, o.la);
    };
    // chain: bf16(W) -> P = K W -> E -> W -= K^T E; returns bf16(W) and E as B fragments.
    auto chain = [&](const Ops& o, uint32_t (&wb)[KS][2], uint32_t& eb0, uint32_t& eb1) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        wb[ks][0] = movm_t(pack_bf16(wc[ks][0], wc[ks][1]));
        wb[ks][1] = movm_t(pack_bf16(wc[ks][2], wc[ks][3]));
      }
      float pa[4] = {}, pb[4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        if (ks & 1)
          mma16816(pb, o.ka[ks][0], o.ka[ks][1], o.ka[ks][2], o.ka[ks][3], wb[ks][0], wb[ks][1]);
        else
          mma16816(pa, o.ka[ks][0], o.ka[ks][1], o.ka[ks][2], o.ka[ks][3], wb[ks][0], wb[ks][1]);
      }
      const float e0 = (pa[0] + pb[0] - bf16_lo(o.v0)) * o.eg;
      const float e1 = (pa[1] + pb[1] - bf16_hi(o.v0)) * o.eg;
      const float e2 = (pa[2] + pb[2] - bf16_lo(o.v1)) * o.eg8;
      const float e3 = (pa[3] + pb[3] - bf16_hi(o.v1)) * o.eg8;
      eb0 = movm_t(pack_bf16(e0, e1));  // B fragment: E tokens 0-7
      eb1 = movm_t(pack_bf16(e2, e3));  // B fragment: E tokens 8-15
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
        mma16816(wc[mt], o.kt[mt][0], o.kt[mt][1], o.kt[mt][2], o.kt[mt][3], eb0 ^ 0x80008000u,
                 eb1 ^ 0x80008000u);
    };
    // outputs: O = Q W - mask(Q K^T) E   (W is the chunk-start state)
    auto output = [&](const Ops& o, const int c, const uint32_t (&wb)[KS][2], uint32_t eb0,
                      uint32_t eb1) {
      float oa[4] = {}, ob[4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        if (ks & 1)
          mma16816(ob, o.qa[ks][0], o.qa[ks][1], o.qa[ks][2], o.qa[ks][3], wb[ks][0], wb[ks][1]);
        else
          mma16816(oa, o.qa[ks][0], o.qa[ks][1], o.qa[ks][2], o.qa[ks][3], wb[ks][0], wb[ks][1]);
      }
      mma16816(oa, o.la[0], o.la[1], o.la[2], o.la[3], eb0, eb1);
      stsm_x2(sO + c * CHUNK_ROWS_OBYTES + o_st, pack_bf16(oa[0] + ob[0], oa[1] + ob[1]),
              pack_bf16(oa[2] + ob[2], oa[3] + ob[3]));
    };
    if (chunks == Cfg::CPS) {
      Ops ops[2];
      load(ops[0], 0);
#pragma unroll
      for (int c = 0; c < Cfg::CPS; ++c) {
        uint32_t wb[KS][2], eb0, eb1;
        chain(ops[c & 1], wb, eb0, eb1);
        if (c + 1 < Cfg::CPS) load(ops[(c + 1) & 1], c + 1);
        output(ops[c & 1], c, wb, eb0, eb1);
      }
    } else {
#pragma unroll 1
      for (int c = 0; c < chunks; ++c) {
        Ops o;
        uint32_t wb[KS][2], eb0, eb1;
        load(o, c);
        chain(o, wb, eb0, eb1);
        output(o, c, wb, eb0, eb1);
      }
    }

    } else {
    // WC = 16: the warp keeps W^T[16 cols, :]; its accumulator layout packed to bf16 is the A
    // operand of the next chunk's W^T K_c^T, so the chain needs no register transposes.
    struct Ops16 {
      uint32_t kb[KS][4], kt[KS][4], qa[KS][4], vt[4];
      float e0, e1, e8, e9;
    };
    auto load16 = [&](Ops16& o, const int c) {
      const uint32_t cb = c * CHUNK_ROWS_BYTES;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        ldsm_x4(sK + cb + o_brow[ks], o.kb[ks]);
        ldsm_x4_t(sK + cb + o_btrn[ks], o.kt[ks]);
      }
      ldsm_x4_t(sV + cb + o_vt, o.vt);
      o.e0 = ld_shared_f32(sEta + 4 * (16 * c + 2 * tq));
      o.e1 = ld_shared_f32(sEta + 4 * (16 * c + 2 * tq + 1));
      o.e8 = ld_shared_f32(sEta + 4 * (16 * c + 8 + 2 * tq));
      o.e9 = ld_shared_f32(sEta + 4 * (16 * c + 9 + 2 * tq));
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) ldsm_x4(sQ + cb + o_arow[ks], o.qa[ks]);
    };
    // chain: bf16(W^T) -> P^T = W^T K^T -> E^T -> W^T -= E^T K; returns the A fragments of
    // bf16(W^T) and of E^T.
    auto chain16 = [&](const Ops16& o, uint32_t (&wa)[KS][4], uint32_t (&ea)[4]) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        wa[ks][0] = pack_bf16(wc[2 * ks][0], wc[2 * ks][1]);
        wa[ks][1] = pack_bf16(wc[2 * ks][2], wc[2 * ks][3]);
        wa[ks][2] = pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]);
        wa[ks][3] = pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]);
      }
      float pa[2][4] = {}, pb[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        float (&acc)[2][4] = (ks & 1) ? pb : pa;
        mma16816(acc[0], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], o.kb[ks][0], o.kb[ks][1]);
        mma16816(acc[1], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], o.kb[ks][2], o.kb[ks][3]);
      }
      float E[2][4];
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        const float ea0 = n ? o.e8 : o.e0, ea1 = n ? o.e9 : o.e1;
        E[n][0] = (pa[n][0] + pb[n][0] - bf16_lo(o.vt[2 * n])) * ea0;
        E[n][1] = (pa[n][1] + pb[n][1] - bf16_hi(o.vt[2 * n])) * ea1;
        E[n][2] = (pa[n][2] + pb[n][2] - bf16_lo(o.vt[2 * n + 1])) * ea0;
        E[n][3] = (pa[n][3] + pb[n][3] - bf16_hi(o.vt[2 * n + 1])) * ea1;
      }
      ea[0] = pack_bf16(E[0][0], E[0][1]);
      ea[1] = pack_bf16(E[0][2], E[0][3]);
      ea[2] = pack_bf16(E[1][0], E[1][1]);
      ea[3] = pack_bf16(E[1][2], E[1][3]);
      const uint32_t n0 = ea[0] ^ 0x80008000u, n1 = ea[1] ^ 0x80008000u;
      const uint32_t n2 = ea[2] ^ 0x80008000u, n3 = ea[3] ^ 0x80008000u;
#pragma unroll
      for (int jp = 0; jp < KS; ++jp) {
        mma16816(wc[2 * jp], n0, n1, n2, n3, o.kt[jp][0], o.kt[jp][1]);
        mma16816(wc[2 * jp + 1], n0, n1, n2, n3, o.kt[jp][2], o.kt[jp][3]);
      }
    };
    // outputs: O[:, 16 cols] = Q W - mask(Q K^T) E. The warp forms the causal scores itself from
    // the Q and K fragments it already holds (A = Q rows, B = K rows), so no scores cross warps.
    auto output16 = [&](const Ops16& o, const int c, const uint32_t (&wa)[KS][4],
                        const uint32_t (&ea)[4]) {
      float lc[2][4] = {}, ld[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        float (&acc)[2][4] = (ks & 1) ? ld : lc;
        mma16816(acc[0], o.qa[ks][0], o.qa[ks][1], o.qa[ks][2], o.qa[ks][3], o.kb[ks][0], o.kb[ks][1]);
        mma16816(acc[1], o.qa[ks][0], o.qa[ks][1], o.qa[ks][2], o.qa[ks][3], o.kb[ks][2], o.kb[ks][3]);
      }
      // keep s <= t: entry (jj, i) is t = g + 8 (i >> 1), s = 8 jj + 2 tq + (i & 1)
      float m[2][4];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          m[jj][i] = (8 * jj + 2 * tq + (i & 1) > g + 8 * (i >> 1)) ? 0.f : -(lc[jj][i] + ld[jj][i]);
      const uint32_t la0 = pack_bf16(m[0][0], m[0][1]), la1 = pack_bf16(m[0][2], m[0][3]);
      const uint32_t la2 = pack_bf16(m[1][0], m[1][1]), la3 = pack_bf16(m[1][2], m[1][3]);
      float oa[2][4] = {}, ob[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        float (&acc)[2][4] = (ks & 1) ? ob : oa;
        mma16816(acc[0], o.qa[ks][0], o.qa[ks][1], o.qa[ks][2], o.qa[ks][3], wa[ks][0], wa[ks][2]);
        mma16816(acc[1], o.qa[ks][0], o.qa[ks][1], o.qa[ks][2], o.qa[ks][3], wa[ks][1], wa[ks][3]);
      }
      mma16816(oa[0], la0, la1, la2, la3, ea[0], ea[2]);
      mma16816(oa[1], la0, la1, la2, la3, ea[1], ea[3]);
      stsm_x4(sO + c * CHUNK_ROWS_OBYTES + o_st16,
              pack_bf16(oa[0][0] + ob[0][0], oa[0][1] + ob[0][1]),
              pack_bf16(oa[0][2] + ob[0][2], oa[0][3] + ob[0][3]),
              pack_bf16(oa[1][0] + ob[1][0], oa[1][1] + ob[1][1]),
              pack_bf16(oa[1][2] + ob[1][2], oa[1][3] + ob[1][3]));
    };
    if (chunks == Cfg::CPS) {
      Ops16 ops[2];
      load16(ops[0], 0);
#pragma unroll
      for (int c = 0; c < Cfg::CPS; ++c) {
        uint32_t wa[KS][4], ea[4];
        chain16(ops[c & 1], wa, ea);
        if (c + 1 < Cfg::CPS) load16(ops[(c + 1) & 1], c + 1);
        output16(ops[c & 1], c, wa, ea);
      }
    } else {
#pragma unroll 1
      for (int c = 0; c < chunks; ++c) {
        Ops16 o;
        uint32_t wa[KS][4], ea[4];
        load16(o, c);
        chain16(o, wa, ea);
        output16(o, c, wa, ea);
      }
    }
    }

    // Inputs of this stage are consumed; hand the slot back to the producer.
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar + 8 * s);
    // Output tile -> global (TMA store).
    fence_proxy_async_smem();
    const bool failed = named_bar_or(1, 32 * NW, !got);
    if (!failed && threadIdx.x == 0) {
#pragma unroll
      for (int os = 0; os < Cfg::NOSUB; ++os)
        tma_store_3d(&tmO, sO + os * Cfg::OSUB_BYTES, col_cta + os * Cfg::OSUB, j * R, stream);
      bulk_commit();
      bulk_wait_read<1>();  // the other output buffer is free again
    }
    named_bar_sync(1, 32 * NW);
    if (failed) {
      ok = false;
      break;
    }
  }
  if (threadIdx.x == 0) bulk_wait<0>();
  if (!ok) return;

  // Final state.
  float* wo = p.Wout + (size_t)stream * D * D;
  if constexpr (WC == 8) {
#pragma unroll
    for (int mt = 0; mt < KS; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        *reinterpret_cast<float2*>(wo + (16 * mt + 8 * h + g) * D + colg + 2 * tq) =
            make_float2(wc[mt][2 * h], wc[mt][2 * h + 1]);
  } else {
#pragma unroll
    for (int jt = 0; jt < D / 8; ++jt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = 8 * jt + 2 * tq + e;
        wo[row * D + colg + g] = wc[jt][e];
        wo[row * D + colg + g + 8] = wc[jt][2 + e];
      }
  }
}

template <int D, int NW, int CPS = 4, int WC = 8>
int launch_cfg(const StateArgs& a, const LaunchCtx& ctx) {
  using Cfg = DualCfg<D, NW, CPS, WC>;
  const int BH = a.B * a.H;
  CUtensorMap tq, tk, tv, to;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)a.T * D * 2};
  const uint32_t box_in[3] = {(uint32_t)Cfg::SUB, (uint32_t)Cfg::R, 1};
  const uint32_t box_out[3] = {(uint32_t)Cfg::OSUB, (uint32_t)Cfg::R, 1};
  auto sw = [](int rb) {
    return rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                     : (rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  };
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_tmap_3d(&tq, a.Q, bf, dims, strides, box_in, sw(Cfg::RB), ctx.msg) ||
      !make_tmap_3d(&tk, a.K, bf, dims, strides, box_in, sw(Cfg::RB), ctx.msg) ||
      !make_tmap_3d(&tv, a.V, bf, dims, strides, box_in, sw(Cfg::RB), ctx.msg) ||
      !make_tmap_3d(&to, a.O, bf, dims, strides, box_out, sw(Cfg::ORB), ctx.msg))
    return kCuda;
  auto kern = dual_mma_kernel<D, NW, CPS, WC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg::SMEM);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  DualParams p{a.eta, a.eta_scalar, a.S0, a.S_out, a.T, ctx.err};
  kern<<<BH * Cfg::NG, Cfg::THREADS, Cfg::SMEM, ctx.stream>>>(tq, tk, tv, to, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual_mma launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

bool dual_mma_supported(int d, int C, int dt) {
  return (dt == 1 && C == 16 && (d == 32 || d == 64 || d == 128)) || dual_tc_supported(d, C, dt);
}

// Whether launch_dual_mma runs the d = 64 stage kernel for this shape under the current tuning
// choices, i.e. whether it accepts O = nullptr (the state-only form).
bool dual_state_only_supported(int d, int C, int dt) {
  const int kernel = tuning(kTuneDualKernel);
  if (kernel == kDualKernelSplit || kernel == kDualKernelGram || kernel == kDualKernelRegGram)
    return false;
  return dual_tc_supported(d, C, dt) &&
         (C != 16 || kernel == kDualKernelAuto || kernel == kDualKernelTensor);
}

int launch_dual_mma(const StateArgs& a, const LaunchCtx& ctx) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int streams = a.B * a.H;
  const int forced_split = tuning(kTuneDualColumnSplit);
  const int kernel = tuning(kTuneDualKernel);
  // d = 64: the chain on warp MMAs with the outputs per 128-token stage on tcgen05 (dual_tc.cu)
  // measured fastest on the 125M- and 1.3B-layer shapes; the all-warp-MMA forms below remain
  // selectable through ttt_set_tuning("dual_kernel", ...).
  // d = 64, C = 16, on request: the chain on some SMs, the stage products on others of the same
  // cluster (dual_xsm.cu). Correct, but measured slower than one SM doing both (the hand-off
  // moves the bound to the output CTA's epilogue and to the chain's wait for its slot), so the
  // automatic choice is the single-SM stage kernel below.
  if (dual_xsm_applicable(a.d, a.C, a.dt) && kernel == kDualKernelSplit) {
    int n_clusters = 0;
    const int ks = dual_xsm_plan(streams, sms, &n_clusters);
    const int r = ks ? launch_dual_xsm(a, ks, n_clusters, ctx) : kUnsupported;
    if (r == kUnsupported)
      *ctx.msg = "dual form: the split form needs one more SM per one or two streams, and its "
                 "clusters resident at once";
    return r;
  }
  if (kernel == kDualKernelGram && dual_gram_supported(a.d, a.C, a.dt))
    return launch_dual_gram(a, ctx);
  if (kernel == kDualKernelRegGram && dual_gram_supported(a.d, a.C, a.dt))
    return launch_dual_rgram(a, ctx);
  // (C = 32 and 64 exist only in that form)
  if (a.d == 64 && (a.C != 16 || kernel == kDualKernelAuto || kernel == kDualKernelTensor)) {
    const int split = (forced_split == 1 || forced_split == 2 || forced_split == 4)
                          ? forced_split
                          : dual_tc_split(streams, sms);
    return launch_dual_tc(a, split, ctx);
  }
  // CTAs per stream for the all-warp-MMA kernels. Each CTA holds one stream's column slice for
  // the whole sequence, and one CTA fits per SM, so a stream is split over two SMs only when
  // all CTAs still fit in one wave.
  const int split =
      (forced_split == 1 || forced_split == 2) ? forced_split : (2 * streams <= sms ? 2 : 1);
  switch (a.d) {
    case 32:
      return split == 2 ? launch_cfg<32, 2>(a, ctx) : launch_cfg<32, 4>(a, ctx);
    case 64: {
      // 16 columns per warp (W^T form, the warp computes its own causal scores) with 8-chunk
      // stages measured faster than 8 columns per warp; chain and output products on paired
      // warps (dual_pair.cu) measured faster when a stream is split over two CTAs. The other
      // forms are kept as tuning choices.
      const int wcols = tuning(kTuneDualWarpCols) == 8 ? 8 : 16;
      const bool pair = kernel == kDualKernelPair ? true
                        : kernel == kDualKernelWarp ? false
                                                    : split == 2;
      if (wcols == 16 && pair) return launch_dual_pair(a, ctx, split);
      if (wcols == 16)
        return split == 2 ? launch_cfg<64, 2, 8, 16>(a, ctx) : launch_cfg<64, 4, 8, 16>(a, ctx);
      if (tuning(kTuneDualStageChunks) == 4)
        return split == 2 ? launch_cfg<64, 4>(a, ctx) : launch_cfg<64, 8>(a, ctx);
      return split == 2 ? launch_cfg<64, 4, 8>(a, ctx) : launch_cfg<64, 8, 8>(a, ctx);
    }
    case 128:
      return split == 2 ? launch_cfg<128, 8>(a, ctx) : launch_cfg<128, 16>(a, ctx);
  }
  *ctx.msg = "dual_mma: unsupported head dim";
  return kUnsupported;
}

}  // namespace ttt
