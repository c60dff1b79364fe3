// TTT-Linear mini-batch dual form, bf16 inputs, chunk C = 16: paired-warp tensor-core path.
//
// Same arithmetic as the single-warp path in dual_mma.cu (source: "Learning to (Learn at Test
// Time)" reading, section on mini-batch TTT and the dual form):
//     G   = K_c W - V_c,   E = diag(eta_c) G
//     O_c = Q_c W - tril(Q_c K_c^T) E
//     W   = W - K_c^T E
// with each 16-column slice of W^T held as m16n8 fp32 accumulators in registers.
//
// The chunk chain (bf16(W^T) -> W^T K_c^T -> E -> W^T -= E^T K_c) and the output products
// (causal scores, Q_c W, scores * E) are split between two warps that share an SM
// sub-partition: the chain warp runs only the recurrence and hands bf16(W^T) and bf16(E) of every
// chunk to its output warp through two shared-memory slots; the output warp forms O_c. The
// output warp's MMAs fill the issue slots that the chain warp leaves idle while it waits on its
// own dependent results. The hand-off runs in lockstep on two named barriers per pair
// (published / consumed): the chain warp computes chunk c+1 while the output warp works on
// chunk c, and publishes c+1 once c has been read.
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace ttt {
namespace {

template <int D, int NP, int CPS_>
struct PairCfg {
  static constexpr int C = 16;
  static constexpr int CPS = CPS_;                 // chunks per pipeline stage
  static constexpr int R = C * CPS;                // token rows per stage
  static constexpr int SUB = D >= 64 ? 64 : D;     // columns per swizzled sub-tile
  static constexpr int RB = SUB * 2;               // bytes per sub-tile row
  static constexpr int NSUB = D / SUB;
  static constexpr int SUB_BYTES = R * RB;
  static constexpr int TILE_BYTES = NSUB * SUB_BYTES;
  static constexpr int COLS = 16 * NP;             // output columns per CTA
  static constexpr int NG = D / COLS;              // CTAs per stream
  static constexpr int OSUB = COLS >= 64 ? 64 : COLS;
  static constexpr int ORB = OSUB * 2;
  static constexpr int NOSUB = COLS / OSUB;
  static constexpr int OSUB_BYTES = R * ORB;
  static constexpr int OTILE_BYTES = NOSUB * OSUB_BYTES;
  static constexpr int ETA_BYTES = R * 4 <= 1024 ? 1024 : 2048;
  static constexpr int STAGE_BYTES = 3 * TILE_BYTES + ETA_BYTES;
  static constexpr int KS = D / 16;                // 16-wide k-steps over d
  // hand-off slot: KS x 4 registers of bf16(W^T) fragments and 4 of bf16(E), per lane
  static constexpr int HREGS = 4 * KS + 4;
  static constexpr int HSLOT_BYTES = HREGS * 32 * 4;
  static constexpr int HS = 2;                     // slots per warp pair
  static constexpr int H_BYTES = NP * HS * HSLOT_BYTES;
  static constexpr int BUDGET = 220 * 1024;
  static constexpr int NSTAGE_FIT = (BUDGET - 2 * OTILE_BYTES - H_BYTES) / STAGE_BYTES;
  static constexpr int NSTAGE = NSTAGE_FIT > 8 ? 8 : NSTAGE_FIT;
  static constexpr int OUT_OFF = NSTAGE * STAGE_BYTES;
  static constexpr int H_OFF = OUT_OFF + 2 * OTILE_BYTES;
  static constexpr int BAR_OFF = H_OFF + H_BYTES;
  static constexpr int SMEM = 1024 + BAR_OFF + 16 * NSTAGE;
  static constexpr int THREADS = 32 * (2 * NP + 1);
  static_assert(NSTAGE >= 2, "pipeline depth");
  static_assert(D % COLS == 0, "column split");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(NP <= 4, "named barrier ids 2 .. 2 + 2 NP");
};

struct PairParams {
  const float* eta;
  float eta_scalar;
  const float* W0;
  float* Wout;
  int T;
  unsigned* err;
  uint64_t wait_ns;   // limit of every pipeline wait (copies in flight: a fixed second)
};

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
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
__device__ __forceinline__ void named_bar_arrive(int id, int threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}

// Warps 0 .. NP-1: chain warps; NP .. 2NP-1: output warps (output warp NP + i pairs with chain
// warp i on the same sub-partition); warp 2NP: TMA producer.
template <int D, int NP, int CPS>
__global__ void __launch_bounds__(PairCfg<D, NP, CPS>::THREADS, 1)
    dual_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmO, const PairParams p) {
  using Cfg = PairCfg<D, NP, CPS>;
  constexpr int R = Cfg::R, KS = Cfg::KS, NSTAGE = Cfg::NSTAGE, RB = Cfg::RB, HS = Cfg::HS;
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
      mbar_init(empty_bar + 8 * s, 2 * NP);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 2 * NP) {
    // ---------------------------------------------------------------- producer (one lane)
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int j = 0; j < nstg; ++j) {
        const int s = j % NSTAGE;
        if (j >= NSTAGE &&
            !mbar_wait(empty_bar + 8 * s, ((j / NSTAGE) - 1) & 1, p.err, p.wait_ns))
          break;
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

  const bool is_chain = warp < NP;
  const int pair = is_chain ? warp : warp - NP;
  const int g = lane >> 2, tq = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;   // ldmatrix: which 8x8 matrix / which row
  const int colw = 16 * pair;                // first column of this pair inside the CTA's slice
  const int colg = col_cta + colw;           // ... and in the stream's W
  auto off = [&](int row, int col) -> uint32_t {
    return (col / Cfg::SUB) * Cfg::SUB_BYTES + swz<RB>(row * RB + (col % Cfg::SUB) * 2);
  };
  constexpr uint32_t CHUNK_ROWS_BYTES = 16 * RB;
  constexpr uint32_t CHUNK_ROWS_OBYTES = 16 * Cfg::ORB;
  // K rows as the B operand of W^T K^T (and of Q K^T), K via ldmatrix.trans as the B operand of
  // the update, Q rows as the A operand, V^T in accumulator order.
  uint32_t o_brow[KS], o_btrn[KS], o_arow[KS];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    o_brow[ks] = off(8 * (mi >> 1) + rr, 16 * ks + 8 * (mi & 1));
    o_btrn[ks] = off(8 * (mi & 1) + rr, 16 * ks + 8 * (mi >> 1));
    o_arow[ks] = off(8 * (mi & 1) + rr, 16 * ks + 8 * (mi >> 1));
  }
  const uint32_t o_vt = off(8 * (mi >> 1) + rr, colg + 8 * (mi & 1));
  const uint32_t o_st16 =
      (colw / Cfg::OSUB) * Cfg::OSUB_BYTES +
      swz<Cfg::ORB>((8 * (mi & 1) + rr) * Cfg::ORB + ((colw + 8 * (mi >> 1)) % Cfg::OSUB) * 2);
  // hand-off slot of this pair: [register group][lane][4 x u32]
  const uint32_t hbase = sbase + Cfg::H_OFF + pair * HS * Cfg::HSLOT_BYTES + lane * 16;
  // named barriers of the pair (64 threads): chunk published / chunk consumed
  const int bar_pub = 2 + pair, bar_con = 2 + NP + pair;

  if (is_chain) {
    // ------------------------------------------------------------------ chain warp
    // W^T[colg .. colg+15, :] as accumulators: tile j holds columns 8j .. 8j+7 of W^T.
    float wc[D / 8][4];
    {
      const float* w0 = p.W0 ? p.W0 + (size_t)stream * D * D : nullptr;
#pragma unroll
      for (int jt = 0; jt < D / 8; ++jt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * jt + 2 * tq + e;
          wc[jt][e] = w0 ? w0[row * D + colg + g] : 0.f;
          wc[jt][2 + e] = w0 ? w0[row * D + colg + g + 8] : 0.f;
        }
    }
    struct Ops {
      uint32_t kb[KS][4], kt[KS][4], vt[4];
      float e0, e1, e8, e9;
    };
    bool ok = true;
    int gc = 0;   // chunks handed off so far
    for (int j = 0; j < nstg; ++j) {
      const int s = j % NSTAGE;
      // After a failed wait the warp keeps the hand-off protocol (with meaningless data) so
      // that its output warp never waits on a barrier that no one will reach.
      if (ok && !mbar_wait(full_bar + 8 * s, (j / NSTAGE) & 1, p.err, p.wait_ns)) ok = false;
      const uint32_t sQ = sbase + s * Cfg::STAGE_BYTES;
      const uint32_t sK = sQ + Cfg::TILE_BYTES;
      const uint32_t sV = sK + Cfg::TILE_BYTES;
      const uint32_t sEta = sQ + 3 * Cfg::TILE_BYTES;
      const int chunks = min(R, T - j * R) / 16;
      auto load = [&](Ops& o, const int c) {
        const uint32_t cb = c * CHUNK_ROWS_BYTES;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          ldsm_x4(sK + cb + o_brow[ks], o.kb[ks]);
          ldsm_x4_t(sK + cb + o_btrn[ks], o.kt[ks]);
        }
        ldsm_x4_t(sV + cb + o_vt, o.vt);
        o.e0 = lds_f32(sEta + 4 * (16 * c + 2 * tq));
        o.e1 = lds_f32(sEta + 4 * (16 * c + 2 * tq + 1));
        o.e8 = lds_f32(sEta + 4 * (16 * c + 8 + 2 * tq));
        o.e9 = lds_f32(sEta + 4 * (16 * c + 9 + 2 * tq));
      };
      // bf16(W^T) -> P^T = W^T K^T -> E^T -> W^T -= E^T K; hands bf16(W^T) and bf16(E^T) over.
      auto step = [&](const Ops& o) {
        uint32_t wa[KS][4];
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
        uint32_t ea[4];
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
        // hand the chunk's operands to the output warp once it has read the previous chunk
        // (slot gc % 2 was last read for chunk gc - 2, before that)
        if (gc >= 1) named_bar_sync(bar_con, 64);
        const uint32_t h = hbase + (gc & 1) * Cfg::HSLOT_BYTES;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
          sts128(h + ks * 512, make_uint4(wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3]));
        sts128(h + KS * 512, make_uint4(ea[0], ea[1], ea[2], ea[3]));
        named_bar_arrive(bar_pub, 64);
        ++gc;
      };
      if (chunks == Cfg::CPS) {
        Ops ops[2];
        load(ops[0], 0);
#pragma unroll
        for (int c = 0; c < Cfg::CPS; ++c) {
          if (c + 1 < Cfg::CPS) load(ops[(c + 1) & 1], c + 1);
          step(ops[c & 1]);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < chunks; ++c) {
          Ops o;
          load(o, c);
          step(o);
        }
      }
      // this warp's reads of the stage are done
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(empty_bar + 8 * s);
    }
    // the output warp's read of the last chunk
    if (gc >= 1) named_bar_sync(bar_con, 64);
    if (!ok) return;
    // Final state.
    float* wo = p.Wout + (size_t)stream * D * D;
#pragma unroll
    for (int jt = 0; jt < D / 8; ++jt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = 8 * jt + 2 * tq + e;
        wo[row * D + colg + g] = wc[jt][e];
        wo[row * D + colg + g + 8] = wc[jt][2 + e];
      }
    return;
  }

  // -------------------------------------------------------------------- output warp
  // O[:, 16 cols] = Q W - mask(Q K^T) E from the hand-off of the paired chain warp; the causal
  // scores come from the Q and K fragments this warp loads itself.
  int gc = 0;
  bool ok = true;
  for (int j = 0; j < nstg; ++j) {
    const int s = j % NSTAGE;
    // as in the chain warp, the hand-off protocol runs for every chunk even after a failure
    if (ok && !mbar_wait(full_bar + 8 * s, (j / NSTAGE) & 1, p.err, p.wait_ns)) ok = false;
    const uint32_t sQ = sbase + s * Cfg::STAGE_BYTES;
    const uint32_t sK = sQ + Cfg::TILE_BYTES;
    const uint32_t sO = sbase + Cfg::OUT_OFF + (j & 1) * Cfg::OTILE_BYTES;
    const int chunks = min(R, T - j * R) / 16;
#pragma unroll 1
    for (int c = 0; c < chunks; ++c) {
      named_bar_sync(bar_pub, 64);
      const uint32_t h = hbase + (gc & 1) * Cfg::HSLOT_BYTES;
      uint32_t wa[KS][4], ea[4];
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const uint4 v = lds128(h + ks * 512);
        wa[ks][0] = v.x;
        wa[ks][1] = v.y;
        wa[ks][2] = v.z;
        wa[ks][3] = v.w;
      }
      {
        const uint4 v = lds128(h + KS * 512);
        ea[0] = v.x;
        ea[1] = v.y;
        ea[2] = v.z;
        ea[3] = v.w;
      }
      named_bar_arrive(bar_con, 64);
      ++gc;
      const uint32_t cb = c * CHUNK_ROWS_BYTES;
      uint32_t qa[KS][4], kb[KS][4];
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        ldsm_x4(sQ + cb + o_arow[ks], qa[ks]);
        ldsm_x4(sK + cb + o_brow[ks], kb[ks]);
      }
      float lc[2][4] = {}, ld[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        float (&acc)[2][4] = (ks & 1) ? ld : lc;
        mma16816(acc[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], kb[ks][0], kb[ks][1]);
        mma16816(acc[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], kb[ks][2], kb[ks][3]);
      }
      // keep s <= t: entry (jj, i) is t = g + 8 (i >> 1), s = 8 jj + 2 tq + (i & 1)
      float m[2][4];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          m[jj][i] = (8 * jj + 2 * tq + (i & 1) > g + 8 * (i >> 1)) ? 0.f
                                                                     : -(lc[jj][i] + ld[jj][i]);
      const uint32_t la0 = pack_bf16(m[0][0], m[0][1]), la1 = pack_bf16(m[0][2], m[0][3]);
      const uint32_t la2 = pack_bf16(m[1][0], m[1][1]), la3 = pack_bf16(m[1][2], m[1][3]);
      float oa[2][4] = {}, ob[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        float (&acc)[2][4] = (ks & 1) ? ob : oa;
        mma16816(acc[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], wa[ks][0], wa[ks][2]);
        mma16816(acc[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], wa[ks][1], wa[ks][3]);
      }
      mma16816(oa[0], la0, la1, la2, la3, ea[0], ea[2]);
      mma16816(oa[1], la0, la1, la2, la3, ea[1], ea[3]);
      stsm_x4(sO + c * CHUNK_ROWS_OBYTES + o_st16,
              pack_bf16(oa[0][0] + ob[0][0], oa[0][1] + ob[0][1]),
              pack_bf16(oa[0][2] + ob[0][2], oa[0][3] + ob[0][3]),
              pack_bf16(oa[1][0] + ob[1][0], oa[1][1] + ob[1][1]),
              pack_bf16(oa[1][2] + ob[1][2], oa[1][3] + ob[1][3]));
    }
    // this warp's reads of the stage are done
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(empty_bar + 8 * s);
    // Output tile -> global (TMA store) by the first output warp, after all output warps.
    fence_proxy_async_smem();
    const bool failed = named_bar_or(1, 32 * NP, !ok);
    if (!failed && warp == NP && lane == 0) {
#pragma unroll
      for (int os = 0; os < Cfg::NOSUB; ++os)
        tma_store_3d(&tmO, sO + os * Cfg::OSUB_BYTES, col_cta + os * Cfg::OSUB, j * R, stream);
      bulk_commit();
      bulk_wait_read<1>();  // the other output buffer is free again
    }
    named_bar_sync(1, 32 * NP);
    ok = ok && !failed;
  }
  if (warp == NP && lane == 0) bulk_wait<0>();
}

template <int D, int NP, int CPS>
int launch_pair(const StateArgs& a, const LaunchCtx& ctx) {
  using Cfg = PairCfg<D, NP, CPS>;
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
  auto kern = dual_pair_kernel<D, NP, CPS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg::SMEM);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  const int limit = tuning(kTuneWaitLimitNs);
  PairParams p{a.eta, a.eta_scalar, a.S0, a.S_out, a.T, ctx.err,
               limit > 0 ? (uint64_t)limit : 4000000000ull};
  kern<<<BH * Cfg::NG, Cfg::THREADS, Cfg::SMEM, ctx.stream>>>(tq, tk, tv, to, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual_pair launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

int launch_dual_pair(const StateArgs& a, const LaunchCtx& ctx, int split) {
  if (a.d == 64) return split == 2 ? launch_pair<64, 2, 8>(a, ctx) : launch_pair<64, 4, 8>(a, ctx);
  *ctx.msg = "dual_pair: unsupported head dim";
  return kUnsupported;
}

}  // namespace ttt
