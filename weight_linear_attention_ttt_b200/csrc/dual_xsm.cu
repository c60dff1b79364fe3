// TTT-Linear mini-batch dual form, bf16 inputs, d = 64, chunk C = 16, with the serial chain and
// the output products on separate SMs of one thread-block cluster.
//
// Computes, per (batch, head) stream and chunk c (source: "RNN의 기억을 작은 모델로 바꾼다면:
// Test-Time Training 읽기", section "gradient를 효율적인 layer로 만드는 작업" for the mini-batch
// update and its dual form; section "읽는 동안 문제를 하나 더 푼다" for reading the updated model):
//     G = K_c W - V_c,   E = diag(eta_c) G,   O_c = Q_c W - tril(Q_c K_c^T) E,   W = W - K_c^T E
// in the stage form of dual_tc.cu: per 128-token stage with start state W_s,
//     O_stage = Q W_s - tril(Q K^T) E_stage.
//
// Why two kinds of CTA. The chain (bf16 W -> K_c W -> E -> W update) is serial over the sequence
// and latency-bound; on an SM that also runs the stage products on tcgen05 and their epilogue,
// the chain measured about 1.4x slower than alone (the output work competes with it for the
// tensor pipe and the issue slots even when nothing waits on it). Here a cluster of KS + 1 CTAs
// (KS = 1 or 2) holds
//   * KS chain CTAs, one per stream: 4 chain warps (16 columns of W each, the state in
//     registers), a TMA producer warp (K, V, rates) and a publisher thread that copies every
//     stage's -E^T and bf16(W_s)^T from its shared memory into the output CTA's pipeline stage
//     (a distributed-shared-memory bulk copy completing on the output CTA's mbarrier);
//   * one output CTA serving the cluster's streams stage by stage: a producer warp loads Q and K
//     by TMA into a pipeline stage, sets the stage's expected bytes (Q, K and the chain's copy)
//     and grants the stage to the chain CTA (a remote mbarrier arrival); an MMA warp issues
//     S = Q K^T, O = Q W_s and O += P (-E) on tcgen05 and, once a stage has landed, frees the
//     chain CTA's buffer (another remote arrival); four epilogue warps mask S into P
//     (TMEM -> TMEM) and store O.
// Every hand-off is an mbarrier phase in shared memory: no global memory, no fence, and the
// cluster's CTAs are co-scheduled. Every wait is bounded; a cluster barrier ends the kernel so
// that no CTA leaves while another may still reach its shared memory.
#include <algorithm>
#include <string>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int XD = 64;              // head dim
constexpr int XC = 16;              // chunk
constexpr int XR = 128;             // tokens per stage
constexpr int XCPS = XR / XC;       // chunks per stage
constexpr int XKS = XD / 16;        // 16-wide k-steps over d
constexpr int XTILE = XR * XD * 2;  // one [128][64] bf16 tile, 128-byte swizzle
constexpr int PART = 64 * 128;      // one [64][64] bf16 sub-tile (8 KB)
constexpr int SLOT = 3 * PART;      // -E^T tokens 0-63, tokens 64-127, bf16 W_s^T
constexpr int NGRANT = 4;           // grant barriers per chain CTA (grants run <= 3 stages ahead)
constexpr uint32_t XTM_S = 0, XTM_P = 256, XTM_O = 384;

template <int NC>
struct XCfg {
  static constexpr int COLS = 16 * NC;             // output columns per chain CTA (all of W)
  static_assert(COLS == XD, "one chain CTA per stream");
  // chain CTA
  static constexpr int C_NST = 3;
  static constexpr int C_STAGE = 2 * XTILE + 1024;  // K, V, rates (512 B, padded)
  static constexpr int C_ESUB = COLS * 128;         // one -E^T sub-tile (= PART)
  static constexpr int C_E_OFF = C_NST * C_STAGE;   // 2 buffers x 2 sub-tiles
  static constexpr int C_W_OFF = C_E_OFF + 4 * C_ESUB;
  static constexpr int C_END = C_W_OFF + 2 * C_ESUB;
  // output CTA
  static constexpr int O_NST = 3;
  static constexpr int O_STAGE = 2 * XTILE + SLOT;  // Q, K, then the chain CTA's copy
  static constexpr int O_OT_OFF = O_NST * O_STAGE;
  static constexpr int O_END = O_OT_OFF + XTILE;
  static constexpr int BAR_OFF = C_END > O_END ? C_END : O_END;
  static constexpr int SMEM = 1024 + BAR_OFF + 256;
  static constexpr int WARPS = NC + 2 > 6 ? NC + 2 : 6;
  static constexpr int THREADS = 32 * WARPS;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(C_ESUB == PART && C_STAGE % 1024 == 0 && O_STAGE % 1024 == 0, "layout");
};

struct XParams {
  const float* eta;
  float eta_scalar;
  const float* W0;
  float* Wout;
  int T, BH;
  int ks;               // streams (chain CTAs) per cluster; the output CTA has rank ks
  unsigned* err;
  uint64_t wait_ns;
};

__device__ __forceinline__ void xbar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ bool xbar_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
// The cluster-window address of a shared-memory location of CTA `rank`.
__device__ __forceinline__ uint32_t map_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void remote_arrive(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
// Bulk copy from this CTA's shared memory into another CTA's, completing on its mbarrier.
__device__ __forceinline__ void dsmem_copy(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                           uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, "
      "[%3];" ::"r"(dst_cluster),
      "r"(src), "r"(bytes), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
template <int RB>
__device__ __forceinline__ uint32_t xswz(uint32_t row, uint32_t colbyte) {
  return swz<RB>(row * RB + colbyte);
}

template <int NC>
__global__ void __launch_bounds__(XCfg<NC>::THREADS, 1)
    dual_xsm_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const XParams p) {
  using Cfg = XCfg<NC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + Cfg::BAR_OFF;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int nst = (T + XR - 1) / XR;
  const int rank = (int)cluster_rank();
  const int cid = (int)cluster_index();
  const int out_rank = p.ks;
  // barriers of both CTA kinds sit at the same offsets, so each side can name the other's
  const uint32_t c_full = bar, c_empty = bar + 24;     // chain: K/V ring (3)
  const uint32_t c_eready = bar + 48;                  // chain: -E and W_s stored (x2)
  const uint32_t c_efree = bar + 64;                   // chain: copy landed (x2, remote)
  const uint32_t c_grant = bar + 80;                   // chain: slot granted (x4, remote)
  const uint32_t o_full = bar + 112;                   // output: stage landed (3)
  const uint32_t o_empty = bar + 136;                  // output: stage consumed (3)
  const uint32_t o_sfull = bar + 160, o_pfull = bar + 176;
  const uint32_t o_ofull = bar + 192, o_ofree = bar + 208;
  const uint32_t o_mdone = bar + 224, o_tslot = bar + 232;
  // streams of this cluster that exist (the last cluster may hold fewer)
  const int nmine = max(0, min(p.ks, p.BH - cid * p.ks));

  if (threadIdx.x == 0) {
    if (rank < out_rank) {
      for (int s = 0; s < Cfg::C_NST; ++s) {
        mbar_init(c_full + 8 * s, 1);
        mbar_init(c_empty + 8 * s, NC);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(c_eready + 8 * b, NC);
        mbar_init(c_efree + 8 * b, 1);
      }
      for (int g = 0; g < NGRANT; ++g) mbar_init(c_grant + 8 * g, 1);
    } else {
      for (int s = 0; s < Cfg::O_NST; ++s) {
        mbar_init(o_full + 8 * s, 1);
        mbar_init(o_empty + 8 * s, 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(o_sfull + 8 * b, 1);
        mbar_init(o_pfull + 8 * b, 4);
        mbar_init(o_ofull + 8 * b, 1);
        mbar_init(o_ofree + 8 * b, 4);
      }
      mbar_init(o_mdone, 1);
    }
    fence_mbar_init();
  }
  if (rank < out_rank) {
    // -E buffers start at zero: a partial last stage leaves the absent chunks' columns as they
    // are, and the masked product multiplies them by zero scores (they must be finite)
    for (int i = threadIdx.x; i < 4 * Cfg::C_ESUB / 16; i += Cfg::THREADS)
      sts128(sbase + Cfg::C_E_OFF + 16 * i, make_uint4(0u, 0u, 0u, 0u));
    fence_proxy_async_smem();
  } else if (warp == 1) {
    umma::tmem_alloc(o_tslot, 512);
  }
  umma::fence_before();
  // every CTA's barriers are initialised before any CTA of the cluster touches them
  cluster_sync_all();
  umma::fence_after();

  if (rank < out_rank) {
    // ================================================================ chain CTA
    const int stream = cid * p.ks + rank;
    const bool active = rank < nmine;
    const int col_cta = 0;
    const uint32_t full = c_full, empty = c_empty, eready = c_eready, efree = c_efree;
    if (active && warp == NC) {
      // ---------------------------------------------------------------- TMA producer
      if (lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        int issued = 0;
        for (int j = 0; j < nst; ++j) {
          const int s = j % Cfg::C_NST;
          if (j >= Cfg::C_NST &&
              !mbar_wait(empty + 8 * s, ((j / Cfg::C_NST) - 1) & 1, p.err, p.wait_ns))
            break;
          const int rows = min(XR, T - j * XR);
          const uint32_t fb = full + 8 * s;
          const uint32_t st = sbase + s * Cfg::C_STAGE;
          if (!p.eta)
            for (int i = 0; i < XR; ++i) stsf(st + 2 * XTILE + 4 * i, p.eta_scalar);
          mbar_arrive_expect_tx(fb, 2 * XTILE + (p.eta ? rows * 4 : 0));
          tma_load_3d(st, &tmK, fb, 0, j * XR, stream);
          tma_load_3d(st + XTILE, &tmV, fb, 0, j * XR, stream);
          if (p.eta)
            bulk_load(st + 2 * XTILE, p.eta + (size_t)stream * T + (size_t)j * XR, rows * 4, fb);
          issued = j + 1;
        }
        for (int j = max(0, issued - Cfg::C_NST); j < issued; ++j)
          mbar_wait(full + 8 * (j % Cfg::C_NST), (j / Cfg::C_NST) & 1, p.err, 1000000000ull);
      }
    } else if (active && warp == NC + 1) {
      // ---------------------------------------------------------------- publisher
      if (lane == 0) {
        int done = 0;
        for (int j = 0; j < nst; ++j) {
          const int b = j & 1;
          if (!mbar_wait(eready + 8 * b, (j >> 1) & 1, p.err, p.wait_ns)) break;
          // the output CTA has set up its pipeline stage for this stage of this stream
          if (!mbar_wait(c_grant + 8 * (j % NGRANT), (j / NGRANT) & 1, p.err, p.wait_ns)) break;
          const int it = j * nmine + rank;
          const uint32_t dst = sbase + (it % Cfg::O_NST) * Cfg::O_STAGE + 2 * XTILE;
          const uint32_t dbar = map_rank(o_full + 8 * (it % Cfg::O_NST), out_rank);
          const uint32_t sE = sbase + Cfg::C_E_OFF + 2 * Cfg::C_ESUB * b;
          const uint32_t sW = sbase + Cfg::C_W_OFF + Cfg::C_ESUB * b;
          dsmem_copy(map_rank(dst, out_rank), sE, PART, dbar);
          dsmem_copy(map_rank(dst + PART, out_rank), sE + PART, PART, dbar);
          dsmem_copy(map_rank(dst + 2 * PART, out_rank), sW, PART, dbar);
          done = j + 1;
        }
        // the last copies have been read out of this CTA's shared memory before it may exit
        for (int j = max(0, done - 2); j < done; ++j)
          mbar_wait(efree + 8 * (j & 1), (j >> 1) & 1, p.err, 1000000000ull);
      }
    } else if (active && warp < NC) {
      // ---------------------------------------------------------------- chain warps
      const int g = lane >> 2, tq = lane & 3;
      const int mi = lane >> 3, rr = lane & 7;
      const int colw = 16 * warp;
      const int colg = col_cta + colw;
      auto off = [&](int row, int col) -> uint32_t { return xswz<128>(row, 2 * col); };
      uint32_t o_brow[XKS], o_btrn[XKS];
#pragma unroll
      for (int ks = 0; ks < XKS; ++ks) {
        o_brow[ks] = off(8 * (mi >> 1) + rr, 16 * ks + 8 * (mi & 1));
        o_btrn[ks] = off(8 * (mi & 1) + rr, 16 * ks + 8 * (mi >> 1));
      }
      const uint32_t o_vt = off(8 * (mi >> 1) + rr, colg + 8 * (mi & 1));
      // stmatrix targets: row colw + 8 (mi & 1) + rr of this CTA's [COLS][64] tiles
      const int srow = colw + 8 * (mi & 1) + rr;
      const int scol = 8 * (mi >> 1);
      constexpr uint32_t CHUNK_BYTES = 16 * 128;
      float wc[XD / 8][4];   // W^T[colg .. colg+15, :]; tile jt holds rows 8jt .. 8jt+7 of W
      {
        const float* w0 = p.W0 ? p.W0 + (size_t)stream * XD * XD : nullptr;
#pragma unroll
        for (int jt = 0; jt < XD / 8; ++jt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int row = 8 * jt + 2 * tq + e;
            wc[jt][e] = w0 ? w0[row * XD + colg + g] : 0.f;
            wc[jt][2 + e] = w0 ? w0[row * XD + colg + g + 8] : 0.f;
          }
      }
      struct Ops {
        uint32_t kb[XKS][4], kt[XKS][4], vt[4];
        float e0, e1, e8, e9;
      };
      bool ok = true;
      for (int j = 0; j < nst; ++j) {
        const int s = j % Cfg::C_NST, b = j & 1;
        bool got = mbar_wait_warp(full + 8 * s, (j / Cfg::C_NST) & 1, p.err, p.wait_ns);
        // the -E and W_s buffers b were last copied out for stage j - 2
        if (got && j >= 2)
          got = mbar_wait_warp(efree + 8 * b, ((j >> 1) - 1) & 1, p.err, p.wait_ns);
        if (!got) {
          ok = false;
          break;
        }
        const uint32_t sK = sbase + s * Cfg::C_STAGE;
        const uint32_t sV = sK + XTILE;
        const uint32_t sEta = sV + XTILE;
        const uint32_t sE = sbase + Cfg::C_E_OFF + 2 * Cfg::C_ESUB * b;
        const uint32_t sW = sbase + Cfg::C_W_OFF + Cfg::C_ESUB * b;
        const int chunks = min(XR, T - j * XR) / XC;
#pragma unroll
        for (int ks = 0; ks < XKS; ++ks)
          stsm_x4(sW + xswz<128>(srow, 2 * (16 * ks + scol)),
                  pack_bf16(wc[2 * ks][0], wc[2 * ks][1]),
                  pack_bf16(wc[2 * ks][2], wc[2 * ks][3]),
                  pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]),
                  pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]));
        auto load = [&](Ops& o, const int c) {
          const uint32_t cb = c * CHUNK_BYTES;
#pragma unroll
          for (int ks = 0; ks < XKS; ++ks) {
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
          uint32_t wa[XKS][4];
#pragma unroll
          for (int ks = 0; ks < XKS; ++ks) {
            wa[ks][0] = pack_bf16(wc[2 * ks][0], wc[2 * ks][1]);
            wa[ks][1] = pack_bf16(wc[2 * ks][2], wc[2 * ks][3]);
            wa[ks][2] = pack_bf16(wc[2 * ks + 1][0], wc[2 * ks + 1][1]);
            wa[ks][3] = pack_bf16(wc[2 * ks + 1][2], wc[2 * ks + 1][3]);
          }
          float pa[2][4] = {}, pb[2][4] = {};
#pragma unroll
          for (int ks = 0; ks < XKS; ++ks) {
            float (&acc)[2][4] = (ks & 1) ? pb : pa;
            mma16816(acc[0], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], o.kb[ks][0],
                     o.kb[ks][1]);
            mma16816(acc[1], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], o.kb[ks][2],
                     o.kb[ks][3]);
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
          const uint32_t n0 = pack_bf16(E[0][0], E[0][1]) ^ 0x80008000u;
          const uint32_t n1 = pack_bf16(E[0][2], E[0][3]) ^ 0x80008000u;
          const uint32_t n2 = pack_bf16(E[1][0], E[1][1]) ^ 0x80008000u;
          const uint32_t n3 = pack_bf16(E[1][2], E[1][3]) ^ 0x80008000u;
#pragma unroll
          for (int jp = 0; jp < XKS; ++jp) {
            mma16816(wc[2 * jp], n0, n1, n2, n3, o.kt[jp][0], o.kt[jp][1]);
            mma16816(wc[2 * jp + 1], n0, n1, n2, n3, o.kt[jp][2], o.kt[jp][3]);
          }
          stsm_x4(sE + (c >> 2) * Cfg::C_ESUB + xswz<128>(srow, 2 * (16 * (c & 3) + scol)), n0,
                  n1, n2, n3);
        };
        if (chunks == XCPS) {
          Ops ops[2];
          load(ops[0], 0);
#pragma unroll
          for (int c = 0; c < XCPS; ++c) {
            if (c + 1 < XCPS) load(ops[(c + 1) & 1], c + 1);
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
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(eready + 8 * b);
          mbar_arrive(empty + 8 * s);
        }
      }
      if (ok) {
        float* wo = p.Wout + (size_t)stream * XD * XD;
#pragma unroll
        for (int jt = 0; jt < XD / 8; ++jt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int row = 8 * jt + 2 * tq + e;
            wo[row * XD + colg + g] = wc[jt][e];
            wo[row * XD + colg + g + 8] = wc[jt][2 + e];
          }
      }
    }
    umma::fence_before();
    __syncthreads();
  } else {
    // ================================================================ output CTA
    const uint32_t full = o_full, empty = o_empty, sfull = o_sfull, pfull = o_pfull;
    const uint32_t ofull = o_ofull, ofree = o_ofree, mdone = o_mdone;
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Cfg::BAR_OFF + 232);
    // items walk stages in order, the cluster's streams inside
    const int nitems = nst * nmine;
    auto item_rank = [&](int it) { return it % nmine; };
    auto item_stream = [&](int it) { return cid * p.ks + it % nmine; };
    auto item_stage = [&](int it) { return it / nmine; };
    if (warp == 0) {
      // ------------------------------------------------------------------ producer
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        int issued = 0;
        for (int it = 0; it < nitems; ++it) {
          const int s = it % Cfg::O_NST;
          const int stream = item_stream(it), j = item_stage(it);
          if (it >= Cfg::O_NST &&
              !mbar_wait(empty + 8 * s, ((it / Cfg::O_NST) - 1) & 1, p.err, p.wait_ns))
            break;
          const uint32_t fb = full + 8 * s;
          const uint32_t st = sbase + s * Cfg::O_STAGE;
          // Q, K of the stage and the chain CTA's copy of -E and W_s all land on this barrier
          mbar_arrive_expect_tx(fb, 2 * XTILE + SLOT);
          tma_load_3d(st, &tmQ, fb, 0, j * XR, stream);
          tma_load_3d(st + XTILE, &tmK, fb, 0, j * XR, stream);
          remote_arrive(map_rank(c_grant + 8 * (j % NGRANT), item_rank(it)));
          issued = it + 1;
        }
        for (int it = max(0, issued - Cfg::O_NST); it < issued; ++it)
          mbar_wait(full + 8 * (it % Cfg::O_NST), (it / Cfg::O_NST) & 1, p.err, 1000000000ull);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ tcgen05 issue warp
      const uint32_t id_s = umma::idesc_bf16(128, 128, false, false);   // Q K^T
      const uint32_t id_o = umma::idesc_bf16(128, 64, false, false);    // Q W_s and P (-E)
      auto issue_s = [&](int it) -> bool {
        const int s = it % Cfg::O_NST, b = it & 1;
        if (!mbar_wait_warp(full + 8 * s, (it / Cfg::O_NST) & 1, p.err, p.wait_ns)) return false;
        umma::fence_after();
        // the copy has landed: the chain CTA's buffer of this stage is free again
        if (lane == 0)
          remote_arrive(map_rank(c_efree + 8 * (item_stage(it) & 1), item_rank(it)));
        const uint32_t sQ = sbase + s * Cfg::O_STAGE, sK = sQ + XTILE;
#pragma unroll
        for (int ks = 0; ks < XKS; ++ks)
          umma::mma_ss_elect(tmem + XTM_S + 128 * b, umma::desc_kmajor(sQ + 32 * ks),
                             umma::desc_kmajor(sK + 32 * ks), id_s, ks > 0);
        umma::commit_elect(sfull + 8 * b);
        return true;
      };
      bool ok = nitems > 0 ? issue_s(0) : true;
      for (int it = 0; ok && it < nitems; ++it) {
        const int s = it % Cfg::O_NST, b = it & 1;
        const uint32_t sQ = sbase + s * Cfg::O_STAGE;
        const uint32_t sE = sQ + 2 * XTILE, sW = sE + 2 * PART;
        const uint32_t dO = tmem + XTM_O + 64 * b;
        if (it >= 2 && !mbar_wait_warp(ofree + 8 * b, ((it >> 1) - 1) & 1, p.err, p.wait_ns))
          break;
        umma::fence_after();
#pragma unroll
        for (int ks = 0; ks < XKS; ++ks)
          umma::mma_ss_elect(dO, umma::desc_kmajor(sQ + 32 * ks),
                             umma::desc_kmajor(sW + 32 * ks), id_o, ks > 0);
        if (!mbar_wait_warp(pfull + 8 * b, (it >> 1) & 1, p.err, p.wait_ns)) break;
        umma::fence_after();
#pragma unroll
        for (int ks = 0; ks < XR / 16; ++ks)
          umma::mma_ts_elect(dO, tmem + XTM_P + 64 * b + 8 * ks,
                             umma::desc_kmajor(sE + (ks >> 2) * PART + 32 * (ks & 3)), id_o,
                             true);
        umma::commit_elect(ofull + 8 * b);
        umma::commit_elect(empty + 8 * s);
        if (it + 1 < nitems) ok = issue_s(it + 1);
      }
      umma::commit_elect(mdone);
      mbar_wait_warp(mdone, 0, p.err, 1000000000ull);
    } else if (warp < 6) {
      // ------------------------------------------------------------------ epilogue warps 2..5
      const int q = warp & 3;
      const int t = 32 * q + lane;
      const uint32_t tl = (uint32_t)(32 * q) << 16;
      const int etid = threadIdx.x - 64;
      const uint32_t sO = sbase + Cfg::O_OT_OFF;
      auto mask = [&](int it) -> bool {
        const int b = it & 1;
        if (!mbar_wait_warp(sfull + 8 * b, (it >> 1) & 1, p.err, p.wait_ns)) return false;
        umma::fence_after();
  #pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
          uint32_t v[32] = {}, v2[32] = {}, w[32];
          if (2 * pp <= q) {
            umma::ld32x32(tmem + tl + XTM_S + 128 * b + 64 * pp, v);
            umma::wait_ld();
            umma::reg_fence(v);
          }
          if (2 * pp + 1 <= q) {
            umma::ld32x32(tmem + tl + XTM_S + 128 * b + 64 * pp + 32, v2);
            umma::wait_ld();
            umma::reg_fence(v2);
          }
  #pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int s0 = 64 * pp + 2 * i, s1 = s0 + 1;
            const uint32_t x0 = i < 16 ? v[2 * i] : v2[2 * i - 32];
            const uint32_t x1 = i < 16 ? v[2 * i + 1] : v2[2 * i - 31];
            w[i] = pack_bf16(s0 <= t ? __uint_as_float(x0) : 0.f,
                             s1 <= t ? __uint_as_float(x1) : 0.f);
          }
          umma::st32x32(tmem + tl + XTM_P + 64 * b + 32 * pp, w);
        }
        umma::wait_st();
        umma::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull + 8 * b);
        return true;
      };
      auto drain = [&](int it) -> bool {
        const int b = it & 1;
        const bool got = mbar_wait_warp(ofull + 8 * b, (it >> 1) & 1, p.err, p.wait_ns);
        if (got && etid == 0) bulk_wait_read<0>();
        if (xbar_or(1, 128, !got)) return false;
        umma::fence_after();
        uint32_t v[64];
  #pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
          umma::ld32x32(tmem + tl + XTM_O + 64 * b + 32 * h, r);
          umma::wait_ld();
          umma::reg_fence(r);
  #pragma unroll
          for (int i = 0; i < 32; ++i) v[32 * h + i] = r[i];
        }
        umma::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ofree + 8 * b);
  #pragma unroll
        for (int k = 0; k < 8; ++k)
          sts128(sO + xswz<128>(t, 16 * k),
                 make_uint4(pack_bf16(__uint_as_float(v[8 * k]), __uint_as_float(v[8 * k + 1])),
                            pack_bf16(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3])),
                            pack_bf16(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5])),
                            pack_bf16(__uint_as_float(v[8 * k + 6]),
                                      __uint_as_float(v[8 * k + 7]))));
        fence_proxy_async_smem();
        xbar_sync(1, 128);
        if (etid == 0) {
          tma_store_3d(&tmO, sO, 0, item_stage(it) * XR, item_stream(it));
          bulk_commit();
        }
        return true;
      };
      for (int it = 0; it < nitems; ++it) {
        const bool ok = mask(it);
        if (xbar_or(1, 128, !ok)) break;
        if (it >= 1 && !drain(it - 1)) break;
        if (it + 1 == nitems) drain(it);
      }
      if (etid == 0) bulk_wait<0>();
    }
    umma::fence_before();
    __syncthreads();
    if (warp == 1) umma::tmem_dealloc(tmem, 512);
  }
  // no CTA leaves while another of the cluster may still reach its shared memory
  cluster_sync_all();
}

}  // namespace

// Streams per cluster (1 or 2; the cluster adds one output CTA) for the split form, or 0 if the
// streams leave too few SMs: every cluster must be resident at once, one CTA per SM.
int dual_xsm_plan(int streams, int sms, int* n_clusters) {
  const int forced = tuning(kTuneDualClusterStreams);
  for (int ks : {1, 2}) {
    if (forced && ks != forced) continue;
    const int clusters = (streams + ks - 1) / ks;
    if (clusters * (ks + 1) <= sms) {
      *n_clusters = clusters;
      return ks;
    }
  }
  return 0;
}

int launch_dual_xsm(const StateArgs& a, int ks, int n_clusters, const LaunchCtx& ctx) {
  using Cfg = XCfg<4>;
  const int BH = a.B * a.H;
  CUtensorMap tq, tk, tv, to;
  const uint64_t dims[3] = {(uint64_t)XD, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)XD * 2, (uint64_t)a.T * XD * 2};
  const uint32_t box[3] = {(uint32_t)XD, (uint32_t)XR, 1};
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tmap_3d(&tq, a.Q, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tk, a.K, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tv, a.V, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&to, a.O, bf, dims, strides, box, sw, ctx.msg))
    return kCuda;
  auto kern = dual_xsm_kernel<4>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_clusters * (ks + 1));
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = ctx.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks + 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // one wave: clusters that could not all be resident would still be correct (they never wait
  // on each other) but slower; the caller falls back to the single-SM form then
  int max_clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
  if (e != cudaSuccess || max_clusters < n_clusters) {
    cudaGetLastError();
    return kUnsupported;
  }
  const int limit = tuning(kTuneWaitLimitNs);
  XParams p{a.eta, a.eta_scalar, a.S0, a.S_out, a.T, BH, ks, ctx.err,
            limit > 0 ? (uint64_t)limit : 4000000000ull};
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, p);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual_xsm launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace ttt
