// TTT-Linear mini-batch dual form, bf16 inputs, d = 64, chunk C = 16, with the serial chain and
// the output products on separate SMs.
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
// the chain measured about 1.5x slower than alone (the output work competes with it for the
// tensor pipe and the issue slots even when nothing waits on it). Here one launch holds
//   * chain CTAs, one per (stream, column group): NC chain warps (16 columns of W each, the state
//     in registers), a TMA producer warp (K, V, rates) and a publisher warp that copies every
//     stage's -E^T and bf16(W_s)^T from shared memory to a ring of slots in the workspace and
//     releases a per-stream counter;
//   * output CTAs, each serving a fixed set of streams stage by stage: a producer warp waits for
//     the counters of the stream (acquire), loads Q and K by TMA and the slot by a bulk copy into
//     one pipeline stage, and releases the slot; an MMA warp issues S = Q K^T, O = Q W_s and
//     O += P (-E) on tcgen05; four epilogue warps mask S into P (TMEM -> TMEM) and store O.
// The launch is cooperative, so every CTA is resident and the counters always make progress:
// a chain CTA only waits for a slot its own output CTA releases after loading it, and an output
// CTA walks stages in order, so no wait can close a cycle. Every wait is bounded.
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
constexpr int RING = 4;             // published stages kept per stream
constexpr int PART = 64 * 128;      // one [64][64] bf16 sub-tile (8 KB)
constexpr int SLOT = 3 * PART;      // -E^T tokens 0-63, tokens 64-127, bf16 W_s^T
constexpr uint32_t XTM_S = 0, XTM_P = 256, XTM_O = 384;

template <int NC>
struct XCfg {
  static constexpr int COLS = 16 * NC;             // output columns per chain CTA
  static constexpr int NG = XD / COLS;             // chain CTAs per stream
  // chain CTA
  static constexpr int C_NST = 3;
  static constexpr int C_STAGE = 2 * XTILE + 1024;  // K, V, rates (512 B, padded)
  static constexpr int C_ESUB = COLS * 128;         // this CTA's rows of one -E^T sub-tile
  static constexpr int C_E_OFF = C_NST * C_STAGE;   // 2 buffers x 2 sub-tiles
  static constexpr int C_W_OFF = C_E_OFF + 4 * C_ESUB;
  static constexpr int C_END = C_W_OFF + 2 * C_ESUB;
  // output CTA
  static constexpr int O_NST = 3;
  static constexpr int O_STAGE = 2 * XTILE + SLOT;  // Q, K, then the slot image
  static constexpr int O_OT_OFF = O_NST * O_STAGE;
  static constexpr int O_END = O_OT_OFF + XTILE;
  static constexpr int BAR_OFF = C_END > O_END ? C_END : O_END;
  static constexpr int SMEM = 1024 + BAR_OFF + 256;
  static constexpr int WARPS = NC + 2 > 6 ? NC + 2 : 6;
  static constexpr int THREADS = 32 * WARPS;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(C_ESUB % 1024 == 0 && C_STAGE % 1024 == 0 && O_STAGE % 1024 == 0, "alignment");
};

struct XParams {
  const float* eta;
  float eta_scalar;
  const float* W0;
  float* Wout;
  int T, BH;
  int n_chain, n_out;
  uint8_t* ring;        // [BH][RING][SLOT]
  int* ready;           // [BH * NG]: stages published by each chain CTA
  int* consumed;        // [BH]: stages whose slot the output CTA has loaded
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
__device__ __forceinline__ int ld_acquire(const int* ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* ptr, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(src), "r"(bytes)
               : "memory");
}
// Bounded wait for a global counter to reach `target` (acquire); false after the limit.
__device__ __forceinline__ bool wait_counter(const int* ptr, int target, unsigned* err,
                                             uint64_t limit_ns) {
  if (ld_acquire(ptr) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  while (ld_acquire(ptr) < target) {
    if (global_timer_ns() - t0 > limit_ns) {
      raise_device_error(err, kErrWaitTimeout);
      return false;
    }
    __nanosleep(64);
  }
  return true;
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

  if ((int)blockIdx.x < p.n_chain) {
    // ================================================================ chain CTA
    const uint32_t full = bar, empty = bar + 24;      // stage ring (3)
    const uint32_t eready = bar + 48;                 // -E and W_s of a stage stored (x2)
    const uint32_t efree = bar + 64;                  // the stage's copy to the slot done (x2)
    const int stream = blockIdx.x / Cfg::NG, cg = blockIdx.x % Cfg::NG;
    const int col_cta = cg * Cfg::COLS;
    if (threadIdx.x == 0) {
      for (int s = 0; s < Cfg::C_NST; ++s) {
        mbar_init(full + 8 * s, 1);
        mbar_init(empty + 8 * s, NC);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(eready + 8 * b, NC);
        mbar_init(efree + 8 * b, 1);
      }
      fence_mbar_init();
    }
    // -E buffers start at zero: a partial last stage leaves the absent chunks' columns as they
    // are, and the masked product multiplies them by zero scores (they must be finite)
    for (int i = threadIdx.x; i < 4 * Cfg::C_ESUB / 16; i += Cfg::THREADS)
      sts128(sbase + Cfg::C_E_OFF + 16 * i, make_uint4(0u, 0u, 0u, 0u));
    fence_proxy_async_smem();
    __syncthreads();

    if (warp == NC) {
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
    } else if (warp == NC + 1) {
      // ---------------------------------------------------------------- publisher
      if (lane == 0) {
        uint8_t* ring = p.ring + (size_t)stream * RING * SLOT;
        for (int j = 0; j < nst; ++j) {
          const int b = j & 1;
          if (!mbar_wait(eready + 8 * b, (j >> 1) & 1, p.err, p.wait_ns)) break;
          // the slot is free once the output CTA has loaded stage j - RING from it
          if (j >= RING && !wait_counter(p.consumed + stream, j - RING + 1, p.err, p.wait_ns))
            break;
          uint8_t* slot = ring + (size_t)(j % RING) * SLOT + (size_t)cg * Cfg::C_ESUB;
          const uint32_t sE = sbase + Cfg::C_E_OFF + 2 * Cfg::C_ESUB * b;
          const uint32_t sW = sbase + Cfg::C_W_OFF + Cfg::C_ESUB * b;
          bulk_store(slot, sE, Cfg::C_ESUB);
          bulk_store(slot + PART, sE + Cfg::C_ESUB, Cfg::C_ESUB);
          bulk_store(slot + 2 * PART, sW, Cfg::C_ESUB);
          bulk_commit();
          bulk_wait<0>();          // written (and read out of shared memory)
          fence_async_global();
          st_release(p.ready + blockIdx.x, j + 1);
          mbar_arrive(efree + 8 * b);
        }
        bulk_wait<0>();
      }
    } else if (warp < NC) {
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
    __syncthreads();
    return;
  }
  // ================================================================== output CTA
  const uint32_t full = bar, empty = bar + 24;      // stage ring (3)
  const uint32_t sfull = bar + 48;    // S accumulator written (x2, MMA commit)
  const uint32_t pfull = bar + 64;    // P written (x2, 4 epilogue warps)
  const uint32_t ofull = bar + 80;    // O accumulator complete (x2, MMA commit)
  const uint32_t ofree = bar + 96;    // O accumulator read out (x2, 4 epilogue warps)
  const uint32_t mdone = bar + 112;   // every MMA issued has completed
  const uint32_t tslot = bar + 128;
  const int oid = blockIdx.x - p.n_chain;
  // this CTA's streams: oid, oid + n_out, ...; items walk stages in order, streams inside
  const int nmine = oid < p.BH ? (p.BH - oid + p.n_out - 1) / p.n_out : 0;
  const int nitems = nst * nmine;
  auto item_stream = [&](int it) { return oid + (it % nmine) * p.n_out; };
  auto item_stage = [&](int it) { return it / nmine; };
  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::O_NST; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sfull + 8 * b, 1);
      mbar_init(pfull + 8 * b, 4);
      mbar_init(ofull + 8 * b, 1);
      mbar_init(ofree + 8 * b, 4);
    }
    mbar_init(mdone, 1);
    fence_mbar_init();
  }
  if (warp == 1) umma::tmem_alloc(tslot, 512);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Cfg::BAR_OFF + 128);

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
        // every chain CTA of the stream has published stage j (acquire), then the slot is read
        // through the async proxy
        bool got = true;
        for (int cg = 0; cg < Cfg::NG && got; ++cg)
          got = wait_counter(p.ready + stream * Cfg::NG + cg, j + 1, p.err, p.wait_ns);
        if (!got) break;
        fence_async_global();
        const uint32_t fb = full + 8 * s;
        const uint32_t st = sbase + s * Cfg::O_STAGE;
        mbar_arrive_expect_tx(fb, 2 * XTILE + SLOT);
        tma_load_3d(st, &tmQ, fb, 0, j * XR, stream);
        tma_load_3d(st + XTILE, &tmK, fb, 0, j * XR, stream);
        bulk_load(st + 2 * XTILE, p.ring + ((size_t)stream * RING + j % RING) * SLOT, SLOT, fb);
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
      // the slot's contents are in shared memory: the chain CTAs may reuse it
      if (lane == 0) st_release(p.consumed + item_stream(it), item_stage(it) + 1);
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
        umma::mma_ss_elect(dO, umma::desc_kmajor(sQ + 32 * ks), umma::desc_kmajor(sW + 32 * ks),
                           id_o, ks > 0);
      if (!mbar_wait_warp(pfull + 8 * b, (it >> 1) & 1, p.err, p.wait_ns)) break;
      umma::fence_after();
#pragma unroll
      for (int ks = 0; ks < XR / 16; ++ks)
        umma::mma_ts_elect(dO, tmem + XTM_P + 64 * b + 8 * ks,
                           umma::desc_kmajor(sE + (ks >> 2) * PART + 32 * (ks & 3)), id_o, true);
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

}  // namespace

// Chain CTAs per stream (1, 2 or 4) and output CTAs for the split form, or 0 if the streams
// leave too few SMs: every CTA must be resident (one per SM) and an output CTA serves at most
// two streams.
int dual_xsm_plan(int streams, int sms, int* n_out) {
  for (int ng : {4, 2, 1}) {
    const int chain = streams * ng;
    const int avail = sms - chain;
    if (avail >= (streams + 1) / 2 && avail >= 1) {
      *n_out = std::min(avail, streams);
      return ng;
    }
  }
  return 0;
}

size_t dual_xsm_workspace_bytes(int B, int H) {
  const size_t bh = (size_t)B * H;
  return bh * RING * SLOT + 256 * ((bh * 5 * sizeof(int) + 255) / 256);
}

int launch_dual_xsm(const StateArgs& a, int ng, int n_out, const LaunchCtx& ctx) {
  const int BH = a.B * a.H;
  const size_t ring_bytes = (size_t)BH * RING * SLOT;
  if (!a.ws || a.ws_bytes < dual_xsm_workspace_bytes(a.B, a.H)) return kWorkspace;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  int* ready = reinterpret_cast<int*>(ws + ring_bytes);      // [BH * 4] (NG <= 4)
  int* consumed = ready + (size_t)BH * 4;                    // [BH]
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
  cudaError_t e = cudaMemsetAsync(ready, 0, sizeof(int) * (size_t)BH * 5, ctx.stream);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual_xsm setup: ") + cudaGetErrorString(e);
    return kCuda;
  }
  const int limit = tuning(kTuneWaitLimitNs);
  XParams p{a.eta, a.eta_scalar, a.S0, a.S_out, a.T, BH, BH * ng, n_out, ws, ready, consumed,
            ctx.err, limit > 0 ? (uint64_t)limit : 4000000000ull};
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, XParams) = nullptr;
  int threads = 0, smem = 0;
  switch (ng) {
    case 1: kern = dual_xsm_kernel<4>; threads = XCfg<4>::THREADS; smem = XCfg<4>::SMEM; break;
    case 2: kern = dual_xsm_kernel<2>; threads = XCfg<2>::THREADS; smem = XCfg<2>::SMEM; break;
    case 4: kern = dual_xsm_kernel<1>; threads = XCfg<1>::THREADS; smem = XCfg<1>::SMEM; break;
    default:
      *ctx.msg = "dual_xsm: chain CTAs per stream must be 1, 2 or 4";
      return kUnsupported;
  }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  // cooperative: every CTA resident at once (the chain and output CTAs wait on each other)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(BH * ng + n_out);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = ctx.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, p);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("dual_xsm launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace ttt
