// TTT-Linear mini-batch dual form, bf16 inputs, chunk C = 16: tensor-core path.
//
// Computes, per (batch, head) stream and chunk c (source: "Learning to (Learn at Test Time)"
// reading, section on mini-batch TTT and the dual form; per-token rule section for reading the
// updated model):
//     G   = K_c W - V_c
//     O_c = Q_c W - tril(Q_c K_c^T) diag(eta_c) G
//     W   = W - K_c^T diag(eta_c) G
//
// Design. The chunk loop is a serial chain through W, and C = 16 tokens give a chunk too little
// work to hide latency, so the kernel is built around the chain's latency:
//   * the state stays in registers for the whole sequence as fp32 MMA accumulators. Columns of W
//     are independent (W's update mixes rows only), so each compute warp owns 16 output columns
//     and keeps W^T[cols, :] (16 x d fp32) in the accumulator layout of m16n8k16;
//   * the accumulator layout of W^T is, packed to bf16, exactly the A-operand layout of the next
//     chunk's products, so no shuffle or shared-memory round trip sits on the chain:
//         P^T = W^T K_c^T          (A = W^T, from registers; B = K_c rows via ldmatrix)
//         E^T = (P^T - V_c^T) diag(eta)
//         W^T -= E^T K_c           (A = E^T, from registers; B = K_c via ldmatrix.trans)
//   * the outputs (Q_c W and the causal correction tril(Q_c K_c^T) diag(eta) G) hang off the
//     chain and overlap with it;
//   * Q/K/V tiles arrive by TMA (3-D tensor maps over [B*H, T, d], 128-byte swizzle) into a
//     multi-stage mbarrier ring filled by one producer warp; outputs leave through a
//     double-buffered shared tile and TMA stores.
// Precision: W is fp32 throughout; its operand copy, the residual and the scores are rounded to
// bf16 once per chunk for the tensor cores (relative error ~2^-9 per product, fp32 accumulate).
#include <algorithm>
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace ttt {
namespace {

template <int D, int NW>
struct DualCfg {
  static constexpr int C = 16;
  static constexpr int CPS = 4;                    // chunks per pipeline stage
  static constexpr int R = C * CPS;                // token rows per stage
  static constexpr int SUB = D >= 64 ? 64 : D;     // columns per swizzled sub-tile
  static constexpr int RB = SUB * 2;               // bytes per sub-tile row
  static constexpr int NSUB = D / SUB;
  static constexpr int SUB_BYTES = R * RB;
  static constexpr int TILE_BYTES = NSUB * SUB_BYTES;
  static constexpr int COLS = 16 * NW;             // output columns per CTA
  static constexpr int NG = D / COLS;              // CTAs per stream
  static constexpr int OSUB = COLS >= 64 ? 64 : COLS;
  static constexpr int ORB = OSUB * 2;
  static constexpr int NOSUB = COLS / OSUB;
  static constexpr int OSUB_BYTES = R * ORB;
  static constexpr int OTILE_BYTES = NOSUB * OSUB_BYTES;
  static constexpr int ETA_BYTES = 1024;           // R floats, padded to keep tiles aligned
  static constexpr int STAGE_BYTES = 3 * TILE_BYTES + ETA_BYTES;
  static constexpr int BUDGET = 200 * 1024;
  static constexpr int NSTAGE_FIT = (BUDGET - 2 * OTILE_BYTES) / STAGE_BYTES;
  static constexpr int NSTAGE = NSTAGE_FIT > 8 ? 8 : NSTAGE_FIT;
  static constexpr int BAR_OFF = NSTAGE * STAGE_BYTES + 2 * OTILE_BYTES;
  static constexpr int SMEM = 1024 + BAR_OFF + 16 * NSTAGE;
  static constexpr int THREADS = 32 * (NW + 1);
  static constexpr int KS = D / 16;                // 16-wide k-steps over d
  static_assert(NSTAGE >= 2, "pipeline depth");
  static_assert(R * 4 <= ETA_BYTES, "eta slot");
  static_assert(D % COLS == 0, "column split");
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

template <int D, int NW>
__global__ void __launch_bounds__(DualCfg<D, NW>::THREADS, 1)
    dual_mma_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmO, const DualParams p) {
  using Cfg = DualCfg<D, NW>;
  constexpr int R = Cfg::R, KS = Cfg::KS, NSTAGE = Cfg::NSTAGE;
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
        mbar_arrive_expect_tx(fb, bytes);
        const uint32_t st = sbase + s * Cfg::STAGE_BYTES;
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
  const int colw = 16 * warp;                // column offset inside the CTA's columns
  const int colg = col_cta + colw;           // global column of this warp's first column

  // Per-stream state: W^T[colg .. colg+15][0 .. D-1] as m16n8 fp32 accumulators.
  float wacc[D / 8][4];
  {
    const float* w0 = p.W0 ? p.W0 + (size_t)stream * D * D : nullptr;
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = 8 * j + 2 * tq + e;
        wacc[j][e] = w0 ? w0[row * D + colg + g] : 0.f;
        wacc[j][2 + e] = w0 ? w0[row * D + colg + g + 8] : 0.f;
      }
  }

  auto tile = [&](uint32_t base, int row, int col) -> uint32_t {
    return base + (col / Cfg::SUB) * Cfg::SUB_BYTES +
           swz<Cfg::RB>(row * Cfg::RB + (col % Cfg::SUB) * 2);
  };
  auto otile = [&](uint32_t base, int row, int col) -> uint32_t {
    return base + (col / Cfg::OSUB) * Cfg::OSUB_BYTES +
           swz<Cfg::ORB>(row * Cfg::ORB + (col % Cfg::OSUB) * 2);
  };

  bool ok = true;
  for (int j = 0; j < nstg; ++j) {
    const int s = j % NSTAGE;
    const bool got = mbar_wait(full_bar + 8 * s, (j / NSTAGE) & 1, p.err);
    const uint32_t sQ = sbase + s * Cfg::STAGE_BYTES;
    const uint32_t sK = sQ + Cfg::TILE_BYTES;
    const uint32_t sV = sK + Cfg::TILE_BYTES;
    const float* sEta = reinterpret_cast<const float*>(smem + s * Cfg::STAGE_BYTES +
                                                       3 * Cfg::TILE_BYTES);
    const uint32_t sO = sbase + NSTAGE * Cfg::STAGE_BYTES + (j & 1) * Cfg::OTILE_BYTES;
    const int chunks = got ? min(R, T - j * R) / 16 : 0;

#pragma unroll 1
    for (int c = 0; c < chunks; ++c) {
      const int r0 = 16 * c;
      // ---- W-independent operands of this chunk
      uint32_t kr[KS][4], qr[KS][4];
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int row = r0 + 8 * (mi >> 1) + rr, col = 16 * ks + 8 * (mi & 1);
        ldsm_x4(tile(sK, row, col), kr[ks]);
        ldsm_x4(tile(sQ, row, col), qr[ks]);
      }
      uint32_t vt[4];
      ldsm_x4_t(tile(sV, r0 + 8 * (mi >> 1) + rr, colg + 8 * (mi & 1)), vt);
      float e0, e1, e8, e9;  // eta of tokens 2tq, 2tq+1, 8+2tq, 9+2tq of the chunk
      if (p.eta) {
        const float2 a = *reinterpret_cast<const float2*>(sEta + r0 + 2 * tq);
        const float2 b = *reinterpret_cast<const float2*>(sEta + r0 + 8 + 2 * tq);
        e0 = a.x; e1 = a.y; e8 = b.x; e9 = b.y;
      } else {
        e0 = e1 = e8 = e9 = p.eta_scalar;
      }

      // ---- chain: W^T (bf16) -> P^T = W^T K^T -> E^T -> W^T -= E^T K
      uint32_t wa[KS][4];
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        wa[ks][0] = pack_bf16(wacc[2 * ks][0], wacc[2 * ks][1]);
        wa[ks][1] = pack_bf16(wacc[2 * ks][2], wacc[2 * ks][3]);
        wa[ks][2] = pack_bf16(wacc[2 * ks + 1][0], wacc[2 * ks + 1][1]);
        wa[ks][3] = pack_bf16(wacc[2 * ks + 1][2], wacc[2 * ks + 1][3]);
      }
      float pt[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        mma16816(pt[0], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], kr[ks][0], kr[ks][1]);
        mma16816(pt[1], wa[ks][0], wa[ks][1], wa[ks][2], wa[ks][3], kr[ks][2], kr[ks][3]);
      }
      uint32_t ea[4];
      ea[0] = pack_bf16((pt[0][0] - bf16_lo(vt[0])) * e0, (pt[0][1] - bf16_hi(vt[0])) * e1);
      ea[1] = pack_bf16((pt[0][2] - bf16_lo(vt[1])) * e0, (pt[0][3] - bf16_hi(vt[1])) * e1);
      ea[2] = pack_bf16((pt[1][0] - bf16_lo(vt[2])) * e8, (pt[1][1] - bf16_hi(vt[2])) * e9);
      ea[3] = pack_bf16((pt[1][2] - bf16_lo(vt[3])) * e8, (pt[1][3] - bf16_hi(vt[3])) * e9);
      const uint32_t na0 = ea[0] ^ 0x80008000u, na1 = ea[1] ^ 0x80008000u;
      const uint32_t na2 = ea[2] ^ 0x80008000u, na3 = ea[3] ^ 0x80008000u;
#pragma unroll
      for (int jp = 0; jp < KS; ++jp) {
        uint32_t kt[4];
        ldsm_x4_t(tile(sK, r0 + 8 * (mi & 1) + rr, 16 * jp + 8 * (mi >> 1)), kt);
        mma16816(wacc[2 * jp], na0, na1, na2, na3, kt[0], kt[1]);
        mma16816(wacc[2 * jp + 1], na0, na1, na2, na3, kt[2], kt[3]);
      }

      // ---- outputs: O = Q W (chunk-start W) - mask(Q K^T) diag(eta) G
      float lc[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        mma16816(lc[0], qr[ks][0], qr[ks][2], qr[ks][1], qr[ks][3], kr[ks][0], kr[ks][1]);
        mma16816(lc[1], qr[ks][0], qr[ks][2], qr[ks][1], qr[ks][3], kr[ks][2], kr[ks][3]);
      }
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (8 * jj + 2 * tq + (i & 1) > g + 8 * (i >> 1)) lc[jj][i] = 0.f;
      const uint32_t la0 = pack_bf16(-lc[0][0], -lc[0][1]), la1 = pack_bf16(-lc[0][2], -lc[0][3]);
      const uint32_t la2 = pack_bf16(-lc[1][0], -lc[1][1]), la3 = pack_bf16(-lc[1][2], -lc[1][3]);
      float o[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        mma16816(o[0], qr[ks][0], qr[ks][2], qr[ks][1], qr[ks][3], wa[ks][0], wa[ks][2]);
        mma16816(o[1], qr[ks][0], qr[ks][2], qr[ks][1], qr[ks][3], wa[ks][1], wa[ks][3]);
      }
      mma16816(o[0], la0, la1, la2, la3, ea[0], ea[2]);
      mma16816(o[1], la0, la1, la2, la3, ea[1], ea[3]);
      stsm_x4(otile(sO, r0 + 8 * (mi & 1) + rr, colw + 8 * (mi >> 1)),
              pack_bf16(o[0][0], o[0][1]), pack_bf16(o[0][2], o[0][3]),
              pack_bf16(o[1][0], o[1][1]), pack_bf16(o[1][2], o[1][3]));
    }

    // Inputs of this stage are consumed; hand the slot back to the producer.
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar + 8 * s);
    // Output tile -> global (TMA store, rows past T are clipped by the tensor map).
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

  // Final state W[:, colg..colg+15].
  float* wo = p.Wout + (size_t)stream * D * D;
#pragma unroll
  for (int j = 0; j < D / 8; ++j)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int row = 8 * j + 2 * tq + e;
      wo[row * D + colg + g] = wacc[j][e];
      wo[row * D + colg + g + 8] = wacc[j][2 + e];
    }
}

template <int D, int NW>
int launch_cfg(const StateArgs& a, const LaunchCtx& ctx) {
  using Cfg = DualCfg<D, NW>;
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
  auto kern = dual_mma_kernel<D, NW>;
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

// Column groups per stream: fewer streams than SMs leave SMs idle, and splitting the
// (independent) columns of W over two CTAs doubles the number of chains in flight.
int column_split(int streams, int d) {
  const char* env = getenv("TTT_DUAL_COLUMN_SPLIT");  // tuning override: 1, 2 or 4
  const int forced = env ? atoi(env) : 0;
  if (forced == 1 || forced == 2 || forced == 4) return std::min(forced, d / 16);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (d >= 64 && streams < sms) return 2;
  return 1;
}

}  // namespace

bool dual_mma_supported(int d, int C, int dt) {
  return dt == 1 && C == 16 && (d == 32 || d == 64 || d == 128);
}

int launch_dual_mma(const StateArgs& a, const LaunchCtx& ctx) {
  const int split = column_split(a.B * a.H, a.d);
  switch (a.d) {
    case 32:
      return launch_cfg<32, 2>(a, ctx);
    case 64:
      return split >= 2 ? launch_cfg<64, 2>(a, ctx) : launch_cfg<64, 4>(a, ctx);
    case 128:
      return split >= 2 ? launch_cfg<128, 4>(a, ctx) : launch_cfg<128, 8>(a, ctx);
  }
  *ctx.msg = "dual_mma: unsupported head dim";
  return kUnsupported;
}

}  // namespace ttt
