// Associative mode with a momentum inner loop, in one pass that carries both states.
//
// Source: "KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다", momentum paragraph: with
// momentum SGD the inner loop is still a weighted sum of linear-attention terms. Per stream,
//     M_t = beta M_(t-1) + u_t,   S_t = S_(t-1) + M_t,   o_t = q_t S_t,   u_t = eta_t k_t^T v_t.
// Over a chunk of C = 64 tokens (local indices i, j) that starts from (S, M), with
// w(n) = sum_{r=0..n} beta^r (so 1 <= w(n) <= n + 1):
//     o_i = q_i S + beta w(i) q_i M + sum_{j<=i} w(i-j) (q_i . k_j) eta_j v_j
//     S'  = S + beta w(63) M + sum_j w(63-j) u_j
//     M'  = beta^64 M + sum_j beta^(63-j) u_j
// Every weight is a sum of non-negative terms formed directly, so no step subtracts two large
// quantities: the evaluation keeps its accuracy for every beta in [0, 1]. (Splitting the
// recurrence into a plain and a decayed one, S = S0 + (A - beta M) / (1 - beta), needs no second
// state but loses accuracy as beta -> 1.)
//
// Products, transposed as in the plain associative kernel (M side = d_out on the TMEM lanes):
//     EVw = diag(eta_j w(63-j)) V (in place of V),   EVb = diag(eta_j beta^(63-j)) V,
//     P'[i][j] = [j <= i] w(i-j) / w(63-j) (q_i . k_j)    (so P' EVw carries w(i-j) eta_j v_j),
//     S^T += EVw^T K,  M^T += EVb^T K       (after the refresh: S += beta w(63) M, M *= beta^64),
//     O^T = Sb^T Q^T + EVw^T P'^T,  Om^T = Mb^T Q^T,  o_i = O[i] + beta w(i) Om[i],
// with Sb, Mb the bf16 copies of the chunk's starting states (A operands read from TMEM).
//
// TMEM (512 columns): S^T fp32 [0,128), M^T fp32 [128,256), bf16 S^T [256,320), bf16 M^T
// [320,384), O^T [384,448), Om^T [448,512). With every column in use, the bf16 copies and the
// output accumulators have one buffer each, and the scores Q K^T are formed on warp MMAs
// (mma.sync, registers) by the operand warps, which apply the causal weights as they go.
//
// Warp roles: 0 TMA producer (3-stage ring of Q/K/V/eta tiles); 1 TMEM owner and MMA issuer;
// 2-5 operands (EVw in place, EVb, scores -> P'); 6-13 state refresh (two per TMEM lane
// quarter, each on half of the d_in columns: bf16 copies of S and M, then S += beta w(63) M and
// M *= beta^64 in fp32); 14-17 outputs (O + beta w(i) Om -> bf16 -> shared tile -> TMA store).
// The serial chain per chunk is refresh -> update and output MMAs -> refresh.
//
// Superchunks: pass 1 (the state-only template) runs each piece of L tokens from zero and
// writes (dS, dM); the piece maps (S, M) to (S + c_L M + dS, beta^L M + dM) with
// c_L = sum_{r=1..L} beta^r, and mom_scan_kernel composes the maps in sequence order into every
// part's starting state; pass 2 runs each part from its start and writes O, and the last part
// writes S_out and M_out.
#include <algorithm>
#include <cmath>
#include <string>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int MD = 128;   // state tile (head dim 128; 64 runs zero-padded)
constexpr int MC = 64;    // tokens per chunk
constexpr int TILE = MC * MD * 2;   // one [64 tokens][128] bf16 tile (two [64][64] sub-tiles)

// Shared-memory map (bytes from the 1024-aligned base); pass 1 loads no Q and writes no O.
template <bool SO>
struct MomSmem {
  static constexpr int Q_BYTES = SO ? 0 : TILE;
  static constexpr int K_OFF = Q_BYTES;
  static constexpr int V_OFF = K_OFF + TILE;
  static constexpr int ETA_OFF = V_OFF + TILE;
  static constexpr int STAGE = ETA_OFF + 1024;          // rates (256 B) padded for alignment
  static constexpr int STAGES = SO ? 4 : 3;
  static constexpr int EVB_OFF = STAGES * STAGE;        // 2 x EVb [64 t][128 d]
  static constexpr int P_OFF = EVB_OFF + 2 * TILE;      // 2 x P' [64 t][64 s]
  static constexpr int O_OFF = P_OFF + (SO ? 0 : 2 * MC * MC * 2);   // O staging [64 t][128 d]
  static constexpr int BAR_OFF = O_OFF + (SO ? 0 : TILE);
  static constexpr int TAB_OFF = BAR_OFF + 256;         // five tables of 64 floats
  static constexpr int BYTES = 1024 + TAB_OFF + 5 * 256;
  // warps: 0 TMA, 1 MMA, 2 .. REF0-1 operands, REF0 .. OUT0-1 refresh, OUT0 .. OUT0+3 outputs
  static constexpr int NOP = SO ? 4 : 8;
  static constexpr int NREF = 4;               // refresh warps: one per TMEM lane quarter
  static constexpr int REF0 = 2 + NOP;
  static constexpr int OUT0 = REF0 + NREF;
  static constexpr int THREADS = 32 * (OUT0 + (SO ? 0 : 4));
  static constexpr uint32_t TM_COLS = SO ? 256 : 512;
  static_assert(STAGE % 1024 == 0 && EVB_OFF % 1024 == 0 && P_OFF % 1024 == 0 &&
                    O_OFF % 1024 == 0, "tile alignment");
  static_assert(BYTES <= 227 * 1024, "shared memory");
};

constexpr uint32_t TM_S = 0, TM_M = 128, TM_SB = 256, TM_MB = 320, TM_O = 384, TM_OM = 448;

struct MomParams {
  const float* eta;      // [BH, T] or null (eta_scalar)
  float eta_scalar;
  float beta;
  const float* S0;       // pass 2 with one part: the caller's [dim][dim] states, or null (zeros)
  const float* M0;
  const float* start;    // pass 2 with several parts: [BH, nslots, 2, D, D] starting states;
                         // part m starts from slot m * slot_mul
  float* inc;            // pass 1: piece k writes (dS, dM) into slot k + 1 of the same layout
  float* S_dst;          // pass 2: S_out, M_out [BH, dim, dim], written by the last part
  float* M_dst;
  int T, P, part_len;    // P: parts (pass 2) or pieces (pass 1) per stream in the grid
  int nslots, slot_mul;
  int dim;               // the caller's head dim, 128 or 64
  unsigned* err;
};

// beta w(63) and beta^64, the refresh coefficients of a chunk
__device__ __forceinline__ void chunk_coeffs(float beta, float& c63, float& b64) {
  double w = 0.0, pw = 1.0;
  for (int r = 0; r < MC; ++r) {
    w += pw;
    pw *= (double)beta;
  }
  c63 = (float)((double)beta * w);
  b64 = (float)pw;
}

template <bool SO>
__global__ void __launch_bounds__(MomSmem<SO>::THREADS, 1)
    mom_chunk_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmO, const MomParams p) {
  using L = MomSmem<SO>;
  constexpr int ST = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + L::BAR_OFF;
  const uint32_t full = bar, empty = bar + 32;       // stage ring (up to 4)
  const uint32_t opready = bar + 64;                 // EVw, EVb, P' of a chunk written (x2)
  const uint32_t sready = bar + 80;                  // refresh of the chunk's states done
  const uint32_t cdone = bar + 88;                   // every MMA of a chunk completed (x2)
  const uint32_t ofree = bar + 104;                  // output accumulators read out
  const uint32_t mdone = bar + 112;                  // every MMA issued has completed
  const uint32_t tslot = bar + 120;
  const uint32_t tab = sbase + L::TAB_OFF;
  // tables by token index: w(63-j), beta^(63-j), w(n), 1 / w(63-j), beta w(i)
  const uint32_t t_evw = tab, t_evb = tab + 256, t_w = tab + 512, t_rw = tab + 768,
                 t_cq = tab + 1024;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stream = blockIdx.x / p.P, part = blockIdx.x % p.P;
  const int tok0 = part * p.part_len;
  const int nch = p.part_len / MC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(opready + 8 * b, L::NOP);
      mbar_init(cdone + 8 * b, 1);
    }
    mbar_init(sready, L::NREF);
    mbar_init(ofree, 4);
    mbar_init(mdone, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < MC) {
    // sums of powers in double, one entry per thread
    const int n = threadIdx.x;
    const double be = (double)p.beta;
    double wn = 0.0, pw = 1.0;
    for (int r = 0; r <= n; ++r) {
      wn += pw;
      pw *= be;
    }
    double wm = 0.0, bm = 1.0;
    pw = 1.0;
    for (int r = 0; r <= MC - 1 - n; ++r) {
      wm += pw;
      pw *= be;
    }
    for (int r = 0; r < MC - 1 - n; ++r) bm *= be;
    float* t = reinterpret_cast<float*>(smem + L::TAB_OFF);
    t[n] = (float)wm;
    t[64 + n] = (float)bm;
    t[128 + n] = (float)wn;
    t[192 + n] = (float)(1.0 / wm);
    t[256 + n] = (float)(be * wn);
  }
  if (warp == 1) umma::tmem_alloc(tslot, L::TM_COLS);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::BAR_OFF + 120);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (!SO) prefetch_tmap(&tmQ);
      const uint32_t bytes = L::Q_BYTES + 2 * TILE + (p.eta ? MC * 4 : 0);
      int issued = 0;
      for (int c = 0; c < nch; ++c) {
        const int s = c % ST;
        if (c >= ST && !mbar_wait(empty + 8 * s, ((c / ST) - 1) & 1, p.err)) break;
        const uint32_t fb = full + 8 * s;
        const uint32_t st = sbase + s * L::STAGE;
        const int t0 = tok0 + c * MC;
        mbar_arrive_expect_tx(fb, bytes);
        if (!SO) {
          tma_load_3d(st, &tmQ, fb, 0, t0, stream);
          tma_load_3d(st + 8192, &tmQ, fb, 64, t0, stream);
        }
        tma_load_3d(st + L::K_OFF, &tmK, fb, 0, t0, stream);
        tma_load_3d(st + L::K_OFF + 8192, &tmK, fb, 64, t0, stream);
        tma_load_3d(st + L::V_OFF, &tmV, fb, 0, t0, stream);
        tma_load_3d(st + L::V_OFF + 8192, &tmV, fb, 64, t0, stream);
        if (p.eta)
          bulk_load(st + L::ETA_OFF, p.eta + (size_t)stream * p.T + t0, MC * 4, fb);
        issued = c + 1;
      }
      // copies still in flight land before the CTA may exit (normally all have)
      for (int c = std::max(0, issued - ST); c < issued; ++c)
        mbar_wait(full + 8 * (c % ST), (c / ST) & 1, p.err, 1000000000ull);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA warp
    // The whole warp runs the loop (warp-uniform waits); an elected lane issues.
    const uint32_t id_u = umma::idesc_bf16(128, 128, true, true);    // EV^T K
    const uint32_t id_o1 = umma::idesc_bf16(128, 64, false, false);  // Sb^T Q^T (A in TMEM)
    const uint32_t id_o2 = umma::idesc_bf16(128, 64, true, false);   // EVw^T P'^T
    for (int c = 0; c < nch; ++c) {
      const int s = c % ST, b = c & 1;
      const uint32_t sQ = sbase + s * L::STAGE, sK = sQ + L::K_OFF, sEVw = sQ + L::V_OFF;
      const uint32_t sEVb = sbase + L::EVB_OFF + b * TILE;
      if (!mbar_wait_warp(full + 8 * s, (c / ST) & 1, p.err)) break;
      if (!mbar_wait_warp(opready + 8 * b, (c >> 1) & 1, p.err)) break;
      if (!mbar_wait_warp(sready, c & 1, p.err)) break;
      umma::fence_after();
      // S^T += EVw^T K and M^T += EVb^T K (the refresh has applied the chunk's coupling)
#pragma unroll
      for (int ks = 0; ks < MC / 16; ++ks)
        umma::mma_ss_elect(tmem + TM_S, umma::desc_mnmajor(sEVw + 2048 * ks, 8192),
                           umma::desc_mnmajor(sK + 2048 * ks, 8192), id_u, true);
#pragma unroll
      for (int ks = 0; ks < MC / 16; ++ks)
        umma::mma_ss_elect(tmem + TM_M, umma::desc_mnmajor(sEVb + 2048 * ks, 8192),
                           umma::desc_mnmajor(sK + 2048 * ks, 8192), id_u, true);
      if (!SO) {
        // the output accumulators of chunk c-1 have been read out
        if (c >= 1 && !mbar_wait_warp(ofree, (c - 1) & 1, p.err)) break;
        umma::fence_after();
        const uint32_t sP = sbase + L::P_OFF + b * (MC * MC * 2);
#pragma unroll
        for (int ks = 0; ks < MD / 16; ++ks)
          umma::mma_ts_elect(tmem + TM_O, tmem + TM_SB + 8 * ks,
                             umma::desc_kmajor(sQ + (ks >> 2) * 8192 + (ks & 3) * 32), id_o1,
                             ks > 0);
#pragma unroll
        for (int ks = 0; ks < MC / 16; ++ks)
          umma::mma_ss_elect(tmem + TM_O, umma::desc_mnmajor(sEVw + 2048 * ks, 8192),
                             umma::desc_kmajor(sP + 32 * ks), id_o2, true);
#pragma unroll
        for (int ks = 0; ks < MD / 16; ++ks)
          umma::mma_ts_elect(tmem + TM_OM, tmem + TM_MB + 8 * ks,
                             umma::desc_kmajor(sQ + (ks >> 2) * 8192 + (ks & 3) * 32), id_o1,
                             ks > 0);
      }
      umma::commit_elect(cdone + 8 * b);
      umma::commit_elect(empty + 8 * s);   // Q, K, EVw of the stage are no longer read
    }
    // every MMA this warp issued completes before TMEM is released
    umma::commit_elect(mdone);
    mbar_wait_warp(mdone, 0, p.err, 1000000000ull);
  } else if (warp < L::REF0) {
    // ---------------------------------------------------------------- operand warps
    constexpr int NT = 32 * L::NOP;           // operand threads
    const int ow = warp - 2;
    const int otid = threadIdx.x - 64;
    const int g = lane >> 2, tq = lane & 3;
    for (int c = 0; c < nch; ++c) {
      const int s = c % ST, b = c & 1;
      const uint32_t stg = sbase + s * L::STAGE;
      // warp-uniform waits: the warp MMAs and ldmatrix below need every lane
      if (!mbar_wait_warp(full + 8 * s, (c / ST) & 1, p.err)) break;
      // EVb and P' buffers b were last read by the MMAs of chunk c-2
      if (c >= 2 && !mbar_wait_warp(cdone + 8 * b, ((c >> 1) - 1) & 1, p.err)) break;
      {
        // EVw (in place) and EVb: the V tile is 1024 16-byte pieces (a token row, eight
        // columns); piece i is row (i & 511) / 8 of sub-tile i / 512
        constexpr int PER = 1024 / NT;
        const uint32_t vt = stg + L::V_OFF;
        const uint32_t eb = sbase + L::EVB_OFF + b * TILE;
        uint4 x[PER];
        float fw[PER], fb[PER];
#pragma unroll
        for (int it = 0; it < PER; ++it) {
          const int i = otid + NT * it;
          const int w = i & 511, row = w >> 3;
          x[it] = lds128(vt + (i >> 9) * 8192 + swz<128>(row * 128 + (w & 7) * 16));
          const float e = p.eta ? ldsf(stg + L::ETA_OFF + 4 * row) : p.eta_scalar;
          fw[it] = e * ldsf(t_evw + 4 * row);
          fb[it] = e * ldsf(t_evb + 4 * row);
        }
#pragma unroll
        for (int it = 0; it < PER; ++it) {
          const int i = otid + NT * it;
          const int w = i & 511;
          const uint32_t off = (i >> 9) * 8192 + swz<128>((w >> 3) * 128 + (w & 7) * 16);
          const float f1 = fw[it], f2 = fb[it];
          const uint4 v = x[it];
          sts128(vt + off, make_uint4(pack_bf16(bf16_lo(v.x) * f1, bf16_hi(v.x) * f1),
                                      pack_bf16(bf16_lo(v.y) * f1, bf16_hi(v.y) * f1),
                                      pack_bf16(bf16_lo(v.z) * f1, bf16_hi(v.z) * f1),
                                      pack_bf16(bf16_lo(v.w) * f1, bf16_hi(v.w) * f1)));
          sts128(eb + off, make_uint4(pack_bf16(bf16_lo(v.x) * f2, bf16_hi(v.x) * f2),
                                      pack_bf16(bf16_lo(v.y) * f2, bf16_hi(v.y) * f2),
                                      pack_bf16(bf16_lo(v.z) * f2, bf16_hi(v.z) * f2),
                                      pack_bf16(bf16_lo(v.w) * f2, bf16_hi(v.w) * f2)));
        }
      }
      if (!SO) {
        // P' block of query rows 16 r .. +15 and keys 32 kh .. +31 (two 16-key blocks): the
        // blocks with keys past the rows are zero; the others take their scores on warp MMAs
        // from the swizzled Q and K tiles, then the causal weights
        const uint32_t sQ = stg, sK = stg + L::K_OFF;
        const int r = ow >> 1, kh = ow & 1;
        const int r0 = 16 * r;
        float acc[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
        const int arow = r0 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int acol = 8 * (lane >> 4);
        const int brow = (lane & 7) + 8 * (lane >> 4);
        const int bcol = 8 * ((lane >> 3) & 1);
        if (2 * kh <= r) {
#pragma unroll
          for (int ks = 0; ks < MD / 16; ++ks) {
            const uint32_t sub = (ks >> 2) * 8192;
            const int k0 = (ks & 3) * 16;
            uint32_t a[4];
            ldsm_x4(sQ + sub + swz<128>(arow * 128 + (k0 + acol) * 2), a);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const int kb = 2 * kh + kk;   // 16-key block
              if (kb <= r) {
                uint32_t bb[4];
                ldsm_x4(sK + sub + swz<128>((16 * kb + brow) * 128 + (k0 + bcol) * 2), bb);
                mma16816(acc[2 * kk], a[0], a[1], a[2], a[3], bb[0], bb[1]);
                mma16816(acc[2 * kk + 1], a[0], a[1], a[2], a[3], bb[2], bb[3]);
              }
            }
          }
        }
        // P'[i][j] = [j <= i] w(i - j) / w(63 - j) score, bf16, K-major [t][s] tile
        const uint32_t sP = sbase + L::P_OFF + b * (MC * MC * 2);
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          const int j0 = 32 * kh + 8 * n + 2 * tq;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int i = r0 + g + 8 * h;
            float v0 = 0.f, v1 = 0.f;
            if (j0 <= i) v0 = acc[n][2 * h] * ldsf(t_w + 4 * (i - j0)) * ldsf(t_rw + 4 * j0);
            if (j0 + 1 <= i)
              v1 = acc[n][2 * h + 1] * ldsf(t_w + 4 * (i - j0 - 1)) * ldsf(t_rw + 4 * (j0 + 1));
            sts32(sP + swz<128>(i * 128 + j0 * 2), pack_bf16(v0, v1));
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(opready + 8 * b);
    }
  } else if (warp < L::OUT0) {
    // ---------------------------------------------------------------- refresh warps 6..13
    const int q = warp & 3, h = (warp - L::REF0) >> 2;   // TMEM lane quarter, d_in part
    constexpr int CW = MD / (L::NREF / 4);              // d_in columns per refresh warp
    constexpr int NPC = CW / 16;                        // 16-column pieces
    const int dout = 32 * q + lane;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    float c63, b64;
    chunk_coeffs(p.beta, c63, b64);
    // the chunk's starting states S^T, M^T (lane = d_out) for d_in = din0 .. din0 + 15: bf16
    // copies for the outputs, then S += beta w(63) M, M *= beta^64 for the updates
    auto refresh_piece = [&](int din0, uint32_t (&sv)[16], uint32_t (&mv)[16]) {
      if (!SO) {
        uint32_t pk[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          pk[j] = pack_bf16(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1]));
        umma::st32x8(tmem + tl + TM_SB + din0 / 2, pk);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          pk[j] = pack_bf16(__uint_as_float(mv[2 * j]), __uint_as_float(mv[2 * j + 1]));
        umma::st32x8(tmem + tl + TM_MB + din0 / 2, pk);
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float m = __uint_as_float(mv[j]);
        sv[j] = __float_as_uint(fmaf(c63, m, __uint_as_float(sv[j])));
        mv[j] = __float_as_uint(b64 * m);
      }
      umma::st32x16(tmem + tl + TM_S + din0, sv);
      umma::st32x16(tmem + tl + TM_M + din0, mv);
    };
    // starting states of the part: pass 1 from zero; pass 2 from the caller's states (one part)
    // or from the prefix slot of the part
    const float* s_src = nullptr;
    const float* m_src = nullptr;
    int ld = MD, lim = MD;
    if (!SO) {
      if (p.start) {
        s_src = p.start + ((size_t)stream * p.nslots + (size_t)part * p.slot_mul) * 2 * MD * MD;
        m_src = s_src + MD * MD;
      } else {
        s_src = p.S0 ? p.S0 + (size_t)stream * p.dim * p.dim : nullptr;
        m_src = p.M0 ? p.M0 + (size_t)stream * p.dim * p.dim : nullptr;
        ld = lim = p.dim;
      }
    }
    // this warp's TMEM stores are complete and ordered before the MMAs that the barrier releases
    auto signal = [&](uint32_t mb) {
      umma::wait_st();
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(mb);
    };
    bool ok = true;
    for (int c = 0; c < nch; ++c) {
      if (c > 0) {
        // the MMAs of chunk c-1 are done: the states are updated and the bf16 copies free
        if (!mbar_wait_warp(cdone + 8 * ((c - 1) & 1), ((c - 1) >> 1) & 1, p.err)) {
          ok = false;
          break;
        }
        umma::fence_after();
      }
      if (c == 0) {
#pragma unroll 1
        for (int pc = 0; pc < NPC; ++pc) {
          const int din0 = CW * h + 16 * pc;
          uint32_t sv[16], mv[16];
          const bool in = dout < lim && din0 < lim;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            sv[j] = __float_as_uint(s_src && in ? s_src[(size_t)(din0 + j) * ld + dout] : 0.f);
            mv[j] = __float_as_uint(m_src && in ? m_src[(size_t)(din0 + j) * ld + dout] : 0.f);
          }
          refresh_piece(din0, sv, mv);
        }
      } else {
        // the loads of the next piece are in flight while a piece is converted and stored
        uint32_t sa[16], ma[16], sb2[16], mb2[16];
        umma::ld32x16(tmem + tl + TM_S + CW * h, sa);
        umma::ld32x16(tmem + tl + TM_M + CW * h, ma);
        umma::wait_ld();
        umma::reg_fence_n(sa);
        umma::reg_fence_n(ma);
#pragma unroll 1
        for (int pc = 0; pc < NPC; pc += 2) {
          const int din0 = CW * h + 16 * pc;
          umma::ld32x16(tmem + tl + TM_S + din0 + 16, sb2);
          umma::ld32x16(tmem + tl + TM_M + din0 + 16, mb2);
          refresh_piece(din0, sa, ma);
          umma::wait_ld();
          umma::reg_fence_n(sb2);
          umma::reg_fence_n(mb2);
          if (pc + 2 < NPC) {
            umma::ld32x16(tmem + tl + TM_S + din0 + 32, sa);
            umma::ld32x16(tmem + tl + TM_M + din0 + 32, ma);
          }
          refresh_piece(din0 + 16, sb2, mb2);
          if (pc + 2 < NPC) {
            umma::wait_ld();
            umma::reg_fence_n(sa);
            umma::reg_fence_n(ma);
          }
        }
      }
      signal(sready);
    }
    // final states: the piece's (dS, dM) in pass 1; S_out, M_out from the last part in pass 2
    if (ok && nch > 0 && (SO || part == p.P - 1) &&
        mbar_wait_warp(cdone + 8 * ((nch - 1) & 1), ((nch - 1) >> 1) & 1, p.err)) {
      umma::fence_after();
#pragma unroll 1
      for (int pc = 0; pc < CW / 32; ++pc) {
        const int din0 = CW * h + 32 * pc;
        uint32_t sv[32], mv[32];
        umma::ld32x32(tmem + tl + TM_S + din0, sv);
        umma::ld32x32(tmem + tl + TM_M + din0, mv);
        umma::wait_ld();
        umma::reg_fence(sv);
        umma::reg_fence(mv);
        if (SO) {
          float* ds = p.inc + ((size_t)stream * p.nslots + part + 1) * 2 * MD * MD;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            ds[(size_t)(din0 + j) * MD + dout] = __uint_as_float(sv[j]);
            ds[(size_t)MD * MD + (din0 + j) * MD + dout] = __uint_as_float(mv[j]);
          }
        } else if (dout < p.dim && din0 < p.dim) {
          float* so = p.S_dst + (size_t)stream * p.dim * p.dim;
          float* mo = p.M_dst + (size_t)stream * p.dim * p.dim;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            so[(size_t)(din0 + j) * p.dim + dout] = __uint_as_float(sv[j]);
            mo[(size_t)(din0 + j) * p.dim + dout] = __uint_as_float(mv[j]);
          }
        }
      }
    }
  } else if (!SO) {
    // ---------------------------------------------------------------- output warps 14..17
    const int q = warp & 3;
    const int dout = 32 * q + lane;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int otid = threadIdx.x - 32 * L::OUT0;   // 0..127
    const bool odd = lane & 1;
    // Lane pairs (2i, 2i+1) exchange one value per token pair (t, t+4) so that each lane stores
    // a 32-bit word of two adjacent output columns: the even lane row t, the odd lane row t+4.
    const uint32_t so = sbase + L::O_OFF + (dout >> 6) * 8192;
    const uint32_t cb = 2 * ((dout & 63) & ~1);
    for (int c = 0; c < nch; ++c) {
      const int b = c & 1;
      const bool got = mbar_wait_warp(cdone + 8 * b, (c >> 1) & 1, p.err);
      if (bar_or_named(1, 128, !got)) break;
      umma::fence_after();
      // the previous store has finished reading the staging tile
      if (otid == 0) bulk_wait_read<0>();
      bar_sync_named(1, 128);
#pragma unroll
      for (int qt = 0; qt < 4; ++qt) {   // tokens 16 qt .. 16 qt + 15
        uint32_t o[16], m[16];
        umma::ld32x16(tmem + tl + TM_O + 16 * qt, o);
        umma::ld32x16(tmem + tl + TM_OM + 16 * qt, m);
        umma::wait_ld();
        umma::reg_fence_n(o);
        umma::reg_fence_n(m);
        if (qt == 3) {   // both accumulators are read out: the next chunk's products may start
          umma::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(ofree);
        }
#pragma unroll
        for (int t = 0; t < 16; t += 4) {
          const uint4 cq = lds128(t_cq + 4 * (16 * qt + t));
          o[t] = __float_as_uint(fmaf(__uint_as_float(cq.x), __uint_as_float(m[t]),
                                      __uint_as_float(o[t])));
          o[t + 1] = __float_as_uint(fmaf(__uint_as_float(cq.y), __uint_as_float(m[t + 1]),
                                          __uint_as_float(o[t + 1])));
          o[t + 2] = __float_as_uint(fmaf(__uint_as_float(cq.z), __uint_as_float(m[t + 2]),
                                          __uint_as_float(o[t + 2])));
          o[t + 3] = __float_as_uint(fmaf(__uint_as_float(cq.w), __uint_as_float(m[t + 3]),
                                          __uint_as_float(o[t + 3])));
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          if (t & 4) continue;
          const float a = __uint_as_float(o[t]), a4 = __uint_as_float(o[t + 4]);
          const float y = __shfl_xor_sync(0xffffffffu, odd ? a : a4, 1);
          const float lo = odd ? y : a, hi = odd ? a4 : y;
          const int row = 16 * qt + (odd ? t + 4 : t);
          sts32(so + swz<128>(row * 128 + cb), pack_bf16(lo, hi));
        }
      }
      fence_proxy_async_smem();
      bar_sync_named(1, 128);
      if (otid == 0) {
        const int t0 = tok0 + c * MC;
        tma_store_3d(&tmO, sbase + L::O_OFF, 0, t0, stream);
        if (p.dim > 64) tma_store_3d(&tmO, sbase + L::O_OFF + 8192, 64, t0, stream);
        bulk_commit();
      }
    }
    if (otid == 0) bulk_wait<0>();
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 1) umma::tmem_dealloc(tmem, L::TM_COLS);
}

// Composes the pieces' maps in sequence order, per stream and state element: slot 0 receives
// the caller's starting states (zero-padded to the tile), slot k + 1 the states after piece k
// (in place of its increments): S <- S + c_L M + dS, M <- beta^L M + dM.
__global__ void mom_scan_kernel(const float* __restrict__ S0, const float* __restrict__ M0,
                                float* slots, int pieces, float cL, float bL, int dim) {
  const int stream = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= MD * MD) return;
  const int r = e / MD, col = e % MD;
  const bool in = r < dim && col < dim;
  const size_t user = (size_t)stream * dim * dim + (size_t)r * dim + col;
  float S = (S0 && in) ? S0[user] : 0.f;
  float M = (M0 && in) ? M0[user] : 0.f;
  float* base = slots + (size_t)stream * (pieces + 1) * 2 * MD * MD + e;
  base[0] = S;
  base[MD * MD] = M;
  for (int k = 1; k <= pieces; ++k) {
    float* sl = base + (size_t)k * 2 * MD * MD;
    const float dS = sl[0], dM = sl[MD * MD];
    S = fmaf(cL, M, S) + dS;
    M = fmaf(bL, M, dM);
    sl[0] = S;
    sl[MD * MD] = M;
  }
}

int mom_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// Parts per stream (pass 2): the most that keep one CTA per SM (a forced "assoc_parts" choice
// wins when it divides the chunks); pieces per part in pass 1 so that about every SM takes one.
void mom_layout(int streams, int T, int& P, int& F) {
  const int nch = T / MC, sms = mom_sms();
  const int forced = tuning(kTuneAssocParts);
  if (forced >= 1 && nch % forced == 0) {
    P = forced;
  } else {
    P = 1;
    while (nch % (2 * P) == 0 && streams * (2 * P) <= sms) P *= 2;
  }
  F = 1;
  if (P > 1) {
    F = std::max(1, std::min(4, sms / (streams * (P - 1))));
    while (F > 1 && (T / P) % (F * MC) != 0) --F;
  }
}

template <bool SO>
int launch_mom_chunk(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& to, const MomParams& p, int grid, const LaunchCtx& ctx) {
  using L = MomSmem<SO>;
  cudaError_t e = cudaFuncSetAttribute(mom_chunk_kernel<SO>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
  if (e == cudaSuccess) {
    mom_chunk_kernel<SO><<<grid, L::THREADS, L::BYTES, ctx.stream>>>(tq, tk, tv, to, p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    *ctx.msg = std::string("assoc momentum launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

size_t assoc_momentum_fused_workspace_bytes(int B, int H, int T, int d, int C_) {
  if (!assoc_supported(d, C_, T, 1)) return 0;
  int P, F;
  mom_layout(B * H, T, P, F);
  if (P <= 1) return 0;
  const size_t pieces = (size_t)(P - 1) * F;
  return (size_t)B * H * (pieces + 1) * 2 * MD * MD * sizeof(float);
}

int launch_assoc_momentum_fused(const AssocMomentumArgs& a, const LaunchCtx& ctx) {
  const int BH = a.B * a.H;
  int P, F;
  mom_layout(BH, a.T, P, F);
  const int pieces = (P - 1) * F;
  if (a.ws_bytes < assoc_momentum_fused_workspace_bytes(a.B, a.H, a.T, a.d, a.C)) {
    *ctx.msg = "ttt_assoc_momentum_fwd: workspace smaller than "
               "ttt_assoc_momentum_workspace_size()";
    return kWorkspace;
  }
  CUtensorMap tq, tk, tv, to;
  // d = 64: the tiles' second 64-wide half lies past the tensor and is filled with zeros, and
  // only the first half of each output tile is stored
  const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)a.T * a.d * 2};
  const uint32_t box[3] = {64, (uint32_t)MC, 1};
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tmap_3d(&tq, a.Q, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tk, a.K, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tv, a.V, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&to, a.O, bf, dims, strides, box, sw, ctx.msg))
    return kCuda;
  MomParams p{};
  p.eta = a.eta;
  p.eta_scalar = a.eta_scalar;
  p.beta = a.beta;
  p.T = a.T;
  p.dim = a.d;
  p.err = ctx.err;
  p.nslots = pieces + 1;
  p.slot_mul = F;
  float* slots = static_cast<float*>(a.ws);
  if (P > 1) {
    // pass 1: every piece of the first P - 1 parts from zero; the scan turns the pieces' maps
    // into the starting states of every part (slot 0 = the caller's states)
    MomParams p1 = p;
    p1.inc = slots;
    p1.P = pieces;
    p1.part_len = a.T / P / F;
    int st = launch_mom_chunk<true>(tq, tk, tv, to, p1, BH * pieces, ctx);
    if (st != kOk) return st;
    // the map of L tokens: c_L = sum_{r=1..L} beta^r, beta^L (beta = 1: c_L = L)
    const double be = a.beta, Lt = p1.part_len;
    const double bL = std::pow(be, Lt);
    const double cL = be == 1.0 ? Lt : be * (1.0 - bL) / (1.0 - be);
    mom_scan_kernel<<<dim3(MD * MD / 256, BH), 256, 0, ctx.stream>>>(
        a.S0, a.M0, slots, pieces, (float)cL, (float)bL, a.d);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      *ctx.msg = std::string("assoc momentum scan launch: ") + cudaGetErrorString(e);
      return kCuda;
    }
    count_launch();
    p.start = slots;
  } else {
    p.S0 = a.S0;
    p.M0 = a.M0;
  }
  p.P = P;
  p.part_len = a.T / P;
  p.S_dst = a.S_out;
  p.M_dst = a.M_out;
  return launch_mom_chunk<false>(tq, tk, tv, to, p, BH * P, ctx);
}

}  // namespace ttt
