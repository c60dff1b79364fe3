// Associative (weight-norm-free, gradient-ascent) linear-attention mode on tcgen05 + TMEM + TMA.
//
// Source: "KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다" (TTT with KV binding is in
// fact linear attention): with a linear bias-free last layer one inner step gives
// o = q(S0 + k^T v); without weight normalisation the state update is associative, so the
// sequence can be evaluated with a parallel prefix scan; per-token learning rates fold into the
// values; the inner loop ascends.
//     S_t = S_(t-1) + eta_t k_t^T v_t,   o_t = q_t S_t
// per chunk of C = 64 tokens:  O_c = Q_c S + (tril(Q_c K_c^T)) (diag(eta_c) V_c),
//                              S  += K_c^T (diag(eta_c) V_c)
//
// Two-pass prefix scan over superchunks. Each stream is cut into P superchunks ("parts") of
// T/P tokens. Pass 1 (assoc_chunk_kernel<true>) computes every part's state increment except
// the last; assoc_scan_kernel turns them, with S0, into each part's starting state; pass 2
// (assoc_chunk_kernel<false>) runs every part from its start, chunk by chunk, and the last part
// writes S_out. With P = 1 pass 1 and the scan vanish.
//
// One CTA per (stream, part) holds the whole state. Every d-sized dimension of the chunk
// contractions is put on the 128-row M side of the tensor core by computing the outputs
// transposed: with EV = diag(eta) V and P = tril(Q K^T),
//     O^T = S^T Q^T + EV^T P^T          (M = d_out, N = 64 tokens)
//     S^T += EV^T K                     (M = d_out, N = d_in, K = 64 tokens)
// The bf16 copy of S^T (refreshed after every update) lives in TMEM and feeds O^T = S^T Q^T as
// the A operand; EV is the V tile scaled by eta in place in shared memory and feeds the other
// two products as an MN-major A operand. TMEM columns: S^T fp32 [0,128), bf16 S^T (x2)
// [128,256), O^T (x2) [256,384), scores Q K^T (x2, M = 64) [384,512).
//
// Warp roles: warp 0 issues the TMA loads (3-stage ring of Q/K/V/eta tiles); warp 1 owns TMEM
// and issues the update and output MMAs; warp 14 issues the score MMAs Q K^T as soon as a stage
// lands; warps 2-5 (operand group) scale V by eta in place and turn the scores into the masked
// bf16 P tile; warps 6-9 (state group) and 10-13 (output group) each convert half of S^T to its
// bf16 copy after every update, and the output group drains O^T through a shared tile and
// TMA-stores it. Each group has one warp per TMEM sub-partition. The MMA-issuing warps run
// converged and issue through elect.sync. The serial chain per chunk is
// update -> bf16 copy -> update; everything else overlaps it.
#include <algorithm>
#include <cstdlib>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int D = 128;         // head dim
constexpr int C = 64;          // chunk
constexpr float H_MID = 0.5f * (C - 1);   // middle of a chunk (decay mode)
constexpr int THREADS = 480;   // TMA warp, MMA warp, 3 groups of 4 warps, score warp

// shared-memory map (bytes from the 1024-aligned base); pass 1 loads no Q and writes no O
template <bool SO>
struct Smem {
  static constexpr int Q_BYTES = SO ? 0 : C * D * 2;   // two [64 t][64 d_in] sub-tiles
  static constexpr int K_BYTES = C * D * 2;            // two [64 s][64 d_in] sub-tiles
  static constexpr int V_BYTES = C * D * 2;            // two [64 s][64 d_out] sub-tiles
  static constexpr int K_OFF = Q_BYTES;
  static constexpr int V_OFF = K_OFF + K_BYTES;
  static constexpr int ETA_OFF = V_OFF + V_BYTES;
  static constexpr int STAGE = ETA_OFF + 1024;         // eta (256 B) padded to keep alignment
  static constexpr int STAGES = SO ? 5 : 3;
  static constexpr int P_OFF = STAGES * STAGE;                // 2 x [64 t][64 s] bf16
  static constexpr int O_OFF = P_OFF + (SO ? 0 : 2 * 8192);   // 2 x [64 t][128 d_out] bf16
  static constexpr int BAR_OFF = O_OFF + (SO ? 0 : 2 * 16384);
  static constexpr int BYTES = 1024 + BAR_OFF + 1024;  // barriers, then three 64-float tables
  static_assert(BYTES <= 227 * 1024, "shared memory");
};

// TMEM columns
constexpr uint32_t TM_S = 0;      // S^T fp32, lanes = d_out, columns = d_in
constexpr uint32_t TM_SBF = 128;  // 2 x 64: bf16 S^T (d_in pairs), one per chunk parity
constexpr uint32_t TM_O = 256;    // 2 x 64: O^T fp32, lanes = d_out, columns = tokens
constexpr uint32_t TM_P = 384;    // 2 x 64: Q K^T (M = 64)
constexpr uint32_t TM_COLS = 512;

struct AssocParams {
  const float* eta;         // [BH, T] or null
  float eta_scalar;
  const float* S0;          // [BH, dim, dim] or null (zeros)
  const float* S_start;     // [BH, nslots, D, D] prefix of the pass-1 pieces (pass 2, P > 1):
                            // part m (m >= 1) starts from slot m * slot_mul - 1
  float* S_dst;             // pass 1: [BH, P-1, D, D] increments, or with dst_user the caller's
                            // [BH, dim, dim] state (single part); pass 2: S_out [BH, dim, dim]
  int T, P, part_len;
  int nslots, slot_mul;     // pass 2: prefix slots per stream and pass-1 pieces per part
  int dim;                  // the caller's head dim: 128, or 64 zero-padded to D in the kernel
  int dst_user;             // pass 1 writes the caller's state (one part) rather than increments
  int reverse;              // chunks last to first, transposed causal mask
  float eta_mul;            // every rate multiplied by this
  // Decay mode (one superchunk): the state follows M_t = beta M_(t-1) + eta_t k_t^T v_t and
  // o_t = q_t M_t (momentum). In a chunk with local token index i and h = (C - 1) / 2 the
  // kernel runs the plain chunk step on values scaled by beta^(h - i) from a state holding
  // beta^(h+1) M, multiplies output row i by beta^(i - h) and the state by beta^C after each
  // update; the final state is beta^h times what TMEM holds.
  // Pass 1 in decay mode sums a superchunk's increment with weights beta^(L - 1 - s) (L the
  // superchunk length, s the token index in it): per chunk c a factor beta^(L - C - cC) times
  // beta^(C - 1 - i) by local index i; the prefix over superchunks applies beta^L.
  int decay;
  float beta;
  const uint16_t* Oadd;     // pass 2, decay mode: O = Oadd + add_scale * (decayed output)
  float add_scale;
  const float* orow;        // pass 2: output row of token t scaled by oscale * orow[t] (or null)
  float oscale;
  unsigned* err;
};

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Barrier over `threads` threads that also returns whether any of them passed `pred` = true.
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

// REV (chunks last to first, transposed mask) and ROWSC (output row scales) are template
// parameters, not runtime flags: as runtime branches they measured 37% slower each on the plain
// forward (the kernel's warp roles are balanced to a few hundred cycles per chunk).
template <bool SO, bool DECAY = false, bool REV = false, bool ROWSC = false>
__global__ void __launch_bounds__(THREADS, 1)
    assoc_chunk_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmO, const AssocParams p) {
  using L = Smem<SO>;
  constexpr int ST = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + L::BAR_OFF;
  const uint32_t full = bar, empty = bar + 40;                  // stage ring (up to 5)
  const uint32_t pfull = bar + 80;                              // score accumulators (x2)
  const uint32_t pready = bar + 96;                             // P tile written (x2)
  const uint32_t go = bar + 112;                                // chunk operands ready (x2)
  const uint32_t afree = bar + 128;                             // chunk c's MMAs done (x2)
  const uint32_t ofull = bar + 144;                             // output accumulators (x2)
  const uint32_t sdone = bar + 160;                             // state update finished
  const uint32_t tslot = bar + 168;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // blockIdx = stream * nparts + part; pass 1 only covers parts 0 .. P-2
  const int nparts = SO ? p.P - 1 : p.P;
  const int stream = blockIdx.x / nparts, part = blockIdx.x % nparts;
  const int tok0 = part * p.part_len;
  const int nch = p.part_len / C;
  // first token of the c-th chunk this CTA processes (in reverse mode the sequence is walked
  // from its end, and part 0 is the last superchunk)
  auto tok = [&](int c) { return REV ? p.T - C - (tok0 + c * C) : tok0 + c * C; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(full + 8 * s, 1);
      // MMA warp + 4 operand warps (+ the score warp in pass 2)
      mbar_init(empty + 8 * s, SO ? 5 : 6);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(pfull + 8 * b, 1);
      mbar_init(pready + 8 * b, 4);
      // Chunk c may start once EV(c) is written (4 operand warps) and, in pass 2, once the
      // bf16 copy of the state before c is written (state and output warps, half each; the
      // output warps also have read out O^T(c-2) by then).
      mbar_init(go + 8 * b, SO ? 4 : 12);
      mbar_init(afree + 8 * b, 1);
      mbar_init(ofull + 8 * b, 1);
    }
    mbar_init(sdone, 1);
    fence_mbar_init();
  }
  if (DECAY && threadIdx.x < C) {
    const float x = (float)threadIdx.x - H_MID;
    reinterpret_cast<float*>(smem + L::BAR_OFF + 256)[threadIdx.x] =
        SO ? powf(p.beta, (float)(C - 1 - (int)threadIdx.x)) : powf(p.beta, -x);
    reinterpret_cast<float*>(smem + L::BAR_OFF + 512)[threadIdx.x] = powf(p.beta, x);
  }
  if (warp == 1) umma::tmem_alloc(tslot, TM_COLS);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::BAR_OFF + 168);
  // decay-mode factors by local token index: beta^(h - i) on values, beta^(i - h) on outputs
  const uint32_t evfac = bar + 256, ocfac = bar + 512;
  const uint32_t rtab = bar + 768;   // pass 2: the current chunk's output row scales

  // State and output warps (pass 2): bf16 copy of 64 of the 128 state columns for `chunk`.
  // Lane = d_out row of S^T; `half` selects d_in columns [64 half, 64 half + 64).
  const float beta_c = DECAY ? powf(p.beta, (float)C) : 1.f;   // decay of the state per chunk
  auto refresh = [&](int chunk, int half, uint32_t tl) {
    uint32_t a0[32], a1[32], o[32];
    umma::ld32x32(tmem + tl + TM_S + 64 * half, a0);
    umma::ld32x32(tmem + tl + TM_S + 64 * half + 32, a1);
    umma::wait_ld();
    umma::reg_fence(a0);
    umma::reg_fence(a1);
    if (DECAY && chunk > 0) {
      // state of the next chunk: beta^C times the updated one, written back in place
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        a0[j] = __float_as_uint(__uint_as_float(a0[j]) * beta_c);
        a1[j] = __float_as_uint(__uint_as_float(a1[j]) * beta_c);
      }
      umma::st32x32(tmem + tl + TM_S + 64 * half, a0);
      umma::st32x32(tmem + tl + TM_S + 64 * half + 32, a1);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      o[j] = pack_bf16(__uint_as_float(a0[2 * j]), __uint_as_float(a0[2 * j + 1]));
      o[16 + j] = pack_bf16(__uint_as_float(a1[2 * j]), __uint_as_float(a1[2 * j + 1]));
    }
    umma::st32x32(tmem + tl + TM_SBF + 64 * (chunk & 1) + 32 * half, o);
    umma::wait_st();
    umma::fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(go + 8 * (chunk & 1));
  };
  // Starting state S (d_in x d_out, row-major) of this part, columns [64 half, 64 half + 64)
  // of S^T, into TMEM.
  auto load_state = [&](int half, uint32_t tl, int dout) {
    // part 0 starts from the caller's [dim][dim] state (zero outside it when dim = 64), later
    // parts from the workspace's [D][D] prefix
    const float* src = nullptr;
    int ld = D;
    if (part == 0) {
      src = p.S0 ? p.S0 + (size_t)stream * p.dim * p.dim : nullptr;
      ld = p.dim;
      if (dout >= p.dim) src = nullptr;
    } else {
      src = p.S_start + ((size_t)stream * p.nslots + part * p.slot_mul - 1) * D * D;
    }
    const float sc = DECAY ? powf(p.beta, H_MID + 1.f) : 1.f;
#pragma unroll 1
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t v[32];
      const int din0 = 64 * half + 32 * cc;
      const bool in = src && din0 < (part == 0 ? p.dim : D);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        v[j] = __float_as_uint(in ? sc * src[(din0 + j) * ld + dout] : 0.f);
      umma::st32x32(tmem + tl + TM_S + din0, v);
    }
    umma::wait_st();
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (!SO) prefetch_tmap(&tmQ);
      const uint32_t bytes = L::Q_BYTES + L::K_BYTES + L::V_BYTES + (p.eta ? C * 4 : 0);
      for (int c = 0; c < nch; ++c) {
        const int s = c % ST;
        if (c >= ST && !mbar_wait(empty + 8 * s, ((c / ST) - 1) & 1, p.err)) break;
        const uint32_t fb = full + 8 * s;
        const uint32_t st = sbase + s * L::STAGE;
        const int t0 = tok(c);
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
          bulk_load(st + L::ETA_OFF, p.eta + (size_t)stream * p.T + t0, C * 4, fb);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- chain MMA warp
    // The whole warp runs this loop: every lane waits (warp-uniform results) and one elected
    // lane issues each MMA / commit, so no divergent branch surrounds them.
    const uint32_t id_o1 = umma::idesc_bf16(128, 64, false, false);  // S^T Q^T (A in TMEM)
    const uint32_t id_o2 = umma::idesc_bf16(128, 64, true, false);   // EV^T P^T
    const uint32_t id_u = umma::idesc_bf16(128, 128, true, true);    // EV^T K
    for (int c = 0; c < nch; ++c) {
      const int s = c % ST, b = c & 1;
      const uint32_t sQ = sbase + s * L::STAGE, sK = sQ + L::K_OFF;
      const uint32_t sEV = sQ + L::V_OFF;
      const uint32_t dO = tmem + TM_O + 64 * b;
      if (!mbar_wait_warp(full + 8 * s, (c / ST) & 1, p.err)) break;
      if (!mbar_wait_warp(go + 8 * b, (c >> 1) & 1, p.err)) break;
      umma::fence_after();
      // S^T += EV^T K: heads the serial chain, so it is issued first
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        umma::mma_ss_elect(tmem + TM_S, umma::desc_mnmajor(sEV + 2048 * ks, 8192),
                           umma::desc_mnmajor(sK + 2048 * ks, 8192), id_u,
                           SO ? (c > 0 || ks > 0) : true);
      // Pass 2 signals every update (the state and output warps refresh the bf16 copy);
      // pass 1 only the final one.
      if (!SO || c + 1 == nch) umma::commit_elect(sdone);
      if (SO) {
        umma::commit_elect(empty + 8 * s);
        umma::commit_elect(afree + 8 * b);
        continue;
      }
      // O^T = S^T Q^T with the bf16 copy of the state before this chunk
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        umma::mma_ts_elect(dO, tmem + TM_SBF + 64 * b + 8 * ks,
                           umma::desc_kmajor(sQ + (ks >> 2) * 8192 + (ks & 3) * 32), id_o1,
                           ks > 0);
      if (!mbar_wait_warp(pready + 8 * b, (c >> 1) & 1, p.err)) break;
      umma::fence_after();
      const uint32_t sP = sbase + L::P_OFF + 8192 * b;
      // O^T += EV^T P^T
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        umma::mma_ss_elect(dO, umma::desc_mnmajor(sEV + 2048 * ks, 8192),
                           umma::desc_kmajor(sP + 32 * ks), id_o2, true);
      umma::commit_elect(ofull + 8 * b);
      umma::commit_elect(afree + 8 * b);
      umma::commit_elect(empty + 8 * s);   // the stage (Q, K, EV) is no longer needed
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------------- operand warps 2..5
    const int q = warp & 3;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const bool rowthr = lane < 16;            // holds an M = 64 score row
    const int r = 16 * q + lane;              // that row (token t of the chunk)
    const int otid = threadIdx.x - 64;       // 0..127
    // decay mode: the value factor of each of this thread's four token rows (rows of pieces
    // it and it + 4 coincide), read from the table once instead of per chunk
    float vfac[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      vfac[j] = DECAY ? ldsf(evfac + 4 * (((otid + 128 * j) & 511) >> 3)) : 1.f;
    for (int c = 0; c < nch; ++c) {
      const int s = c % ST, b = c & 1;
      const uint32_t stg = sbase + s * L::STAGE;
      if (!mbar_wait(full + 8 * s, (c / ST) & 1, p.err)) break;
      // The arrival on go(c) below must not come before go(c-2) has been consumed, or it
      // would complete that phase in place of the state warps: the MMAs of chunk c-2
      // finishing (afree(c-2)) shows that it has.
      if (c >= 2 && !mbar_wait(afree + 8 * b, ((c >> 1) - 1) & 1, p.err)) break;
      // EV = diag(eta) V in place: the V tile is 1024 16-byte pieces (row = token, eight
      // columns each); piece i is row i / 16 of the two sub-tiles' swizzled layout.
      {
        const float cf = (DECAY && SO) ? powf(p.beta, (float)(p.part_len - C - c * C)) : 1.f;
        const uint32_t vt = stg + L::V_OFF;
        uint4 x[8];
        float e[4];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int i = otid + 128 * it;                // 0..1023
          const int sub = i >> 9, w = i & 511;          // sub-tile, piece within it
          const uint32_t a = vt + sub * 8192 + swz<128>((w >> 3) * 128 + (w & 7) * 16);
          x[it] = lds128(a);
          // pieces it and it + 4 share a token row: four rate loads per thread, not eight
          if (it < 4) e[it] = p.eta ? ldsf(stg + L::ETA_OFF + 4 * (w >> 3)) : p.eta_scalar;
        }
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int i = otid + 128 * it;
          const int sub = i >> 9, w = i & 511;
          const uint32_t a = vt + sub * 8192 + swz<128>((w >> 3) * 128 + (w & 7) * 16);
          const float f = e[it & 3] * p.eta_mul * (DECAY ? cf * vfac[it & 3] : 1.f);
          sts128(a, make_uint4(pack_bf16(bf16_lo(x[it].x) * f, bf16_hi(x[it].x) * f),
                               pack_bf16(bf16_lo(x[it].y) * f, bf16_hi(x[it].y) * f),
                               pack_bf16(bf16_lo(x[it].z) * f, bf16_hi(x[it].z) * f),
                               pack_bf16(bf16_lo(x[it].w) * f, bf16_hi(x[it].w) * f)));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(go + 8 * b);
        mbar_arrive(empty + 8 * s);
      }
      if (SO) continue;
      // masked scores -> P tile [t][s]; P tile b was last read by the MMAs of chunk c-2
      if (!mbar_wait(pfull + 8 * b, (c >> 1) & 1, p.err)) break;
      umma::fence_after();
      uint32_t v0[32], v1[32];
      umma::ld32x32(tmem + tl + TM_P + 64 * b, v0);
      umma::ld32x32(tmem + tl + TM_P + 64 * b + 32, v1);
      umma::wait_ld();
      umma::reg_fence(v0);
      umma::reg_fence(v1);
      umma::fence_before();
      if (rowthr) {
        const uint32_t prow = sbase + L::P_OFF + 8192 * b;
#pragma unroll
        for (int j = 0; j < 64; j += 8) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int sidx = j + e;
            const float x = __uint_as_float(sidx < 32 ? v0[sidx] : v1[sidx - 32]);
            f[e] = (REV ? sidx >= r : sidx <= r) ? x : 0.f;
          }
          sts128(prow + swz<128>(r * 128 + 2 * j),
                 make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                            pack_bf16(f[6], f[7])));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      // pready(c) also tells the score warp that score buffer b has been read
      if (lane == 0) mbar_arrive(pready + 8 * b);
    }
  } else if (warp < 10) {
    // ---------------------------------------------------------------- state warps 6..9
    const int q = warp & 3;
    const int dout = 32 * q + lane;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    bool ok = true;
    if (!SO) {
      load_state(0, tl, dout);
      refresh(0, 0, tl);
      for (int c = 0; c < nch; ++c) {
        if (!mbar_wait(sdone, c & 1, p.err)) { ok = false; break; }
        umma::fence_after();
        if (c + 1 < nch) refresh(c + 1, 0, tl);
      }
    } else {
      ok = mbar_wait(sdone, 0, p.err);
      umma::fence_after();
    }
    // ---- final state of the part: increment (pass 1) or S_out (pass 2, last part)
    if (ok && (SO || part == p.P - 1)) {
      // the caller's [dim][dim] state (pass 2, or pass 1 over one part), else a [D][D]
      // workspace increment
      const bool user = !SO || p.dst_user;
      const int ld = user ? p.dim : D;
      float* dst = user ? p.S_dst + (size_t)stream * p.dim * p.dim
                        : p.S_dst + ((size_t)stream * (p.P - 1) + part) * D * D;
      // pass 2 in decay mode holds beta^(h+1) M and ends with beta^h times the state; pass 1
      // accumulates the weighted increment itself
      const float sc = (DECAY && !SO) ? powf(p.beta, H_MID) : 1.f;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        umma::ld32x32(tmem + tl + TM_S + 32 * cc, v);
        umma::wait_ld();
        umma::reg_fence(v);
        if (dout < ld && 32 * cc < ld) {
#pragma unroll
          for (int j = 0; j < 32; ++j) dst[(32 * cc + j) * ld + dout] = sc * __uint_as_float(v[j]);
        }
      }
    }
  } else if (warp < 14) {
    // ---------------------------------------------------------------- output warps 10..13
    if (SO) goto done;   // pass 1 has no outputs
    {
      const int q = warp & 3;
      const int dout = 32 * q + lane;
      const uint32_t tl = (uint32_t)(32 * q) << 16;
      const int otid = threadIdx.x - 320;        // 0..127
      const bool odd = lane & 1;
      // Lane pairs (2i, 2i+1) exchange one value per token pair (t, t+4) so that each lane
      // stores a 32-bit word of two adjacent output columns: the even lane row t, the odd
      // lane row t+4 (the two rows fall in disjoint bank halves of the swizzled tile).
      const uint32_t ocol = (dout >> 6) * 8192;
      const uint32_t cb = 2 * ((dout & 63) & ~1);
      // Row scales (p.orow): chunk c+1's are loaded into registers at the top of iteration c
      // and written to the table after iteration c's epilogue has read chunk c's, so the load
      // never stalls the half refresh these warps run on the chain; the barrier that ends the
      // iteration publishes them.
      const bool rows_scaled = ROWSC && p.orow && otid < C / 4;
      auto load_rows = [&](int c) {   // volatile asm: stays where it is issued
        uint4 v;
        asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "l"(p.orow + (size_t)stream * p.T + tok(c) + 4 * otid));
        return v;
      };
      uint4 rnext = make_uint4(0u, 0u, 0u, 0u);
      if (rows_scaled) sts128(rtab + 16 * otid, load_rows(0));
      load_state(1, tl, dout);
      refresh(0, 1, tl);
      for (int c = 0; c < nch; ++c) {
        const int b = c & 1;
        if (rows_scaled && c + 1 < nch) rnext = load_rows(c + 1);
        // decay mode: the words this lane rewrites, read back before the waits below (all
        // loads in flight at once; each word is read once, before this kernel stores that row)
        uint32_t oadd[DECAY ? 32 : 1];
        if (DECAY && p.Oadd && dout < p.dim) {
          const uint32_t* ob = reinterpret_cast<const uint32_t*>(
              p.Oadd + ((size_t)stream * p.T + tok(c)) * p.dim + (dout & ~1));
#pragma unroll
          for (int t = 0; t < C; ++t) {
            if (t & 4) continue;
            // volatile asm keeps the load here, ahead of the waits, instead of at its use
            asm volatile("ld.global.u32 %0, [%1];"
                         : "=r"(oadd[(t >> 3) * 4 + (t & 3)])
                         : "l"(ob + (size_t)(odd ? t + 4 : t) * (p.dim / 2)));
          }
        }
        // second half of the bf16 state copy for chunk c+1; the go(c+1) arrival also says
        // that O^T(c-1) has been read out
        bool got = mbar_wait(sdone, c & 1, p.err);
        if (got) {
          umma::fence_after();
          if (c + 1 < nch) refresh(c + 1, 1, tl);
          got = mbar_wait(ofull + 8 * b, (c >> 1) & 1, p.err);
        }
        if (named_bar_or(2, 128, !got)) break;
        umma::fence_after();
        uint32_t v0[32], v1[32];
        umma::ld32x32(tmem + tl + TM_O + 64 * b, v0);
        umma::ld32x32(tmem + tl + TM_O + 64 * b + 32, v1);
        umma::wait_ld();
        umma::reg_fence(v0);
        umma::reg_fence(v1);
        umma::fence_before();
        const uint32_t so = sbase + L::O_OFF + 16384 * b + ocol;
        auto epilogue = [&](auto scaled_c) {
          constexpr bool SCALED = decltype(scaled_c)::value;
          uint4 of0 = make_uint4(0u, 0u, 0u, 0u), of4 = of0;
#pragma unroll
          for (int t = 0; t < C; ++t) {
            if (t & 4) continue;
            const uint32_t* vv = t < 32 ? v0 : v1;
            const int tt = t & 31;
            float a = __uint_as_float(vv[tt]), a4 = __uint_as_float(vv[tt + 4]);
            if (DECAY) {   // row factors of rows t0..t0+3 and t0+4..t0+7, four per load
              if ((t & 3) == 0) {
                of0 = lds128(ocfac + 4 * t);
                of4 = lds128(ocfac + 4 * (t + 4));
              }
              const int k = t & 3;
              a *= __uint_as_float(k == 0 ? of0.x : k == 1 ? of0.y : k == 2 ? of0.z : of0.w);
              a4 *= __uint_as_float(k == 0 ? of4.x : k == 1 ? of4.y : k == 2 ? of4.z : of4.w);
            }
            const float y = __shfl_xor_sync(0xffffffffu, odd ? a : a4, 1);
            float lo = odd ? y : a, hi = odd ? a4 : y;   // columns (dout & ~1) and (dout | 1)
            const int row = odd ? t + 4 : t;
            if constexpr (SCALED) {
              const float sr = p.oscale * (p.orow ? ldsf(rtab + 4 * row) : 1.f);
              lo *= sr, hi *= sr;
            }
            if (DECAY && p.Oadd) {
              const uint32_t base = oadd[(t >> 3) * 4 + (t & 3)];
              lo = __uint_as_float(base << 16) + p.add_scale * lo;
              hi = __uint_as_float(base & 0xffff0000u) + p.add_scale * hi;
            }
            const uint32_t w = pack_bf16(lo, hi);
            sts32(so + swz<128>(row * 128 + cb), w);
          }
        };
        epilogue(std::integral_constant<bool, ROWSC>{});
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (otid == 0) {
          const uint32_t sO = sbase + L::O_OFF + 16384 * b;
          tma_store_3d(&tmO, sO, 0, tok(c), stream);
          if (p.dim > 64) tma_store_3d(&tmO, sO + 8192, 64, tok(c), stream);
          bulk_commit();
          bulk_wait_read<1>();  // the other staging buffer is free again
        }
        if (rows_scaled && c + 1 < nch) sts128(rtab + 16 * otid, rnext);
        named_bar_sync(2, 128);
      }
      if (otid == 0) bulk_wait<0>();
    }
  } else if (!SO) {
    // ---------------------------------------------------------------- score warp 14
    // D_P(c) = Q_c K_c^T into score buffer c % 2, issued as soon as the tiles land and the
    // operand warps have read the scores of chunk c-2.
    const uint32_t id_s = umma::idesc_bf16(64, 64, false, false);
    for (int c = 0; c < nch; ++c) {
      const int s = c % ST, b = c & 1;
      if (!mbar_wait_warp(full + 8 * s, (c / ST) & 1, p.err)) break;
      if (c >= 2 && !mbar_wait_warp(pready + 8 * b, ((c >> 1) - 1) & 1, p.err)) break;
      umma::fence_after();
      const uint32_t sQ = sbase + s * L::STAGE, sK = sQ + L::K_OFF;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t o = (ks >> 2) * 8192 + (ks & 3) * 32;
        umma::mma_ss_elect(tmem + TM_P + 64 * b, umma::desc_kmajor(sQ + o),
                           umma::desc_kmajor(sK + o), id_s, ks > 0);
      }
      umma::commit_elect(pfull + 8 * b);
      umma::commit_elect(empty + 8 * s);
    }
  }
done:
  umma::fence_before();
  __syncthreads();
  if (warp == 1) umma::tmem_dealloc(tmem, TM_COLS);
}

// Exclusive prefix over the parts' increments, in place: slot p-1 becomes the start of part p.
// (decay mode: each step first multiplies the running state by decay_L = beta^L.)
// S0 is the caller's [dim][dim] state (zero outside it in the [D][D] increments when dim = 64).
__global__ void assoc_scan_kernel(const float* __restrict__ S0, float* inc, int P, float decay_L,
                                  int dim) {
  const int stream = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;   // element of the D x D state
  if (e >= D * D) return;
  const int r = e / D, col = e % D;
  float run = (S0 && r < dim && col < dim) ? S0[(size_t)stream * dim * dim + r * dim + col] : 0.f;
  float* base = inc + (size_t)stream * (P - 1) * D * D + e;
  for (int pp = 0; pp < P - 1; ++pp) {
    run = decay_L * run + base[(size_t)pp * D * D];
    base[(size_t)pp * D * D] = run;
  }
}

int choose_parts(int streams, int T) {
  const int nchunks = T / C;
  const int f = tuning(kTuneAssocParts);
  if (f >= 1 && nchunks % f == 0) return f;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int P = 1;
  while (nchunks % (2 * P) == 0 && streams * (2 * P) <= sms) P *= 2;
  return P;
}

template <bool STATE_ONLY>
int launch_chunk(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const CUtensorMap& to, const AssocParams& p, int grid, const LaunchCtx& ctx) {
  using Kern = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, AssocParams);
  Kern kern = assoc_chunk_kernel<STATE_ONLY, false, false, false>;
  const bool rows = !STATE_ONLY && (p.orow || p.oscale != 1.f);
  if (p.decay) {
    kern = assoc_chunk_kernel<STATE_ONLY, true, false, false>;
  } else if (p.reverse) {
    kern = assoc_chunk_kernel<STATE_ONLY, false, true, false>;
    if constexpr (!STATE_ONLY)
      if (rows) kern = assoc_chunk_kernel<false, false, true, true>;
  } else if constexpr (!STATE_ONLY) {
    if (rows) kern = assoc_chunk_kernel<false, false, false, true>;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Smem<STATE_ONLY>::BYTES);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  kern<<<grid, THREADS, Smem<STATE_ONLY>::BYTES, ctx.stream>>>(tq, tk, tv, to, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("assoc launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

bool assoc_supported(int d, int C_, int T, int dt) {
  return dt == 1 && (d == D || d == 64) && (C_ == 16 || C_ == 32 || C_ == C) && T % C == 0;
}

int launch_assoc_state(const StateArgs& a, const LaunchCtx& ctx) {
  // Pass 1 over the whole sequence as a single superchunk: S_out = sum_t eta_t k_t^T v_t.
  const int BH = a.B * a.H;
  CUtensorMap tq, tk, tv, to;
  // d = 64: the tiles' second 64-wide half lies past the tensor and is filled with zeros
  const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)a.T * a.d * 2};
  const uint32_t box[3] = {64, (uint32_t)C, 1};
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tmap_3d(&tk, a.K, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tv, a.V, bf, dims, strides, box, sw, ctx.msg))
    return kCuda;
  tq = tk;  // unused in state-only mode
  to = tk;
  AssocParams p;
  p.eta = a.eta;
  p.eta_scalar = a.eta_scalar;
  p.S0 = nullptr;
  p.S_start = nullptr;
  p.S_dst = a.S_out;
  p.nslots = 1;
  p.slot_mul = 1;
  p.dst_user = 1;
  p.dim = a.d;
  p.T = a.T;
  p.P = 2;             // parts 0 .. P-2 = the single part [0, T)
  p.part_len = a.T;
  p.reverse = a.reverse;
  p.eta_mul = a.eta_mul;
  p.decay = a.decay;
  p.beta = a.beta;
  p.Oadd = static_cast<const uint16_t*>(a.Oadd);
  p.add_scale = a.add_scale;
  p.orow = a.orow;
  p.oscale = a.oscale;
  p.err = ctx.err;
  return launch_chunk<true>(tq, tk, tv, to, p, BH, ctx);
}

// Pass-1 pieces per superchunk: pass 1 covers the first P - 1 superchunks, each cut into F
// pieces so that about every SM takes a piece (F <= 4, pieces of whole chunks).
int choose_pieces(int streams, int T, int P) {
  if (P <= 1) return 1;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int F = std::max(1, std::min(4, sms / (streams * (P - 1))));
  while (F > 1 && (T / P) % (F * C) != 0) --F;
  return F;
}

size_t assoc_workspace_bytes(int B, int H, int T, int d, int C_) {
  if (!assoc_supported(d, C_, T, 1)) return 0;
  const int P = choose_parts(B * H, T);
  const int F = choose_pieces(B * H, T, P);
  return (size_t)B * H * (P - 1) * F * D * D * sizeof(float);
}

namespace {

// Tensor maps and the launch parameters shared by both passes of one call.
int assoc_setup(const StateArgs& a, CUtensorMap* tq, CUtensorMap* tk, CUtensorMap* tv,
                CUtensorMap* to, AssocParams* pp, const LaunchCtx& ctx) {
  const int BH = a.B * a.H;
  // d = 64: the tiles' second 64-wide half lies past the tensor and is filled with zeros, and
  // only the first half of each output tile is stored
  const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)a.T * a.d * 2};
  const uint32_t box[3] = {64, (uint32_t)C, 1};
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tmap_3d(tq, a.Q, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(tk, a.K, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(tv, a.V, bf, dims, strides, box, sw, ctx.msg) ||
      (a.O ? !make_tmap_3d(to, a.O, bf, dims, strides, box, sw, ctx.msg) : (*to = *tk, false)))
    return kCuda;
  AssocParams& p = *pp;
  p.eta = a.eta;
  p.eta_scalar = a.eta_scalar;
  p.S0 = a.S0;
  p.S_start = static_cast<const float*>(a.ws);
  p.dim = a.d;
  p.dst_user = 0;
  p.T = a.T;
  p.reverse = a.reverse;
  p.eta_mul = a.eta_mul;
  p.decay = a.decay;
  p.beta = a.beta;
  p.Oadd = static_cast<const uint16_t*>(a.Oadd);
  p.add_scale = a.add_scale;
  p.orow = a.orow;
  p.oscale = a.oscale;
  p.err = ctx.err;
  return kOk;
}

// Pass 1 and the prefix: the increments of the first P - 1 superchunks, F pieces each (a part of
// T / (P F) tokens per CTA), turned by the scan into the starting state of every piece.
int run_pass1_prefix(const StateArgs& a, int P, int F, const CUtensorMap& tq,
                     const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                     const AssocParams& p, const LaunchCtx& ctx) {
  const int BH = a.B * a.H, pieces = (P - 1) * F;
  AssocParams p1 = p;
  p1.S_dst = static_cast<float*>(a.ws);
  p1.P = pieces + 1;
  p1.part_len = a.T / P / F;
  int st = launch_chunk<true>(tq, tk, tv, to, p1, BH * pieces, ctx);
  if (st != kOk) return st;
  const float decay_L = a.decay ? powf(a.beta, (float)p1.part_len) : 1.f;
  assoc_scan_kernel<<<dim3(D * D / 256, BH), 256, 0, ctx.stream>>>(a.S0, p1.S_dst, pieces + 1,
                                                                   decay_L, a.d);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("assoc scan launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

int launch_assoc_prefix(const StateArgs& a, AssocPrefix* out, const LaunchCtx& ctx) {
  const int BH = a.B * a.H;
  const int P = choose_parts(BH, a.T);
  const int F = choose_pieces(BH, a.T, P);
  const int pieces = (P - 1) * F;
  if (a.ws_bytes < (size_t)BH * pieces * D * D * sizeof(float)) {
    *ctx.msg = "associative prefix: workspace smaller than the pass-1 increments";
    return kWorkspace;
  }
  out->P = P;
  out->nslots = pieces;
  out->slot_mul = F;
  out->slots = static_cast<const float*>(a.ws);
  if (P <= 1) return kOk;
  CUtensorMap tq, tk, tv, to;
  AssocParams p;
  StateArgs s = a;
  s.Q = a.K;   // pass 1 reads no queries
  s.O = nullptr;
  int st = assoc_setup(s, &tq, &tk, &tv, &to, &p, ctx);
  if (st != kOk) return st;
  return run_pass1_prefix(s, P, F, tq, tk, tv, to, p, ctx);
}

int launch_assoc(const StateArgs& a, const LaunchCtx& ctx) {
  const int BH = a.B * a.H;
  const int P = choose_parts(BH, a.T);
  const int F = choose_pieces(BH, a.T, P);
  const int pieces = (P - 1) * F;   // pass-1 increments per stream
  const size_t need = (size_t)BH * pieces * D * D * sizeof(float);
  if (a.ws_bytes < need) {
    *ctx.msg = "ttt_assoc_scan_fwd: workspace smaller than ttt_assoc_scan_workspace_size()";
    return kWorkspace;
  }
  CUtensorMap tq, tk, tv, to;
  AssocParams p;
  int st = assoc_setup(a, &tq, &tk, &tv, &to, &p, ctx);
  if (st != kOk) return st;
  p.P = P;
  p.part_len = a.T / P;
  p.nslots = pieces;
  p.slot_mul = F;
  if (P > 1 && (st = run_pass1_prefix(a, P, F, tq, tk, tv, to, p, ctx)) != kOk) return st;
  p.S_dst = a.S_out;
  return launch_chunk<false>(tq, tk, tv, to, p, BH * P, ctx);
}

}  // namespace ttt
