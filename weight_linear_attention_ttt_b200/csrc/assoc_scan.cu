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
// writes S_out. P is chosen so that streams x parts x 2 column halves fill the GPU; with P = 1
// pass 1 and the scan vanish.
//
// Pass-2 CTA = (stream, part, half of the output columns). The state S^T[half] (64 x 128 fp32)
// stays in TMEM (M = 64 accumulator) for the whole part. Per chunk:
//   MMA-S  D_P = Q_c K_c^T                        (A = Q, B = K; both K-major TMA tiles)
//   warps  mask D_P (s <= t) -> bf16 P tile; eta-scale the V half -> bf16 EV tile
//   MMA-O  D_O = Q_c bf16(S) + P * EV             (B = bf16 copy of S^T, K-major)
//   MMA-U  D_S += EV^T K_c                        (A = EV, MN-major; B = K, MN-major)
//   warps  D_S -> bf16 copy of S^T for the next chunk; D_O -> bf16 O tile -> TMA store
// Warp 0 issues TMA loads (3-stage ring); warp 1 owns TMEM and issues the MMAs from one thread;
// warps 2-5 ("attention" group) turn scores into the masked P tile, scale V by eta and drain O;
// warps 6-9 ("state" group) only refresh the bf16 copy of S after each update. The serial
// chain per chunk is therefore MMA-U -> S readout -> MMA-U; the attention work of the next
// chunk and the outputs of this one run beside it. Each group has one warp per TMEM
// sub-partition.
#include <algorithm>
#include <cstdlib>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int D = 128;       // head dim
constexpr int C = 64;        // chunk
constexpr int HALF = 64;     // output columns per CTA
constexpr int THREADS = 320;   // TMA warp, MMA warp, 4 attention warps, 4 state warps
constexpr int STAGES = 3;

// shared-memory map (bytes from the 1024-aligned base)
constexpr int Q_BYTES = C * D * 2;        // two [64][64] sub-tiles
constexpr int K_BYTES = C * D * 2;
constexpr int V_BYTES = C * HALF * 2;     // one [64][64] sub-tile
constexpr int ETA_BYTES = 1024;
constexpr int STAGE_BYTES = Q_BYTES + K_BYTES + V_BYTES + ETA_BYTES;
constexpr int P_OFF = STAGES * STAGE_BYTES;              // 2 x [64 t][64 s] bf16
constexpr int EV_OFF = P_OFF + 2 * 8192;                 // 2 x [64 s][64 dout] bf16
constexpr int SB_OFF = EV_OFF + 2 * 8192;                // 2 x S^T bf16 [64 dout][128 din]
constexpr int O_OFF = SB_OFF + 2 * 16384;                // 2 x [64 t][64 dout] bf16
constexpr int BAR_OFF = O_OFF + 2 * 8192;
constexpr int SMEM = 1024 + BAR_OFF + 256;
static_assert(SMEM <= 227 * 1024, "shared memory");

// TMEM columns
constexpr uint32_t TM_S = 0;     // 128 columns: S^T half (M = 64)
constexpr uint32_t TM_P = 128;   // 2 x 64: scores
constexpr uint32_t TM_O = 256;   // 2 x 64: outputs
constexpr uint32_t TM_COLS = 512;

struct AssocParams {
  const float* eta;         // [BH, T] or null
  float eta_scalar;
  const float* S0;          // [BH, D, D] or null (zeros)
  const float* S_start;     // [BH, P-1, D, D] starting states of parts 1.. (pass 2, P > 1)
  float* S_dst;             // pass 1: [BH, P-1, D, D] increments; pass 2: S_out [BH, D, D]
  int T, P, part_len;
  unsigned* err;
};

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Row r (0..63) of an M = 64 accumulator lives in TMEM lane 32 * (r / 16) + r % 16: compute
// warp with sub-partition q holds rows 16q .. 16q+15 in its threads 0..15.
template <bool STATE_ONLY>
__global__ void __launch_bounds__(THREADS, 1)
    assoc_chunk_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmO, const AssocParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + BAR_OFF;
  const uint32_t full = bar, empty = bar + 8 * STAGES;          // stage ring
  const uint32_t pfull = bar + 48, pempty = bar + 64;           // score accumulators
  const uint32_t aready = bar + 80;                             // P / EV tiles written
  const uint32_t sdone = bar + 96;                              // state update finished
  const uint32_t sready = bar + 104;                            // bf16 S copy written (x2)
  const uint32_t ofull = bar + 120, oempty = bar + 136;         // output accumulators
  const uint32_t tslot = bar + 160;
  const uint32_t evfree = bar + 168;                            // pass 1: EV tile reusable (x2)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // pass 2: blockIdx = (stream * P + part) * 2 + half; pass 1 only covers parts 0 .. P-2
  const int nparts = STATE_ONLY ? p.P - 1 : p.P;
  const int half = blockIdx.x & 1;
  const int sp = blockIdx.x >> 1;
  const int stream = sp / nparts, part = sp % nparts;
  const int tok0 = part * p.part_len;
  const int nch = p.part_len / C;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 5);  // MMA commit + 4 compute warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(pfull + 8 * b, 1);
      mbar_init(pempty + 8 * b, 4);
      mbar_init(aready + 8 * b, 4);
      mbar_init(sready + 8 * b, 4);
      mbar_init(ofull + 8 * b, 1);
      mbar_init(oempty + 8 * b, 4);
    }
    mbar_init(sdone, 1);
    mbar_init(evfree, 1);
    mbar_init(evfree + 8, 1);
    fence_mbar_init();
  }
  if (warp == 1) umma::tmem_alloc(tslot, TM_COLS);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + BAR_OFF + 160);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (!STATE_ONLY) prefetch_tmap(&tmQ);
      const uint32_t bytes = K_BYTES + V_BYTES + (STATE_ONLY ? 0 : Q_BYTES) + (p.eta ? C * 4 : 0);
      for (int c = 0; c < nch; ++c) {
        const int s = c % STAGES;
        if (c >= STAGES && !mbar_wait(empty + 8 * s, ((c / STAGES) - 1) & 1, p.err)) break;
        const uint32_t fb = full + 8 * s;
        const uint32_t st = sbase + s * STAGE_BYTES;
        const int t0 = tok0 + c * C;
        mbar_arrive_expect_tx(fb, bytes);
        if (!STATE_ONLY) {
          tma_load_3d(st, &tmQ, fb, 0, t0, stream);
          tma_load_3d(st + 8192, &tmQ, fb, 64, t0, stream);
        }
        tma_load_3d(st + Q_BYTES, &tmK, fb, 0, t0, stream);
        tma_load_3d(st + Q_BYTES + 8192, &tmK, fb, 64, t0, stream);
        tma_load_3d(st + Q_BYTES + K_BYTES, &tmV, fb, HALF * half, t0, stream);
        if (p.eta)
          bulk_load(st + Q_BYTES + K_BYTES + V_BYTES, p.eta + (size_t)stream * p.T + t0, C * 4,
                    fb);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = umma::idesc_bf16(64, 64, false, false);   // Q K^T
      const uint32_t id_o1 = umma::idesc_bf16(64, 64, false, false);  // Q S
      const uint32_t id_o2 = umma::idesc_bf16(64, 64, false, true);   // P EV
      const uint32_t id_u = umma::idesc_bf16(64, 128, true, true);    // EV^T K
      auto mma_scores = [&](int c) -> bool {
        const int s = c % STAGES, b = c & 1;
        if (!mbar_wait(full + 8 * s, (c / STAGES) & 1, p.err)) return false;
        if (c >= 2 && !mbar_wait(pempty + 8 * b, ((c >> 1) - 1) & 1, p.err)) return false;
        umma::fence_after();
        const uint32_t sQ = sbase + s * STAGE_BYTES, sK = sQ + Q_BYTES;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t o = (ks >> 2) * 8192 + (ks & 3) * 32;
          umma::mma_ss(tmem + TM_P + 64 * b, umma::desc_kmajor(sQ + o), umma::desc_kmajor(sK + o),
                       id_s, ks > 0);
        }
        umma::commit(pfull + 8 * b);
        return true;
      };
      bool ok = true;
      if (!STATE_ONLY) {
        ok = mma_scores(0);
        if (ok && nch > 1) ok = mma_scores(1);
      }
      for (int c = 0; ok && c < nch; ++c) {
        const int s = c % STAGES, b = c & 1;
        const uint32_t sQ = sbase + s * STAGE_BYTES, sK = sQ + Q_BYTES;
        const uint32_t sEV = sbase + EV_OFF + 8192 * b;
        if (STATE_ONLY && !mbar_wait(full + 8 * s, (c / STAGES) & 1, p.err)) break;
        if (!mbar_wait(aready + 8 * b, (c >> 1) & 1, p.err)) break;
        if (!STATE_ONLY && !mbar_wait(sready + 8 * b, (c >> 1) & 1, p.err)) break;
        umma::fence_after();
        // state update first: it heads the serial chain
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          umma::mma_ss(tmem + TM_S, umma::desc_mnmajor(sEV + 2048 * ks, 8192),
                       umma::desc_mnmajor(sK + 2048 * ks, 8192), id_u,
                       STATE_ONLY ? (c > 0 || ks > 0) : true);
        // Pass 2 signals every update (the state warps refresh the bf16 copy); pass 1 only
        // frees the EV tile per chunk and signals the final update.
        if (!STATE_ONLY || c + 1 == nch) umma::commit(sdone);
        if (STATE_ONLY) umma::commit(evfree + 8 * b);
        if (!STATE_ONLY) {
          if (c >= 2 && !mbar_wait(oempty + 8 * b, ((c >> 1) - 1) & 1, p.err)) break;
          umma::fence_after();
          const uint32_t sS = sbase + SB_OFF + 16384 * b, sP = sbase + P_OFF + 8192 * b;
          const uint32_t dO = tmem + TM_O + 64 * b;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t o = (ks >> 2) * 8192 + (ks & 3) * 32;
            umma::mma_ss(dO, umma::desc_kmajor(sQ + o), umma::desc_kmajor(sS + o), id_o1, ks > 0);
          }
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks)
            umma::mma_ss(dO, umma::desc_kmajor(sP + 32 * ks),
                         umma::desc_mnmajor(sEV + 2048 * ks, 8192), id_o2, true);
          umma::commit(ofull + 8 * b);
        }
        umma::commit(empty + 8 * s);
        if (!STATE_ONLY && c + 2 < nch && !mma_scores(c + 2)) break;
      }
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------------- attention warps 2..5
    const int q = warp & 3;
    const int ctid = threadIdx.x - 64;        // 0..127
    const bool rowthr = lane < 16;            // holds an M = 64 accumulator row
    const int r = 16 * q + lane;              // that row (token t of the chunk)
    const uint32_t tl = (uint32_t)(32 * q) << 16;

    // Produce chunk c's operands: masked scores -> P tile, eta * V half -> EV tile.
    auto produce = [&](int c) -> bool {
      const int s = c % STAGES, b = c & 1;
      const uint8_t* stg = smem + s * STAGE_BYTES;
      if (!STATE_ONLY) {
        if (!mbar_wait(pfull + 8 * b, (c >> 1) & 1, p.err)) return false;
        umma::fence_after();
        uint32_t v0[32], v1[32];
        umma::ld32x32(tmem + tl + TM_P + 64 * b, v0);
        umma::ld32x32(tmem + tl + TM_P + 64 * b + 32, v1);
        umma::wait_ld();
        umma::reg_fence(v0);
        umma::reg_fence(v1);
        umma::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pempty + 8 * b);
        if (rowthr) {
          const uint32_t prow = sbase + P_OFF + 8192 * b;
#pragma unroll
          for (int j = 0; j < 64; j += 8) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int sidx = j + e;
              const float x = __uint_as_float(sidx < 32 ? v0[sidx] : v1[sidx - 32]);
              f[e] = sidx <= r ? x : 0.f;
            }
            sts128(prow + swz<128>(r * 128 + 2 * j),
                   make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                              pack_bf16(f[6], f[7])));
          }
        }
      }
      if (!mbar_wait(full + 8 * s, (c / STAGES) & 1, p.err)) return false;
      {
        const uint32_t vt = sbase + s * STAGE_BYTES + Q_BYTES + K_BYTES;
        const uint32_t et = vt + V_BYTES;
        const uint32_t ev = sbase + EV_OFF + 8192 * b;
        // 8192 bytes = 512 x 16-byte pieces; piece i covers row (i / 8), eight columns; the
        // EV tile uses the same swizzled layout as the TMA tile.
        uint4 x[4];
        float e[4];
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int i = ctid + 128 * it;
          x[it] = lds128(vt + swz<128>((i >> 3) * 128 + (i & 7) * 16));
          e[it] = p.eta ? ldsf(et + 4 * (i >> 3)) : p.eta_scalar;
        }
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int i = ctid + 128 * it;
          const float f = e[it];
          sts128(ev + swz<128>((i >> 3) * 128 + (i & 7) * 16),
                 make_uint4(pack_bf16(bf16_lo(x[it].x) * f, bf16_hi(x[it].x) * f),
                            pack_bf16(bf16_lo(x[it].y) * f, bf16_hi(x[it].y) * f),
                            pack_bf16(bf16_lo(x[it].z) * f, bf16_hi(x[it].z) * f),
                            pack_bf16(bf16_lo(x[it].w) * f, bf16_hi(x[it].w) * f)));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(aready + 8 * b);
        mbar_arrive(empty + 8 * s);
      }
      return true;
    };
    // Drain chunk c's outputs: D_O -> bf16 O tile -> TMA store.
    auto consume = [&](int c) -> bool {
      const int b = c & 1;
      if (!mbar_wait(ofull + 8 * b, (c >> 1) & 1, p.err)) return false;
      umma::fence_after();
      uint32_t v0[32], v1[32];
      umma::ld32x32(tmem + tl + TM_O + 64 * b, v0);
      umma::ld32x32(tmem + tl + TM_O + 64 * b + 32, v1);
      umma::wait_ld();
      umma::reg_fence(v0);
      umma::reg_fence(v1);
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(oempty + 8 * b);
      if (rowthr) {
        const uint32_t orow = sbase + O_OFF + 8192 * b;
#pragma unroll
        for (int j = 0; j < 64; j += 8) {
          const uint32_t* vv = j < 32 ? v0 + j : v1 + (j - 32);
          sts128(orow + swz<128>(r * 128 + 2 * j),
                 make_uint4(pack_bf16(__uint_as_float(vv[0]), __uint_as_float(vv[1])),
                            pack_bf16(__uint_as_float(vv[2]), __uint_as_float(vv[3])),
                            pack_bf16(__uint_as_float(vv[4]), __uint_as_float(vv[5])),
                            pack_bf16(__uint_as_float(vv[6]), __uint_as_float(vv[7]))));
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (ctid == 0) {
        tma_store_3d(&tmO, sbase + O_OFF + 8192 * b, HALF * half, tok0 + c * C, stream);
        bulk_commit();
        bulk_wait_read<1>();
      }
      named_bar_sync(1, 128);
      return true;
    };
    // Chunk c+1's operands are produced before chunk c's outputs are drained, so the MMA
    // thread always has the next chunk's P / EV when the state chain allows it to go on.
    // Buffer (c+1) % 2 is free: chunk c-1's MMAs finished before its outputs were drained.
    bool ok = produce(0);
    for (int c = 0; ok && c < nch; ++c) {
      // pass 1 has no outputs to wait for: wait until the update of chunk c-1 released its
      // EV tile instead.
      if (STATE_ONLY && c >= 1 && c + 1 < nch &&
          !mbar_wait(evfree + 8 * ((c + 1) & 1), (((c + 1) >> 1) - 1) & 1, p.err))
        break;
      if (c + 1 < nch && !produce(c + 1)) break;
      if (!STATE_ONLY && !consume(c)) break;
    }
    if (ctid == 0) bulk_wait<0>();
  } else {
    // ---------------------------------------------------------------- state warps 6..9
    const int q = warp & 3;
    const bool rowthr = lane < 16;
    const int r = 16 * q + lane;              // row of S^T[half] = output column index
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int dcol = HALF * half + r;         // global output column of S row r

    // Writes the fp32 state rows in TMEM as the bf16 copy (K-major [64 dout][128 din]).
    auto to_bf16 = [&](int nb) {
      const uint32_t sb = sbase + SB_OFF + 16384 * nb;
      uint32_t v[2][32];
      umma::ld32x32(tmem + tl + TM_S, v[0]);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        umma::wait_ld();
        umma::reg_fence(v[cc & 1]);
        if (cc + 1 < 4) umma::ld32x32(tmem + tl + TM_S + 32 * (cc + 1), v[(cc + 1) & 1]);
        const uint32_t* vv = v[cc & 1];
        if (rowthr) {
          const uint32_t row = sb + (cc >> 1) * 8192;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            const int k = (32 * cc + j) & 63;
            sts128(row + swz<128>(r * 128 + 2 * k),
                   make_uint4(pack_bf16(__uint_as_float(vv[j]), __uint_as_float(vv[j + 1])),
                              pack_bf16(__uint_as_float(vv[j + 2]), __uint_as_float(vv[j + 3])),
                              pack_bf16(__uint_as_float(vv[j + 4]), __uint_as_float(vv[j + 5])),
                              pack_bf16(__uint_as_float(vv[j + 6]), __uint_as_float(vv[j + 7]))));
          }
        }
      }
      fence_proxy_async_smem();
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sready + 8 * nb);
    };

    // Initial state S^T[half] -> TMEM (fp32) and its bf16 copy for chunk 0.
    if (!STATE_ONLY) {
      const float* src = nullptr;
      if (part == 0) src = p.S0 ? p.S0 + (size_t)stream * D * D : nullptr;
      else src = p.S_start + ((size_t)stream * (p.P - 1) + (part - 1)) * D * D;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
          v[j] = __float_as_uint((rowthr && src) ? src[(32 * cc + j) * D + dcol] : 0.f);
        umma::st32x32(tmem + tl + TM_S + 32 * cc, v);
      }
      umma::wait_st();
      to_bf16(0);
    }
    bool ok = true;
    if (STATE_ONLY) {
      ok = mbar_wait(sdone, 0, p.err);
      umma::fence_after();
    } else {
      for (int c = 0; c < nch; ++c) {
        if (!mbar_wait(sdone, c & 1, p.err)) { ok = false; break; }
        umma::fence_after();
        if (c + 1 < nch) to_bf16((c + 1) & 1);
      }
    }
    // ---- final state of the part: increment (pass 1) or S_out (pass 2, last part)
    if (ok && (STATE_ONLY || part == p.P - 1)) {
      float* dst = STATE_ONLY ? p.S_dst + ((size_t)stream * (p.P - 1) + part) * D * D
                              : p.S_dst + (size_t)stream * D * D;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        umma::ld32x32(tmem + tl + TM_S + 32 * cc, v);
        umma::wait_ld();
        umma::reg_fence(v);
        if (rowthr)
#pragma unroll
          for (int j = 0; j < 32; ++j) dst[(32 * cc + j) * D + dcol] = __uint_as_float(v[j]);
      }
    }
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 1) umma::tmem_dealloc(tmem, TM_COLS);
}

// Exclusive prefix over the parts' increments, in place: slot p-1 becomes the start of part p.
__global__ void assoc_scan_kernel(const float* __restrict__ S0, float* inc, int P) {
  const int stream = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;   // element of the d x d state
  if (e >= D * D) return;
  float run = S0 ? S0[(size_t)stream * D * D + e] : 0.f;
  float* base = inc + (size_t)stream * (P - 1) * D * D + e;
  for (int pp = 0; pp < P - 1; ++pp) {
    run += base[(size_t)pp * D * D];
    base[(size_t)pp * D * D] = run;
  }
}

int choose_parts(int streams, int T) {
  const int nchunks = T / C;
  const char* env = getenv("TTT_ASSOC_PARTS");  // tuning override
  if (env) {
    const int f = atoi(env);
    if (f >= 1 && nchunks % f == 0) return f;
  }
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int P = 1;
  while (nchunks % (2 * P) == 0 && streams * 2 * (2 * P) <= sms) P *= 2;
  return P;
}

template <bool STATE_ONLY>
int launch_chunk(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const CUtensorMap& to, const AssocParams& p, int grid, const LaunchCtx& ctx) {
  auto kern = assoc_chunk_kernel<STATE_ONLY>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return kCuda;
  }
  kern<<<grid, THREADS, SMEM, ctx.stream>>>(tq, tk, tv, to, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("assoc launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

bool assoc_supported(int d, int C_, int dt) { return dt == 1 && d == D && C_ == C; }

int launch_assoc_state(const StateArgs& a, const LaunchCtx& ctx) {
  // Pass 1 over the whole sequence as a single superchunk: S_out = sum_t eta_t k_t^T v_t.
  const int BH = a.B * a.H;
  CUtensorMap tq, tk, tv, to;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)a.T * D * 2};
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
  p.T = a.T;
  p.P = 2;             // parts 0 .. P-2 = the single part [0, T)
  p.part_len = a.T;
  p.err = ctx.err;
  return launch_chunk<true>(tq, tk, tv, to, p, BH * 2, ctx);
}

size_t assoc_workspace_bytes(int B, int H, int T, int d, int C_) {
  if (d != D || C_ != C || T % C != 0) return 0;
  const int P = choose_parts(B * H, T);
  return (size_t)B * H * (P - 1) * D * D * sizeof(float);
}

int launch_assoc(const StateArgs& a, const LaunchCtx& ctx) {
  const int BH = a.B * a.H;
  const int P = choose_parts(BH, a.T);
  const size_t need = (size_t)BH * (P - 1) * D * D * sizeof(float);
  if (a.ws_bytes < need) {
    *ctx.msg = "ttt_assoc_scan_fwd: workspace smaller than ttt_assoc_scan_workspace_size()";
    return kWorkspace;
  }
  CUtensorMap tq, tk, tv, to;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)a.T * D * 2};
  const uint32_t box[3] = {64, (uint32_t)C, 1};
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tmap_3d(&tq, a.Q, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tk, a.K, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tv, a.V, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&to, a.O, bf, dims, strides, box, sw, ctx.msg))
    return kCuda;
  AssocParams p;
  p.eta = a.eta;
  p.eta_scalar = a.eta_scalar;
  p.S0 = a.S0;
  p.S_start = static_cast<const float*>(a.ws);
  p.T = a.T;
  p.P = P;
  p.part_len = a.T / P;
  p.err = ctx.err;
  if (P > 1) {
    p.S_dst = static_cast<float*>(a.ws);
    int st = launch_chunk<true>(tq, tk, tv, to, p, BH * (P - 1) * 2, ctx);
    if (st != kOk) return st;
    assoc_scan_kernel<<<dim3(D * D / 256, BH), 256, 0, ctx.stream>>>(a.S0, p.S_dst, P);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      *ctx.msg = std::string("assoc scan launch: ") + cudaGetErrorString(e);
      return kCuda;
    }
    count_launch();
  }
  p.S_dst = a.S_out;
  return launch_chunk<false>(tq, tk, tv, to, p, BH * P * 2, ctx);
}

}  // namespace ttt
