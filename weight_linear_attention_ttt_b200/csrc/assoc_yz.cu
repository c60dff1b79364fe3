// Backward of the associative mode: the two reverse-order outputs Y and Z in one pass.
//
// Source: "KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다" (associativity paragraph): with
// S_t = S_(t-1) + eta_t k_t^T v_t and o_t = q_t S_t, the gradient with respect to S_t is
// A_t = dS_out + sum_{u >= t} q_u^T dO_u, and
//     Y_t = k_t A_t   = k_t A' + sum_{u >= t, u in the chunk} (k_t . q_u) dO_u
//     Z_t = v_t A_t^T = v_t A'^T + sum_{u >= t, u in the chunk} (v_t . dO_u) q_u
// with A' the gradient after the chunk (walking the chunks from the last). dV = eta Y (a later
// elementwise pass, which also forms deta = Y . v), dK = eta Z (here), dS0 = A_0.
// The separate form runs Y and Z as two reverse associative scans; both carry the same state A
// (as A and A^T), so one pass reads Q, K, V and dO once and writes both.
//
// Products per 64-token chunk (M side = 128 feature rows on the TMEM lanes):
//     Y^T = A'^T K^T + dO^T P1^T,   P1[t][u] = [u >= t] (k_t . q_u)
//     Z^T = A'   V^T + Q^T  P2^T,   P2[t][u] = [u >= t] (v_t . dO_u)
//     A  += Q^T dO
// A is fp32 in TMEM (rows i on the lanes); its bf16 copy for the products lives in shared memory
// as [128 rows i][128 columns j] in two 128-byte-swizzled [128][64] blocks, which serves A'^T as
// an MN-major operand (Y) and A' as a K-major operand (Z). TMEM: A [0,128), Y^T x2 [128,256),
// Z^T x2 [256,384), scores P1 [384,448), P2 [448,512) (M = 64).
//
// Warps: 0 TMA (2-stage ring of Q/K/V/dO tiles); 1 MMA issue; 2-5 scores -> masked bf16 P1, P2;
// 6-9 state refresh (A -> bf16 copy); 10-13 Y -> dV (unscaled); 14-17 eta Z -> dK (each group
// drains its accumulator through a shared tile to TMA stores).
// The serial chain per chunk is refresh -> products and update -> refresh.
#include <algorithm>
#include <string>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int YD = 128;                 // feature tile (d = 64 runs zero-padded)
constexpr int YC = 64;                  // tokens per chunk
constexpr int YT = YC * YD * 2;         // one [64][128] bf16 tile (two [64][64] sub-tiles)
constexpr int Y_STAGES = 2;
constexpr int Y_Q = 0, Y_K = YT, Y_V = 2 * YT, Y_DO = 3 * YT;
constexpr int Y_STAGE = 4 * YT;
constexpr int Y_A = Y_STAGES * Y_STAGE;            // bf16 A: two [128][64] blocks
constexpr int Y_P1 = Y_A + 2 * YD * 64 * 2;        // [64 t][64 u] bf16
constexpr int Y_P2 = Y_P1 + YC * YC * 2;
constexpr int Y_OY = Y_P2 + YC * YC * 2;           // output staging [64 t][128] bf16
constexpr int Y_OZ = Y_OY + YT;
constexpr int Y_BAR = Y_OZ + YT;
constexpr int Y_SMEM = 1024 + Y_BAR + 512;   // barriers, then the Z group's rate table
constexpr int Y_THREADS = 18 * 32;
static_assert(Y_SMEM <= 227 * 1024, "shared memory");
constexpr uint32_t TY_A = 0, TY_Y = 128, TY_Z = 256, TY_P1 = 384, TY_P2 = 448;

struct YzParams {
  const float* eta;       // [BH, T] rates for dK = eta Z, or null (eta_scalar)
  float eta_scalar;
  const float* dS_out;    // the caller's [dim][dim] gradient of the final state, or null
  const float* start;     // [BH, nslots, D, D] reverse prefix of the pass-1 pieces, or null
  float* dS0;             // [BH, dim, dim], written by the part that ends at token 0
  int T, P, part_len, nslots, slot_mul, dim;
  unsigned* err;
};

__global__ void __launch_bounds__(Y_THREADS, 1)
    assoc_yz_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmD,
                    const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmZ,
                    const YzParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + Y_BAR;
  const uint32_t full = bar, empty = bar + 16;   // stage ring (x2)
  const uint32_t sfull = bar + 32;               // scores of a chunk in TMEM (MMA commit)
  const uint32_t pready = bar + 48;              // P1, P2 tiles written (4 operand warps)
  const uint32_t sready = bar + 56;              // bf16 copy of A refreshed (4 state warps)
  const uint32_t cdone = bar + 64;               // products and update of a chunk done (x2)
  const uint32_t ofree = bar + 80;               // Y^T, Z^T buffer read out (x2, 8 warps)
  const uint32_t mdone = bar + 96;
  const uint32_t tslot = bar + 104;
  const uint32_t sA = sbase + Y_A;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stream = blockIdx.x / p.P, part = blockIdx.x % p.P;
  const int tok0 = part * p.part_len;
  const int nch = p.part_len / YC;
  // first token of the c-th chunk processed (the sequence is walked from its end; part 0 is the
  // last superchunk)
  auto tok = [&](int c) { return p.T - YC - (tok0 + c * YC); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < Y_STAGES; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    mbar_init(sfull, 1);
    mbar_init(pready, 4);
    mbar_init(sready, 4);
    for (int b = 0; b < 2; ++b) {
      mbar_init(cdone + 8 * b, 1);
      mbar_init(ofree + 8 * b, 8);
    }
    mbar_init(mdone, 1);
    fence_mbar_init();
  }
  if (warp == 1) umma::tmem_alloc(tslot, 512);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Y_BAR + 104);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmD);
      int issued = 0;
      for (int c = 0; c < nch; ++c) {
        const int s = c % Y_STAGES;
        if (c >= Y_STAGES && !mbar_wait(empty + 8 * s, ((c / Y_STAGES) - 1) & 1, p.err)) break;
        const uint32_t fb = full + 8 * s;
        const uint32_t st = sbase + s * Y_STAGE;
        const int t0 = tok(c);
        mbar_arrive_expect_tx(fb, Y_STAGE);
        tma_load_3d(st + Y_Q, &tmQ, fb, 0, t0, stream);
        tma_load_3d(st + Y_Q + 8192, &tmQ, fb, 64, t0, stream);
        tma_load_3d(st + Y_K, &tmK, fb, 0, t0, stream);
        tma_load_3d(st + Y_K + 8192, &tmK, fb, 64, t0, stream);
        tma_load_3d(st + Y_V, &tmV, fb, 0, t0, stream);
        tma_load_3d(st + Y_V + 8192, &tmV, fb, 64, t0, stream);
        tma_load_3d(st + Y_DO, &tmD, fb, 0, t0, stream);
        tma_load_3d(st + Y_DO + 8192, &tmD, fb, 64, t0, stream);
        issued = c + 1;
      }
      // copies still in flight land before the CTA may exit (normally all have)
      for (int c = std::max(0, issued - Y_STAGES); c < issued; ++c)
        mbar_wait(full + 8 * (c % Y_STAGES), (c / Y_STAGES) & 1, p.err, 1000000000ull);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA warp
    const uint32_t id_s = umma::idesc_bf16(64, 64, false, false);    // scores, M = 64 tokens
    const uint32_t id_ym = umma::idesc_bf16(128, 64, true, false);   // MN-major A, K-major B
    const uint32_t id_yk = umma::idesc_bf16(128, 64, false, false);  // K-major A and B
    const uint32_t id_u = umma::idesc_bf16(128, 128, true, true);    // Q^T dO
    // scores of chunk c: P1 = K Q^T, P2 = V dO^T
    auto issue_scores = [&](int c) -> bool {
      const int s = c % Y_STAGES;
      if (!mbar_wait_warp(full + 8 * s, (c / Y_STAGES) & 1, p.err)) return false;
      umma::fence_after();
      const uint32_t st = sbase + s * Y_STAGE;
#pragma unroll
      for (int ks = 0; ks < YD / 16; ++ks) {
        const uint32_t o = (ks >> 2) * 8192 + (ks & 3) * 32;
        umma::mma_ss_elect(tmem + TY_P1, umma::desc_kmajor(st + Y_K + o),
                           umma::desc_kmajor(st + Y_Q + o), id_s, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < YD / 16; ++ks) {
        const uint32_t o = (ks >> 2) * 8192 + (ks & 3) * 32;
        umma::mma_ss_elect(tmem + TY_P2, umma::desc_kmajor(st + Y_V + o),
                           umma::desc_kmajor(st + Y_DO + o), id_s, ks > 0);
      }
      umma::commit_elect(sfull);
      return true;
    };
    bool ok = nch > 0 ? issue_scores(0) : true;
    for (int c = 0; ok && c < nch; ++c) {
      const int s = c % Y_STAGES, b = c & 1;
      const uint32_t st = sbase + s * Y_STAGE;
      if (!mbar_wait_warp(sready, c & 1, p.err)) break;           // A' in shared memory
      if (!mbar_wait_warp(pready, c & 1, p.err)) break;           // P1, P2 of chunk c
      if (c >= 2 && !mbar_wait_warp(ofree + 8 * b, ((c >> 1) - 1) & 1, p.err)) break;
      umma::fence_after();
      const uint32_t dY = tmem + TY_Y + 64 * b, dZ = tmem + TY_Z + 64 * b;
      // Y^T = A'^T K^T + dO^T P1^T
#pragma unroll
      for (int ks = 0; ks < YD / 16; ++ks)
        umma::mma_ss_elect(dY, umma::desc_mnmajor(sA + 2048 * ks, 16384),
                           umma::desc_kmajor(st + Y_K + (ks >> 2) * 8192 + (ks & 3) * 32), id_ym,
                           ks > 0);
#pragma unroll
      for (int ks = 0; ks < YC / 16; ++ks)
        umma::mma_ss_elect(dY, umma::desc_mnmajor(st + Y_DO + 2048 * ks, 8192),
                           umma::desc_kmajor(sbase + Y_P1 + 32 * ks), id_ym, true);
      // Z^T = A' V^T + Q^T P2^T
#pragma unroll
      for (int ks = 0; ks < YD / 16; ++ks)
        umma::mma_ss_elect(dZ, umma::desc_kmajor(sA + (ks >> 2) * 16384 + (ks & 3) * 32),
                           umma::desc_kmajor(st + Y_V + (ks >> 2) * 8192 + (ks & 3) * 32), id_yk,
                           ks > 0);
#pragma unroll
      for (int ks = 0; ks < YC / 16; ++ks)
        umma::mma_ss_elect(dZ, umma::desc_mnmajor(st + Y_Q + 2048 * ks, 8192),
                           umma::desc_kmajor(sbase + Y_P2 + 32 * ks), id_ym, true);
      // A += Q^T dO
#pragma unroll
      for (int ks = 0; ks < YC / 16; ++ks)
        umma::mma_ss_elect(tmem + TY_A, umma::desc_mnmajor(st + Y_Q + 2048 * ks, 8192),
                           umma::desc_mnmajor(st + Y_DO + 2048 * ks, 8192), id_u, true);
      umma::commit_elect(cdone + 8 * b);
      umma::commit_elect(empty + 8 * s);
      // the scores of chunk c+1 (the score warps have read those of chunk c: pready(c))
      if (c + 1 < nch) ok = issue_scores(c + 1);
    }
    umma::commit_elect(mdone);
    mbar_wait_warp(mdone, 0, p.err, 1000000000ull);
  } else if (warp < 6) {
    // ---------------------------------------------------------------- score warps 2..5
    const int q = warp & 3;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int r = 16 * q + lane;              // token row of the M = 64 scores (lanes < 16)
    for (int c = 0; c < nch; ++c) {
      // the scores of chunk c are issued after the products of chunk c-1, so waiting for those
      // (which frees the P tiles) costs nothing
      if (c >= 1 && !mbar_wait_warp(cdone + 8 * ((c - 1) & 1), ((c - 1) >> 1) & 1, p.err)) break;
      if (!mbar_wait_warp(sfull, c & 1, p.err)) break;
      umma::fence_after();
      // masked rows (keys u >= t in the reversed order) as bf16 pairs into the K-major tiles
#pragma unroll
      for (int m = 0; m < 2; ++m) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[32];
          umma::ld32x32(tmem + tl + (m ? TY_P2 : TY_P1) + 32 * h, v);
          umma::wait_ld();
          umma::reg_fence(v);
          if (lane < 16) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int u = 32 * h + 8 * k + 2 * e;
                const float x0 = u >= r ? __uint_as_float(v[8 * k + 2 * e]) : 0.f;
                const float x1 = u + 1 >= r ? __uint_as_float(v[8 * k + 2 * e + 1]) : 0.f;
                w[e] = pack_bf16(x0, x1);
              }
              sts128(sbase + (m ? Y_P2 : Y_P1) + swz<128>(r * 128 + 64 * h + 16 * k),
                     make_uint4(w[0], w[1], w[2], w[3]));
            }
          }
        }
      }
      umma::fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(pready);
    }
  } else if (warp < 10) {
    // ---------------------------------------------------------------- state warps 6..9
    const int q = warp & 3;
    const int i = 32 * q + lane;              // row of A
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    // bf16 copy of A's row i, columns j0 .. j0 + 31 (two [128][64] swizzled blocks)
    auto put_copy = [&](int j0, const uint32_t (&v)[32]) {
      const uint32_t rowb = sA + (j0 >> 6) * 16384;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        sts128(rowb + swz<128>(i * 128 + (j0 & 63) * 2 + 16 * k),
               make_uint4(pack_bf16(__uint_as_float(v[8 * k]), __uint_as_float(v[8 * k + 1])),
                          pack_bf16(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3])),
                          pack_bf16(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5])),
                          pack_bf16(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7]))));
    };
    bool ok = true;
    for (int c = 0; c < nch; ++c) {
      if (c == 0) {
        // the part's starting gradient: the caller's dS_out (part 0, the last superchunk) or
        // the reverse prefix of the later superchunks
        const float* src = nullptr;
        int ld = YD;
        bool in = true;
        if (p.start && part > 0) {
          src = p.start + ((size_t)stream * p.nslots + (size_t)part * p.slot_mul - 1) * YD * YD;
        } else if (p.dS_out) {
          src = p.dS_out + (size_t)stream * p.dim * p.dim;
          ld = p.dim;
          in = i < p.dim;
        }
#pragma unroll 1
        for (int pc = 0; pc < 4; ++pc) {
          const int j0 = 32 * pc;
          uint32_t v[32];
          const bool ok_j = in && src && (ld == YD || j0 < p.dim);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            v[j] = __float_as_uint(ok_j ? src[(size_t)i * ld + j0 + j] : 0.f);
          umma::st32x32(tmem + tl + TY_A + j0, v);
          put_copy(j0, v);
        }
        umma::wait_st();
      } else {
        // the update of chunk c-1 is in A, and its products have read the previous copy
        if (!mbar_wait_warp(cdone + 8 * ((c - 1) & 1), ((c - 1) >> 1) & 1, p.err)) {
          ok = false;
          break;
        }
        umma::fence_after();
#pragma unroll 1
        for (int pc = 0; pc < 4; ++pc) {
          uint32_t v[32];
          umma::ld32x32(tmem + tl + TY_A + 32 * pc, v);
          umma::wait_ld();
          umma::reg_fence(v);
          put_copy(32 * pc, v);
        }
      }
      fence_proxy_async_smem();
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sready);
    }
    // dS0: the gradient after the whole sequence, from the part that ends at token 0
    if (ok && nch > 0 && part == p.P - 1 &&
        mbar_wait_warp(cdone + 8 * ((nch - 1) & 1), ((nch - 1) >> 1) & 1, p.err)) {
      umma::fence_after();
      float* dst = p.dS0 + (size_t)stream * p.dim * p.dim;
#pragma unroll 1
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t v[32];
        umma::ld32x32(tmem + tl + TY_A + 32 * pc, v);
        umma::wait_ld();
        umma::reg_fence(v);
        if (i < p.dim && 32 * pc < p.dim) {
#pragma unroll
          for (int j = 0; j < 32; ++j) dst[(size_t)i * p.dim + 32 * pc + j] = __uint_as_float(v[j]);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- output warps 10..17
    const bool zg = warp >= 14;                // warps 14..17 drain Z^T, 10..13 Y^T
    const int q = warp & 3;
    const int row = 32 * q + lane;             // feature: j of Y^T, i of Z^T
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int gtid = threadIdx.x - (zg ? 448 : 320);   // 0..127 within the group
    const int gbar = zg ? 2 : 1;               // the group's named barrier
    const bool odd = lane & 1;
    const uint32_t ocol = (row >> 6) * 8192;
    const uint32_t cb = 2 * ((row & 63) & ~1);
    const uint32_t tile = sbase + (zg ? Y_OZ : Y_OY);
    const uint32_t acc = tmem + tl + (zg ? TY_Z : TY_Y);
    for (int c = 0; c < nch; ++c) {
      const int b = c & 1;
      // Z group: the chunk's 64 rates, loaded before the wait so that their latency hides there
      float4 e4 = make_float4(p.eta_scalar, p.eta_scalar, p.eta_scalar, p.eta_scalar);
      if (zg && p.eta && gtid < 16)
        e4 = __ldg(reinterpret_cast<const float4*>(p.eta + (size_t)stream * p.T + tok(c)) + gtid);
      const bool got = mbar_wait_warp(cdone + 8 * b, (c >> 1) & 1, p.err);
      if (bar_or_named(gbar, 128, !got)) break;
      umma::fence_after();
      const uint32_t etab = sbase + Y_BAR + 256;   // the Z group's rates of the chunk
      if (zg && gtid < 16)
        sts128(etab + 16 * gtid, make_uint4(__float_as_uint(e4.x), __float_as_uint(e4.y),
                                            __float_as_uint(e4.z), __float_as_uint(e4.w)));
      // the previous chunk's store has read the staging tile (and the rates are in place)
      if (gtid == 0) bulk_wait_read<0>();
      bar_sync_named(gbar, 128);
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {   // tokens 32 hf .. 32 hf + 31
        uint32_t v[32];
        umma::ld32x32(acc + 64 * b + 32 * hf, v);
        umma::wait_ld();
        umma::reg_fence(v);
        if (hf == 1) {   // this warp's part of buffer b is read out
          umma::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(ofree + 8 * b);
        }
        if (zg) {
          // dK = eta Z: token t is column t of Z^T
#pragma unroll
          for (int t = 0; t < 32; t += 4) {
            const uint4 e = lds128(etab + 4 * (32 * hf + t));
            v[t] = __float_as_uint(__uint_as_float(e.x) * __uint_as_float(v[t]));
            v[t + 1] = __float_as_uint(__uint_as_float(e.y) * __uint_as_float(v[t + 1]));
            v[t + 2] = __float_as_uint(__uint_as_float(e.z) * __uint_as_float(v[t + 2]));
            v[t + 3] = __float_as_uint(__uint_as_float(e.w) * __uint_as_float(v[t + 3]));
          }
        }
        // Lane pairs (2i, 2i+1) exchange one value per token pair (t, t+4) so that each lane
        // stores a 32-bit word of two adjacent output columns: the even lane row t, the odd
        // lane row t+4.
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          if (t & 4) continue;
          const float a = __uint_as_float(v[t]), a4 = __uint_as_float(v[t + 4]);
          const float y = __shfl_xor_sync(0xffffffffu, odd ? a : a4, 1);
          const float lo = odd ? y : a, hi = odd ? a4 : y;
          sts32(tile + ocol + swz<128>((32 * hf + (odd ? t + 4 : t)) * 128 + cb),
                pack_bf16(lo, hi));
        }
      }
      fence_proxy_async_smem();
      bar_sync_named(gbar, 128);
      if (gtid == 0) {
        const int t0 = tok(c);
        const CUtensorMap* tm = zg ? &tmZ : &tmY;
        tma_store_3d(tm, tile, 0, t0, stream);
        if (p.dim > 64) tma_store_3d(tm, tile + 8192, 64, t0, stream);
        bulk_commit();
      }
    }
    if (gtid == 0) bulk_wait<0>();
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 1) umma::tmem_dealloc(tmem, 512);
}

}  // namespace

int launch_assoc_yz(const AssocBwdArgs& a, void* ws, size_t ws_bytes, const LaunchCtx& ctx) {
  // the reverse prefix of A = dS_out + sum q^T dO over superchunks: the associative scan's
  // pass 1 and prefix with keys Q and values dO, walked from the end
  StateArgs y{a.K, a.Q, a.dO, nullptr, 1.0f, a.dS_out, nullptr, nullptr, a.B, a.H, a.T, a.d,
              a.C, 1, ws, ws_bytes};
  y.reverse = 1;
  AssocPrefix pre;
  int st = launch_assoc_prefix(y, &pre, ctx);
  if (st != kOk) return st;
  const int BH = a.B * a.H;
  CUtensorMap tq, tk, tv, td, ty, tz;
  const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)a.T, (uint64_t)BH};
  const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)a.T * a.d * 2};
  const uint32_t box[3] = {64, (uint32_t)YC, 1};
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tmap_3d(&tq, a.Q, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tk, a.K, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tv, a.V, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&td, a.dO, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&ty, a.dV, bf, dims, strides, box, sw, ctx.msg) ||
      !make_tmap_3d(&tz, a.dK, bf, dims, strides, box, sw, ctx.msg))
    return kCuda;
  YzParams p;
  p.eta = a.eta;
  p.eta_scalar = a.eta_scalar;
  p.dS_out = a.dS_out;
  p.start = pre.P > 1 ? pre.slots : nullptr;
  p.dS0 = a.dS0;
  p.T = a.T;
  p.P = pre.P;
  p.part_len = a.T / pre.P;
  p.nslots = pre.nslots;
  p.slot_mul = pre.slot_mul;
  p.dim = a.d;
  p.err = ctx.err;
  cudaError_t e = cudaFuncSetAttribute(assoc_yz_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Y_SMEM);
  if (e == cudaSuccess) {
    assoc_yz_kernel<<<BH * pre.P, Y_THREADS, Y_SMEM, ctx.stream>>>(tq, tk, tv, td, ty, tz, p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    *ctx.msg = std::string("assoc bwd Y/Z launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace ttt
