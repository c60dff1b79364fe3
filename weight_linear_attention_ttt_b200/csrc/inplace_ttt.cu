// In-Place TTT W_down chunk update on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Source: "In-Place Test-Time Training" (aitrends.kr): W_down of the gated MLP is the fast
// weight; the sequence is cut into chunks; each chunk takes one gradient step on W_down, and the
// updated weight serves the next chunk; per-chunk deltas combine by a prefix sum.
//     W = W0;  for chunk i:  O_i = Z_i W;  W = W + eta Z_i^T Vhat_i
//
// Design. Within chunk i the read O_i = Z_i W_(i-1) and the update W_i = W_(i-1) + eta Z_i^T
// Vhat_i are independent, so one persistent kernel per chunk runs both as tiles of one tile
// list: 128x256 read tiles (K = Dff) and 128x256 update tiles (K = C). Read tiles are long, so
// they are scheduled first, and every CTA takes the next tile from a global atomic counter.
// The fp32 master W lives in W_out; the tensor cores read a bf16 copy of W, kept in a
// double-buffered workspace (the update of chunk i writes copy i % 2 while the read of chunk i
// still reads copy (i-1) % 2; chunk 0 reads the bf16 W0 input directly).
// Warp roles per CTA: warp 0 issues TMA loads into a 4-stage shared-memory ring and fetches
// tiles from the counter; warp 1 owns TMEM and issues tcgen05.mma from one thread into one of
// two TMEM accumulators; warps 2-5 drain the other accumulator: bf16 O for read tiles,
// W_out = W + eta * acc (fp32) and its bf16 copy for update tiles.
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int BM = 128;     // tile rows (tokens for read tiles, Dff rows for update tiles)
constexpr int BK = 64;      // K per pipeline stage
constexpr int STAGES = 4;
constexpr int THREADS = 192;

template <int BN>
struct IpCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BK * BN * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // epilogue staging, per 16-column piece of a tile: 2 x [128 rows][16 fp32] (the running W,
  // loaded and stored in place) and 2 x [128 rows][16 bf16] (O or the bf16 copy of W)
  static constexpr int WST_OFF = STAGES * STAGE_BYTES;
  static constexpr int HST_OFF = WST_OFF + 2 * 8192;
  static constexpr int BAR_OFF = HST_OFF + 2 * 4096;
  static constexpr int SMEM = 1024 + BAR_OFF + 256;
  static constexpr int TMEM_COLS = 2 * BN;
};

struct IpParams {
  const __nv_bfloat16* W0;   // [Dff, D] bf16 (source of chunk 0's update)
  float* Wout;               // [Dff, D] fp32 running master
  __nv_bfloat16* Wbf_next;   // [Dff, D] bf16 copy written by this launch's update (or null)
  __nv_bfloat16* O;          // [T, D]
  float eta;
  int first;                 // the launch holds chunk 0: the update reads W0
  int tok0;                  // first token of the launch's (first) chunk
  int C, Dff, D;
  int pair;                  // 1: the launch covers chunks i and i+1 (see the tile list below)
  int n_p;                   // pair launches: tiles of eta Z_(i+1) Z_i^T
  int n_read;                // read tiles per chunk
  int n_total;
  int* counter;
  int* pdone;                // pair launches: finished eta Z Z^T tiles per 128-row block
  unsigned* err;
};

// Tile list of a launch, in the order the global counter hands it out:
//   single chunk:  read tiles of the chunk (K = Dff), update tiles (K = C);
//   chunk pair:    tiles of Pc = eta Z_(i+1) Z_i^T (C x C, K = Dff, stored bf16 in the
//                  workspace), read tiles of chunk i+1 (K = Dff from Z_(i+1) and the bf16 W_(i-1),
//                  then K = C from Pc and Vhat_i: the exact correction for chunk i's update, which
//                  chunk i+1 must see), read tiles of chunk i, update tiles over both chunks
//                  (K = 2C: W_(i+1) = W_(i-1) + eta [Z_i; Z_(i+1)]^T [Vhat_i; Vhat_(i+1)]).
// The fp32 master is then read and written once per pair. A read tile of chunk i+1 waits for
// its row block of Pc only after its K = Dff part; Pc tiles come first in the list.
enum TileKind : int { kRead = 0, kUpdate = 1, kPc = 2, kReadNext = 3 };
struct Tile {
  int kind, mt, nt, nkb;
};
template <int BN>
__device__ __forceinline__ Tile decode_tile(const IpParams& p, int t) {
  const int ntn = p.D / BN;
  Tile x;
  if (p.pair && t < p.n_p) {
    const int per = p.C / BN;
    x.kind = kPc, x.mt = t / per, x.nt = t % per, x.nkb = p.Dff / BK;
    return x;
  }
  int u = t - (p.pair ? p.n_p : 0);
  if (p.pair && u < p.n_read) {
    x.kind = kReadNext, x.mt = u / ntn, x.nt = u % ntn, x.nkb = (p.Dff + p.C) / BK;
    return x;
  }
  if (p.pair) u -= p.n_read;
  if (u < p.n_read) {
    x.kind = kRead, x.mt = u / ntn, x.nt = u % ntn, x.nkb = p.Dff / BK;
    return x;
  }
  u -= p.n_read;
  x.kind = kUpdate, x.mt = u / ntn, x.nt = u % ntn, x.nkb = (p.pair ? 2 * p.C : p.C) / BK;
  return x;
}
__device__ __forceinline__ int ld_acquire_gpu(const int* ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(int* ptr, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          tmap),
      "r"(src), "r"(c0), "r"(c1)
      : "memory");
}

template <int BN>
__global__ void __launch_bounds__(THREADS, 1)
    inplace_chunk_kernel(const __grid_constant__ CUtensorMap tmZk,   // Z, box 64 x 128
                         const __grid_constant__ CUtensorMap tmZm,   // Z, box 64 x 64
                         const __grid_constant__ CUtensorMap tmW,    // bf16 W read source
                         const __grid_constant__ CUtensorMap tmV,    // Vhat, box 64 x 64
                         const __grid_constant__ CUtensorMap tmWf,   // W_out fp32, box 16 x 128
                         const __grid_constant__ CUtensorMap tmO,    // O bf16, box 16 x 128
                         const __grid_constant__ CUtensorMap tmWb,   // next bf16 W, box 16 x 128
                         const __grid_constant__ CUtensorMap tmPl,   // Pc, box 64 x 128 (loads)
                         const __grid_constant__ CUtensorMap tmPs,   // Pc, box 16 x 128 (stores)
                         const IpParams p) {
  using Cfg = IpCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + Cfg::BAR_OFF;
  const uint32_t full = bar, empty = bar + 8 * STAGES;
  const uint32_t tfull = bar + 16 * STAGES, tempty = tfull + 16;
  const uint32_t sfull = tempty + 16, sempty = sfull + 16;
  const uint32_t tslot = sempty + 16;                  // TMEM base address
  const uint32_t wfull = tslot + 32;                   // W staging buffers loaded (x2)
  volatile int* sched = reinterpret_cast<volatile int*>(smem + Cfg::BAR_OFF + 16 * STAGES + 80);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + 8 * b, 1);
      mbar_init(tempty + 8 * b, 4);
      mbar_init(sfull + 8 * b, 1);
      mbar_init(sempty + 8 * b, 5);
      mbar_init(wfull + 8 * b, 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) umma::tmem_alloc(tslot, Cfg::TMEM_COLS);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Cfg::BAR_OFF + 16 * STAGES +
                                                              64);

  if (warp == 0) {
    // ------------------------------------------------------------ scheduler + TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmZk);
      prefetch_tmap(&tmZm);
      prefetch_tmap(&tmW);
      prefetch_tmap(&tmV);
      uint32_t kbt = 0;
      for (int j = 0;; ++j) {
        const int slot = j & 1;
        if (j >= 2 && !mbar_wait(sempty + 8 * slot, ((j >> 1) - 1) & 1, p.err)) break;
        const int t = atomicAdd(p.counter, 1);
        sched[slot] = t;
        mbar_arrive(sfull + 8 * slot);
        if (t >= p.n_total) break;
        const Tile x = decode_tile<BN>(p, t);
        const int kbz = p.Dff / BK;   // k-blocks over Dff
        const int rows = x.kind == kReadNext ? p.tok0 + p.C + BM * x.mt : p.tok0 + BM * x.mt;
        bool ok = true;
        for (int kb = 0; kb < x.nkb; ++kb, ++kbt) {
          const int s = kbt % STAGES;
          if (kbt >= STAGES && !mbar_wait(empty + 8 * s, ((kbt / STAGES) - 1) & 1, p.err)) {
            ok = false;
            break;
          }
          if (x.kind == kReadNext && kb == kbz) {
            // the correction part needs this row block of Pc, written by other CTAs' TMA stores:
            // wait (bounded) for its tiles' release, then order the loads after it
            const uint64_t t0 = global_timer_ns();
            while (ld_acquire_gpu(p.pdone + x.mt) < p.C / BN) {
              if (global_timer_ns() - t0 > 4000000000ull) {
                raise_device_error(p.err, kErrWaitTimeout);
                break;
              }
              __nanosleep(256);
            }
            fence_proxy_async_global();
          }
          const uint32_t fb = full + 8 * s;
          const uint32_t sA = sbase + s * Cfg::STAGE_BYTES, sB = sA + Cfg::A_BYTES;
          mbar_arrive_expect_tx(fb, Cfg::STAGE_BYTES);
          if (x.kind == kPc) {
            // A = Z_(i+1) rows, B = Z_i rows (K-major, N = 256 tokens of chunk i)
            tma_load_2d(sA, &tmZk, fb, kb * BK, p.tok0 + p.C + BM * x.mt);
            tma_load_2d(sB, &tmZk, fb, kb * BK, p.tok0 + BN * x.nt);
            tma_load_2d(sB + 16384, &tmZk, fb, kb * BK, p.tok0 + BN * x.nt + 128);
          } else if (x.kind == kRead || (x.kind == kReadNext && kb < kbz)) {
            tma_load_2d(sA, &tmZk, fb, kb * BK, rows);
#pragma unroll
            for (int nb = 0; nb < BN / 64; ++nb)
              tma_load_2d(sB + nb * 8192, &tmW, fb, BN * x.nt + 64 * nb, kb * BK);
          } else if (x.kind == kReadNext) {
            // A = Pc rows of chunk i+1, B = Vhat_i (MN-major, like the update's B)
            const int k2 = kb - kbz;
            tma_load_2d(sA, &tmPl, fb, k2 * BK, BM * x.mt);
#pragma unroll
            for (int nb = 0; nb < BN / 64; ++nb)
              tma_load_2d(sB + nb * 8192, &tmV, fb, BN * x.nt + 64 * nb, p.tok0 + k2 * BK);
          } else {
#pragma unroll
            for (int mb = 0; mb < 2; ++mb)
              tma_load_2d(sA + mb * 8192, &tmZm, fb, BM * x.mt + 64 * mb, p.tok0 + kb * BK);
#pragma unroll
            for (int nb = 0; nb < BN / 64; ++nb)
              tma_load_2d(sB + nb * 8192, &tmV, fb, BN * x.nt + 64 * nb, p.tok0 + kb * BK);
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      const uint32_t idesc_rd = umma::idesc_bf16(BM, BN, false, true);
      const uint32_t idesc_up = umma::idesc_bf16(BM, BN, true, true);
      const uint32_t idesc_pc = umma::idesc_bf16(BM, BN, false, false);
      uint32_t kbt = 0;
      for (int j = 0;; ++j) {
        const int slot = j & 1;
        if (!mbar_wait(sfull + 8 * slot, (j >> 1) & 1, p.err)) break;
        const int t = sched[slot];
        mbar_arrive(sempty + 8 * slot);
        if (t >= p.n_total) break;
        const Tile x = decode_tile<BN>(p, t);
        const int b = j & 1;
        if (j >= 2 && !mbar_wait(tempty + 8 * b, ((j >> 1) - 1) & 1, p.err)) break;
        umma::fence_after();
        const uint32_t dt = tmem + b * BN;
        bool ok = true;
        for (int kb = 0; kb < x.nkb; ++kb, ++kbt) {
          const int s = kbt % STAGES;
          if (!mbar_wait(full + 8 * s, (kbt / STAGES) & 1, p.err)) {
            ok = false;
            break;
          }
          umma::fence_after();
          const uint32_t sA = sbase + s * Cfg::STAGE_BYTES, sB = sA + Cfg::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            uint64_t ad, bd;
            uint32_t id;
            if (x.kind == kUpdate) {
              ad = umma::desc_mnmajor(sA + 2048 * ks, 8192);
              bd = umma::desc_mnmajor(sB + 2048 * ks, 8192);
              id = idesc_up;
            } else if (x.kind == kPc) {
              ad = umma::desc_kmajor(sA + 32 * ks);
              bd = umma::desc_kmajor(sB + 32 * ks);
              id = idesc_pc;
            } else {
              ad = umma::desc_kmajor(sA + 32 * ks);
              bd = umma::desc_mnmajor(sB + 2048 * ks, 8192);
              id = idesc_rd;
            }
            umma::mma_ss(dt, ad, bd, id, kb > 0 || ks > 0);
          }
          umma::commit(empty + 8 * s);
        }
        if (!ok) break;
        umma::commit(tfull + 8 * b);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2..5
    // A tile leaves in 16-column pieces through shared staging tiles and TMA stores (a thread
    // owns one row of the accumulator, so direct global stores would scatter one row segment
    // per thread). Update tiles read the running fp32 W by TMA into the fp32 staging tile two
    // pieces ahead, add eta * acc in place and store the tile back, with its bf16 copy; the
    // first chunk's update reads the bf16 W0 directly.
    const int q = warp & 3;  // TMEM subpartition this warp may read
    const int row = 32 * q + lane;
    const int ctid = threadIdx.x - 64;
    constexpr int NCC = BN / 16;
    uint32_t ec = 0;             // pieces processed so far: piece e uses staging buffers e & 1
    uint32_t nld[2] = {0u, 0u};  // W loads consumed per fp32 staging buffer (their phases)
    auto fbuf = [&](uint32_t e) { return sbase + Cfg::WST_OFF + 8192 * (e & 1); };
    auto hbuf = [&](uint32_t e) { return sbase + Cfg::HST_OFF + 4096 * (e & 1); };
    for (int j = 0;; ++j) {
      const int slot = j & 1;
      if (!mbar_wait(sfull + 8 * slot, (j >> 1) & 1, p.err)) break;
      const int t = sched[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty + 8 * slot);
      if (t >= p.n_total) break;
      const Tile x = decode_tile<BN>(p, t);
      const bool rd = x.kind != kUpdate;   // read and Pc tiles: a bf16 result, no W
      const int mt = x.mt, nt = x.nt;
      const int b = j & 1;
      if (!mbar_wait(tfull + 8 * b, (j >> 1) & 1, p.err)) break;
      umma::fence_after();
      const bool staged = !rd && !p.first;
      const float rscale = x.kind == kPc ? p.eta : 1.f;
      const int orow = x.kind == kReadNext ? p.tok0 + p.C + BM * mt : p.tok0 + BM * mt;
      // W of piece cc into its fp32 staging tile (one thread; the tile's previous store has
      // been read out, see the end of every piece)
      auto issue_w = [&](int cc) {
        const uint32_t e = ec + cc;
        mbar_arrive_expect_tx(wfull + 8 * (e & 1), 8192);
        tma_load_2d(fbuf(e), &tmWf, wfull + 8 * (e & 1), BN * nt + 16 * cc, BM * mt);
      };
      if (staged && ctid == 0) {
        issue_w(0);
        if (NCC > 1) issue_w(1);
      }
      uint32_t r[2][16];
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + b * BN;
      umma::ld32x16(tbase, r[0]);
#pragma unroll
      for (int cc = 0; cc < NCC; ++cc) {
        const uint32_t e = ec + cc;
        umma::wait_ld();
        umma::reg_fence_n(r[cc & 1]);
        if (cc + 1 < NCC) umma::ld32x16(tbase + 16 * (cc + 1), r[(cc + 1) & 1]);
        const uint32_t* rv = r[cc & 1];
        const int col = BN * nt + 16 * cc;
        const uint32_t hb = hbuf(e), fb = fbuf(e);
        if (rd) {
          float o[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = rscale * __uint_as_float(rv[k]);
          sts128(hb + swz<32>(row * 32),
                 make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                            pack_bf16(o[6], o[7])));
          sts128(hb + swz<32>(row * 32 + 16),
                 make_uint4(pack_bf16(o[8], o[9]), pack_bf16(o[10], o[11]),
                            pack_bf16(o[12], o[13]), pack_bf16(o[14], o[15])));
        } else {
          float w[16];
          if (staged) {
            // a wait that gives up only raises the error word: every thread must still reach
            // the named barrier below
            mbar_wait(wfull + 8 * (e & 1), nld[e & 1] & 1, p.err);
            ++nld[e & 1];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 x = lds128(fb + swz<64>(row * 64 + 16 * v));
              w[4 * v] = __uint_as_float(x.x);
              w[4 * v + 1] = __uint_as_float(x.y);
              w[4 * v + 2] = __uint_as_float(x.z);
              w[4 * v + 3] = __uint_as_float(x.w);
            }
          } else {
            const uint4* src =
                reinterpret_cast<const uint4*>(p.W0 + (size_t)(BM * mt + row) * p.D + col);
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              const uint4 x = src[v];
              const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                w[8 * v + 2 * k] = bf16_lo(xs[k]);
                w[8 * v + 2 * k + 1] = bf16_hi(xs[k]);
              }
            }
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) w[k] = fmaf(p.eta, __uint_as_float(rv[k]), w[k]);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            sts128(fb + swz<64>(row * 64 + 16 * v),
                   make_uint4(__float_as_uint(w[4 * v]), __float_as_uint(w[4 * v + 1]),
                              __float_as_uint(w[4 * v + 2]), __float_as_uint(w[4 * v + 3])));
          if (p.Wbf_next) {
            sts128(hb + swz<32>(row * 32),
                   make_uint4(pack_bf16(w[0], w[1]), pack_bf16(w[2], w[3]),
                              pack_bf16(w[4], w[5]), pack_bf16(w[6], w[7])));
            sts128(hb + swz<32>(row * 32 + 16),
                   make_uint4(pack_bf16(w[8], w[9]), pack_bf16(w[10], w[11]),
                              pack_bf16(w[12], w[13]), pack_bf16(w[14], w[15])));
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (ctid == 0) {
          if (x.kind == kPc) {
            tma_store_2d(&tmPs, hb, col, BM * mt);
          } else if (rd) {
            tma_store_2d(&tmO, hb, col, orow);
          } else {
            tma_store_2d(&tmWf, fb, col, BM * mt);
            if (p.Wbf_next) tma_store_2d(&tmWb, hb, col, BM * mt);
          }
          bulk_commit();
          // this piece's staging tiles are read out before anyone rewrites them (the next
          // piece with the same parity comes after the next named barrier)
          bulk_wait_read<0>();
          if (staged && cc + 2 < NCC) issue_w(cc + 2);
        }
      }
      ec += NCC;
      if (x.kind == kPc && ctid == 0) {
        // the tile is in global memory before it is announced to the read tiles of chunk i+1
        bulk_wait<0>();
        fence_proxy_async_global();
        red_release_gpu_add(p.pdone + mt, 1);
      }
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + 8 * b);
    }
    if (ctid == 0) bulk_wait<0>();
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 1) umma::tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int pick_bn(int D) { return D % 256 == 0 ? 256 : (D % 128 == 0 ? 128 : 64); }

// Workspace: two bf16 copies of W (n > 1), the tile counter of every launch, the Pc counters of
// every launch (C / 128 each) and one C x C bf16 Pc buffer (n > 1).
struct IpWorkspace {
  size_t wbf, counters, pc, bytes;
};
IpWorkspace ip_workspace(int T, int Dff, int D, int C) {
  const int n = T / C;
  IpWorkspace w{};
  const size_t wbf_bytes = n > 1 ? align256((size_t)Dff * D * 2) : 0;
  w.wbf = 0;
  w.counters = 2 * wbf_bytes;
  const size_t nct = (size_t)std::max(n, 1) * (1 + C / BM);
  w.pc = w.counters + align256(sizeof(int) * nct);
  w.bytes = w.pc + (n > 1 ? align256((size_t)C * C * 2) : 0);
  return w;
}

// Chunks per launch: 2 (the pair form above) where the tiles allow it (256-wide tiles, C a
// multiple of 256) unless a tuning choice asks for 1.
bool pairs_enabled(int BN, int C) {
  const int choice = tuning(kTuneInplaceChunksPerLaunch);
  return choice != 1 && BN == 256 && C % 256 == 0;
}

template <int BN>
int launch_bn(const InplaceArgs& a, const LaunchCtx& ctx) {
  using Cfg = IpCfg<BN>;
  const int n = a.T / a.C;
  const IpWorkspace wsl = ip_workspace(a.T, a.Dff, a.D, a.C);
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  __nv_bfloat16* wbf[2] = {nullptr, nullptr};
  if (n > 1) {
    wbf[0] = reinterpret_cast<__nv_bfloat16*>(ws + wsl.wbf);
    wbf[1] = reinterpret_cast<__nv_bfloat16*>(ws + wsl.wbf + (wsl.counters - wsl.wbf) / 2);
  }
  int* counters = reinterpret_cast<int*>(ws + wsl.counters);   // one per launch
  int* pdone = counters + n;                                    // C / 128 per launch
  void* pc = n > 1 ? static_cast<void*>(ws + wsl.pc) : nullptr;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap tzk, tzm, tv, tw0, tw[2], twf, to, twb[2], tpl, tps;
  {
    const uint64_t dz[2] = {(uint64_t)a.Dff, (uint64_t)a.T};
    const uint32_t bk[2] = {64, 128}, bm[2] = {64, 64};
    const uint64_t dv[2] = {(uint64_t)a.D, (uint64_t)a.T};
    const uint64_t dw[2] = {(uint64_t)a.D, (uint64_t)a.Dff};
    const uint32_t bpiece[2] = {16, 128};   // epilogue pieces: 16 columns x 128 rows
    if (!make_tmap_2d(&tzk, a.Z, bf, dz, (uint64_t)a.Dff * 2, bk, sw, ctx.msg) ||
        !make_tmap_2d(&tzm, a.Z, bf, dz, (uint64_t)a.Dff * 2, bm, sw, ctx.msg) ||
        !make_tmap_2d(&tv, a.Vhat, bf, dv, (uint64_t)a.D * 2, bm, sw, ctx.msg) ||
        !make_tmap_2d(&tw0, a.W0, bf, dw, (uint64_t)a.D * 2, bm, sw, ctx.msg) ||
        !make_tmap_2d(&twf, a.W_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, dw, (uint64_t)a.D * 4,
                      bpiece, CU_TENSOR_MAP_SWIZZLE_64B, ctx.msg) ||
        !make_tmap_2d(&to, a.O, bf, dv, (uint64_t)a.D * 2, bpiece, CU_TENSOR_MAP_SWIZZLE_32B,
                      ctx.msg))
      return kCuda;
    for (int b = 0; b < 2; ++b) {
      twb[b] = to;   // a valid map fills the slot when there is no bf16 copy to write
      if (wbf[b] &&
          (!make_tmap_2d(&tw[b], wbf[b], bf, dw, (uint64_t)a.D * 2, bm, sw, ctx.msg) ||
           !make_tmap_2d(&twb[b], wbf[b], bf, dw, (uint64_t)a.D * 2, bpiece,
                         CU_TENSOR_MAP_SWIZZLE_32B, ctx.msg)))
        return kCuda;
    }
    tpl = tzk;   // valid maps fill the Pc slots of launches without Pc tiles
    tps = to;
    if (pc) {
      const uint64_t dp[2] = {(uint64_t)a.C, (uint64_t)a.C};
      if (!make_tmap_2d(&tpl, pc, bf, dp, (uint64_t)a.C * 2, bk, sw, ctx.msg) ||
          !make_tmap_2d(&tps, pc, bf, dp, (uint64_t)a.C * 2, bpiece, CU_TENSOR_MAP_SWIZZLE_32B,
                        ctx.msg))
        return kCuda;
    }
  }
  auto kern = inplace_chunk_kernel<BN>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(counters, 0, sizeof(int) * (size_t)n * (1 + a.C / BM), ctx.stream);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("inplace setup: ") + cudaGetErrorString(e);
    return kCuda;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntn = a.D / BN;
  const int n_read = (a.C / BM) * ntn, n_up = (a.Dff / BM) * ntn;
  const bool pairs = n > 1 && pairs_enabled(BN, a.C);
  int L = 0;   // launch index: selects the bf16 copy this launch writes
  for (int i = 0; i < n; ++L) {
    const bool pair = pairs && i + 1 < n;
    const int span = pair ? 2 : 1;
    IpParams p;
    p.W0 = static_cast<const __nv_bfloat16*>(a.W0);
    p.Wout = a.W_out;
    p.Wbf_next = (i + span < n) ? wbf[L & 1] : nullptr;
    p.O = static_cast<__nv_bfloat16*>(a.O);
    p.eta = a.eta;
    p.first = i == 0;
    p.tok0 = i * a.C;
    p.C = a.C;
    p.Dff = a.Dff;
    p.D = a.D;
    p.pair = pair;
    p.n_p = pair ? (a.C / BM) * (a.C / BN) : 0;
    p.n_read = n_read;
    p.n_total = p.n_p + (pair ? 2 : 1) * n_read + n_up;
    p.counter = counters + L;
    p.pdone = pdone + (size_t)L * (a.C / BM);
    p.err = ctx.err;
    const CUtensorMap& wsrc = L == 0 ? tw0 : tw[(L - 1) & 1];
    const int grid = std::min(sms, p.n_total);
    kern<<<grid, THREADS, Cfg::SMEM, ctx.stream>>>(tzk, tzm, wsrc, tv, twf, to, twb[L & 1], tpl,
                                                   tps, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
      *ctx.msg = std::string("inplace launch: ") + cudaGetErrorString(e);
      return kCuda;
    }
    count_launch();
    i += span;
  }
  return kOk;
}

// Plain projection Out[M, N] = A[M, K] B[K, N] (bf16 in, fp32 accumulate, bf16 out) on the read
// tiles of the kernel above: one "chunk" of M rows whose tile list has no update tiles.
template <int BN>
int launch_proj_bn(const void* A, const void* B, void* Out, int M, int K, int N, int* counter,
                   const LaunchCtx& ctx) {
  using Cfg = IpCfg<BN>;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap tak, tam, tb, to;
  const uint64_t da[2] = {(uint64_t)K, (uint64_t)M};
  const uint64_t db[2] = {(uint64_t)N, (uint64_t)K};
  const uint64_t dout[2] = {(uint64_t)N, (uint64_t)M};
  const uint32_t bk[2] = {64, 128}, bm[2] = {64, 64}, bpiece[2] = {16, 128};
  if (!make_tmap_2d(&tak, A, bf, da, (uint64_t)K * 2, bk, sw, ctx.msg) ||
      !make_tmap_2d(&tam, A, bf, da, (uint64_t)K * 2, bm, sw, ctx.msg) ||
      !make_tmap_2d(&tb, B, bf, db, (uint64_t)N * 2, bm, sw, ctx.msg) ||
      !make_tmap_2d(&to, Out, bf, dout, (uint64_t)N * 2, bpiece, CU_TENSOR_MAP_SWIZZLE_32B,
                    ctx.msg))
    return kCuda;
  auto kern = inplace_chunk_kernel<BN>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e == cudaSuccess) e = cudaMemsetAsync(counter, 0, sizeof(int), ctx.stream);
  if (e != cudaSuccess) {
    *ctx.msg = std::string("projection setup: ") + cudaGetErrorString(e);
    return kCuda;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  IpParams p;
  p.W0 = static_cast<const __nv_bfloat16*>(B);
  p.Wout = nullptr;
  p.Wbf_next = nullptr;
  p.O = static_cast<__nv_bfloat16*>(Out);
  p.eta = 0.f;
  p.first = 1;
  p.tok0 = 0;
  p.C = M;
  p.Dff = K;
  p.D = N;
  p.pair = 0;
  p.n_p = 0;
  p.n_read = (M / BM) * (N / BN);
  p.n_total = p.n_read;
  p.counter = counter;
  p.pdone = nullptr;
  p.err = ctx.err;
  // a read-only tile list: the update-tile and Pc maps are never used, valid maps fill their
  // slots
  kern<<<std::min(sms, p.n_read), THREADS, Cfg::SMEM, ctx.stream>>>(tak, tam, tb, tam, to, to,
                                                                     to, tak, to, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *ctx.msg = std::string("projection launch: ") + cudaGetErrorString(e);
    return kCuda;
  }
  count_launch();
  return kOk;
}

}  // namespace

size_t inplace_workspace_bytes(int T, int Dff, int D, int C) {
  return ip_workspace(T, Dff, D, C).bytes;
}

bool inplace_supported(int T, int Dff, int D, int C, std::string* why) {
  if (C % BM != 0) {
    *why = "C must be a multiple of 128";
    return false;
  }
  if (Dff % BM != 0) {
    *why = "Dff must be a multiple of 128";
    return false;
  }
  if (D % 64 != 0) {
    *why = "D must be a multiple of 64";
    return false;
  }
  if ((long long)T * Dff >= (1ll << 40) || T / C > (1 << 20)) {
    *why = "too large";
    return false;
  }
  return true;
}

int launch_projection(const void* A, const void* B, void* Out, int M, int K, int N, int* counter,
                      const LaunchCtx& ctx) {
  switch (pick_bn(N)) {
    case 256: return launch_proj_bn<256>(A, B, Out, M, K, N, counter, ctx);
    case 128: return launch_proj_bn<128>(A, B, Out, M, K, N, counter, ctx);
    default: return launch_proj_bn<64>(A, B, Out, M, K, N, counter, ctx);
  }
}

int launch_inplace(const InplaceArgs& a, const LaunchCtx& ctx) {
  switch (pick_bn(a.D)) {
    case 256: return launch_bn<256>(a, ctx);
    case 128: return launch_bn<128>(a, ctx);
    default: return launch_bn<64>(a, ctx);
  }
}

}  // namespace ttt
