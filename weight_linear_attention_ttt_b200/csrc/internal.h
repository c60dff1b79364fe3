// Internal launcher interface between the C ABI (ttt_api.cu) and the kernel translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime_api.h>
#include <cstddef>
#include <cstdint>
#include <string>

namespace ttt {

enum Status : int { kOk = 0, kInvalid = 1, kUnsupported = 2, kWorkspace = 3, kCuda = 4 };

// Arguments of one dual-form or associative call, already validated by the ABI layer.
struct StateArgs {
  const void* Q;
  const void* K;
  const void* V;
  const float* eta;  // [B,H,T] or nullptr
  float eta_scalar;
  const float* S0;   // [B,H,d,d] fp32 or nullptr (zeros)
  void* O;
  float* S_out;
  int B, H, T, d, C;
  int dt;            // 0 = fp32, 1 = bf16
  void* ws;
  size_t ws_bytes;
  // Associative mode only: run the chunks from the last to the first and keep, inside a chunk,
  // the pairs with key token >= query token (the transposed causal mask). Used by the backward.
  int reverse = 0;
  // Associative mode only: every rate multiplied by eta_mul; decay != 0 runs the momentum
  // (decayed) recurrence M_t = beta M_(t-1) + eta_t k_t^T v_t, o_t = q_t M_t.
  float eta_mul = 1.f;
  int decay = 0;
  float beta = 0.f;
  // decay mode: O = Oadd + add_scale * (decayed output), Oadd [B,H,T,d] bf16 (may equal O)
  const void* Oadd = nullptr;
  float add_scale = 0.f;
  // output row i of token t (pass 2) multiplied by oscale * orow[t] (orow [B,H,T] fp32 or
  // nullptr), before any Oadd combination
  const float* orow = nullptr;
  float oscale = 1.f;
};

struct InplaceArgs {
  const void* Z;
  const void* Vhat;
  const void* W0;
  float eta;
  void* O;
  float* W_out;
  int T, Dff, D, C;
  void* ws;
  size_t ws_bytes;
};

// Per-launch context handed to the launchers.
struct LaunchCtx {
  cudaStream_t stream;
  unsigned* err;        // device error word (bounded waits report here)
  std::string* msg;     // detail for a non-OK status
};

void count_launch(uint64_t n = 1);

// Tuning choices set through ttt_set_tuning() (0 = the library's automatic choice). They exist to
// compare kernel variants; nothing reads the environment.
enum TuneKey : int {
  kTuneDualColumnSplit = 0,   // CTAs per stream of the dual form: 1, 2 or 4
  kTuneDualKernel,            // kDualKernel* below
  kTuneDualWarpCols,          // all-warp-MMA dual form, d = 64: 8 or 16 columns per warp
  kTuneDualStageChunks,       // all-warp-MMA dual form, d = 64, 8 columns: 4 or 8 chunks/stage
  kTuneAssocParts,            // superchunks per stream of the associative mode
  kTuneWaitLimitNs,           // limit of the d = 64 dual-form pipeline waits, ns (0: 4 s)
  kTuneInplaceChunksPerLaunch,  // In-Place: 1 = one chunk per launch, 0 / 2 = chunk pairs
  kTuneDualClusterStreams,    // dual form split across SMs: streams per cluster, 1 or 2
  kTuneMomentumForm,          // momentum: 0 = one pass carrying (S, M), 1 = plain + decayed
  kTuneDualBwdForm,           // dual backward, d = 64: 0 = stage form, 1 = one kernel, 2 = chunk checkpoints
  kTuneAssocBwdForm,          // associative backward: 0 = fused Y/Z pass, 1 = separate passes
  kTuneCount
};
enum DualKernel : int { kDualKernelAuto = 0, kDualKernelWarp = 1, kDualKernelPair = 2,
                        kDualKernelTensor = 3, kDualKernelSplit = 4, kDualKernelGram = 5,
                        kDualKernelRegGram = 6 };
int tuning(TuneKey key);
// Records the detail returned by ttt_last_error_message() on this thread.
void set_last_error(const std::string& msg);

// 3-D tiled tensor map (dims innermost first; strides in bytes for dims 1 and 2).
bool make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                  const uint64_t dims[3], const uint64_t strides[2], const uint32_t box[3],
                  CUtensorMapSwizzle swizzle, std::string* msg);
// 2-D tiled tensor map (dims innermost first; stride of dim 1 in bytes).
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                  const uint64_t dims[2], uint64_t stride1, const uint32_t box[2],
                  CUtensorMapSwizzle swizzle, std::string* msg);

// Dual form.
bool dual_mma_supported(int d, int C, int dt);
int launch_dual_mma(const StateArgs& a, const LaunchCtx& ctx);
int launch_dual_pair(const StateArgs& a, const LaunchCtx& ctx, int split);
int launch_dual_simt(const StateArgs& a, const LaunchCtx& ctx);
// d = 64, C = 16, 32 or 64, bf16: chain on warp MMAs, outputs per stage on tcgen05; split =
// CTAs per stream (1, 2 or 4), dual_tc_split() the automatic choice.
bool dual_tc_supported(int d, int C, int dt);
// d = 64, C = 16, bf16: the chain and the output products on separate SMs of one cluster
// (dual_xsm.cu). dual_xsm_plan returns the streams per cluster (0: not possible) and the
// cluster count; launch_dual_xsm returns kUnsupported when the clusters cannot all be resident.
inline bool dual_xsm_applicable(int d, int C, int dt) { return dt == 1 && d == 64 && C == 16; }
int dual_xsm_plan(int streams, int sms, int* n_clusters);
int launch_dual_xsm(const StateArgs& a, int ks, int n_clusters, const LaunchCtx& ctx);
int dual_tc_split(int streams, int sms);
// d = 64, C = 16, 32 or 64, bf16: the state in TMEM, updated once per 128-token stage on
// tcgen05; the chain is a blocked substitution over the stage's key Gram blocks (dual_gram.cu).
bool dual_gram_supported(int d, int C, int dt);
int launch_dual_gram(const StateArgs& a, const LaunchCtx& ctx);
// The same shapes: the state in registers and the stage's Gram-block substitution on warp MMAs,
// the data-only products on tcgen05 (dual_rgram.cu).
int launch_dual_rgram(const StateArgs& a, const LaunchCtx& ctx);
int launch_dual_tc(const StateArgs& a, int split, const LaunchCtx& ctx);
// The chunk-start states of every 16-token chunk as bf16 d x d checkpoints ([streams, T / 16,
// d, d], the dual-form backward's layout), from the stage kernel's state-only chain (bf16,
// d = 64, C = 16; S0 = W0, S_out may be null).
int launch_dual_tc_checkpoints(const StateArgs& a, uint16_t* ckpt, const LaunchCtx& ctx);
// The same chain writing what the stage-form backward reads: the state at the start of every
// 128-token stage ([streams, ceil(T / 128), d, d] bf16) and of every token the residual
// G = K W_c - V and -E = -diag(eta) G ([streams, T, d] bf16 each).
int launch_dual_tc_stage_checkpoints(const StateArgs& a, uint16_t* Ws, uint16_t* G, uint16_t* NE,
                                     const LaunchCtx& ctx);
// True when launch_dual_mma takes O = nullptr for this shape (the stage kernel's state-only
// form: the final state and no outputs).
bool dual_state_only_supported(int d, int C, int dt);

// Associative mode.
size_t assoc_workspace_bytes(int B, int H, int T, int d, int C);
// bf16, d = 64 or 128, C = 16, 32 or 64 with T % 64 == 0. The associative result does not
// depend on C (the recurrence is per token), so every C runs on the 64-token tiles; d = 64
// runs zero-padded to 128 inside the kernel (TMA fills the missing half, no extra traffic).
bool assoc_supported(int d, int C, int T, int dt);
int launch_assoc(const StateArgs& a, const LaunchCtx& ctx);
int launch_assoc_state(const StateArgs& a, const LaunchCtx& ctx);
size_t assoc_bwd_workspace_bytes(int B, int H, int T, int d, int C);
struct AssocBwdArgs {
  const void* Q;
  const void* K;
  const void* V;
  const float* eta;  // [B,H,T] or nullptr
  float eta_scalar;
  const float* S0;   // [B,H,d,d] or nullptr
  const void* dO;
  const float* dS_out;  // [B,H,d,d] or nullptr
  void* dQ;
  void* dK;
  void* dV;
  float* deta;       // [B,H,T]
  float* dS0;        // [B,H,d,d]
  int B, H, T, d, C;
  void* ws;
  size_t ws_bytes;
};
int launch_assoc_bwd(const AssocBwdArgs& a, const LaunchCtx& ctx);
// The associative scan's pass 1 and prefix alone (keys a.K, values a.V, the rate and order of
// `a`): with P > 1 superchunks, part m >= 1 starts from slot m * slot_mul - 1 of `slots`
// ([B*H, nslots, 128, 128] fp32 in a.ws); with P = 1 nothing is launched.
struct AssocPrefix {
  int P, nslots, slot_mul;
  const float* slots;
};
int launch_assoc_prefix(const StateArgs& a, AssocPrefix* out, const LaunchCtx& ctx);
// Backward of the associative mode, fused reverse pass: dV <- Y (unscaled), dK <- eta Z, dS0,
// in one pass over Q, K, V and dO (bf16, d = 64 or 128); `ws` holds the prefix slots.
int launch_assoc_yz(const AssocBwdArgs& a, void* ws, size_t ws_bytes, const LaunchCtx& ctx);
// Sequence-parallel dual form (segment-affine scan over the dual-form kernels). segments: the
// caller's count (must divide T / C) or 0 for the automatic choice; returns -1 if invalid.
int dual_seg_choose_segments(int B, int H, int T, int C, int requested);
size_t dual_seg_workspace_bytes(int B, int H, int d, int S);
int launch_dual_seg(const StateArgs& a, int S, const LaunchCtx& ctx);
// Dual-form backward (one kernel; S0 / dS_out / dS0 of the arguments are W0 / dW_out / dW0; the
// workspace holds one bf16 d x d checkpoint per chunk).
bool dual_bwd_supported(int d, int C, int dt);
size_t dual_bwd_workspace_bytes(int B, int H, int T, int d);
int launch_dual_bwd(const AssocBwdArgs& a, const LaunchCtx& ctx);
// The stage form (d = 64, C = 16, dual_bwd_tc.cu): the forward's residual rows and stage-start
// states from the stage kernel's state-only chain (in the workspace), then one kernel with the
// state gradient's chain on warp MMAs and the stage products on tcgen05.
size_t dual_bwd_stage_workspace_bytes(int B, int H, int T);
int launch_dual_bwd_stage(const AssocBwdArgs& a, const LaunchCtx& ctx);
// Context parallelism of the dual form: a slice's affine maps, and the fold of gathered maps.
size_t dual_slice_maps_workspace_bytes(int B, int H, int T, int d, int dt);
int launch_dual_slice_maps(const StateArgs& a, float* A_out, float* B_out, const LaunchCtx& ctx);
int launch_dual_state_fold(const float* W0, const float* A, const float* B, int upto, int bh,
                           int d, float* W_out, const LaunchCtx& ctx);
// Dual-form backward over S segments (S <= 1: launch_dual_bwd).
size_t dual_seg_bwd_workspace_bytes(int B, int H, int T, int d, int S);
int launch_dual_seg_bwd(const AssocBwdArgs& a, int S, const LaunchCtx& ctx);
size_t assoc_momentum_workspace_bytes(int B, int H, int T, int d, int C);
struct AssocMomentumArgs {
  const void* Q;
  const void* K;
  const void* V;
  const float* eta;
  float eta_scalar;
  float beta;
  const float* S0;   // [B,H,d,d] or nullptr
  const float* M0;   // [B,H,d,d] or nullptr
  void* O;
  float* S_out;
  float* M_out;
  int B, H, T, d, C;
  void* ws;
  size_t ws_bytes;
};
int launch_assoc_momentum(const AssocMomentumArgs& a, const LaunchCtx& ctx);
// The one-pass form (both states carried through the chunks; every beta in [0, 1]).
size_t assoc_momentum_fused_workspace_bytes(int B, int H, int T, int d, int C);
int launch_assoc_momentum_fused(const AssocMomentumArgs& a, const LaunchCtx& ctx);
// The two-pass form (plain + decayed associative passes; beta in [0.25, 0.9]).
size_t assoc_momentum_split_workspace_bytes(int B, int H, int T, int d, int C);
int launch_assoc_momentum_split(const AssocMomentumArgs& a, const LaunchCtx& ctx);
// Out[M, N] = A[M, K] B[K, N], bf16, on the In-Place kernel's read tiles (M % 128 == 0,
// K % 64 == 0, N % 64 == 0); `counter` is one int of device memory.
int launch_projection(const void* A, const void* B, void* Out, int M, int K, int N, int* counter,
                      const LaunchCtx& ctx);
size_t lm_target_workspace_bytes(int T, int Dm, int D, int k);
int launch_lm_target(const void* X, const float* Wc, const void* Wp, void* Vhat, int T, int Dm,
                     int D, int k, void* ws, size_t ws_bytes, const LaunchCtx& ctx);

// In-Place W_down.
size_t inplace_workspace_bytes(int T, int Dff, int D, int C);
bool inplace_supported(int T, int Dff, int D, int C, std::string* why);
int launch_inplace(const InplaceArgs& a, const LaunchCtx& ctx);

}  // namespace ttt
