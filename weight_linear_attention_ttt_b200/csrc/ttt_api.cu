// C ABI of libttt_b200: argument validation, dispatch, tensor-map encoding, status reporting.
// Declarations and the contract of every entry point live in include/ttt.h.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "internal.h"
#include "ttt.h"

namespace ttt {

static std::atomic<uint64_t> g_launches{0};
void count_launch(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Device error word written by bounded waits in the kernels (one per device context).
__device__ unsigned g_device_error;

static std::atomic<int> g_tuning[kTuneCount];
int tuning(TuneKey key) { return g_tuning[key].load(std::memory_order_relaxed); }

struct TuneName {
  const char* name;
  TuneKey key;
};
static const TuneName kTuneNames[] = {{"dual_column_split", kTuneDualColumnSplit},
                                      {"dual_kernel", kTuneDualKernel},
                                      {"dual_warp_cols", kTuneDualWarpCols},
                                      {"dual_stage_chunks", kTuneDualStageChunks},
                                      {"assoc_parts", kTuneAssocParts},
                                      {"wait_limit_ns", kTuneWaitLimitNs},
                                      {"inplace_chunks_per_launch",
                                       kTuneInplaceChunksPerLaunch},
                                      {"dual_cluster_streams", kTuneDualClusterStreams},
                                      {"momentum_form", kTuneMomentumForm},
                                      {"dual_bwd_form", kTuneDualBwdForm},
                                      {"assoc_bwd_form", kTuneAssocBwdForm}};
static int tune_key(const char* name) {
  if (!name) return -1;
  for (const auto& t : kTuneNames)
    if (std::strcmp(t.name, name) == 0) return t.key;
  return -1;
}

static thread_local std::string t_last_error;
void set_last_error(const std::string& msg) { t_last_error = msg; }

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn(std::string* msg) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!fn && msg) *msg = "cuTensorMapEncodeTiled entry point not available";
  return fn;
}

bool make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                  const uint64_t dims[3], const uint64_t strides[2], const uint32_t box[3],
                  CUtensorMapSwizzle swizzle, std::string* msg) {
  auto fn = encode_fn(msg);
  if (!fn) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (msg) *msg = "cuTensorMapEncodeTiled (3-D) failed with CUresult " + std::to_string(r);
    return false;
  }
  return true;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                  const uint64_t dims[2], uint64_t stride1, const uint32_t box[2],
                  CUtensorMapSwizzle swizzle, std::string* msg) {
  auto fn = encode_fn(msg);
  if (!fn) return false;
  const cuuint32_t estr[2] = {1, 1};
  const cuuint64_t strides[1] = {stride1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (msg) *msg = "cuTensorMapEncodeTiled (2-D) failed with CUresult " + std::to_string(r);
    return false;
  }
  return true;
}

static unsigned* device_error_word(std::string* msg) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_device_error);
  if (e != cudaSuccess) {
    *msg = std::string("cudaGetSymbolAddress(error word): ") + cudaGetErrorString(e);
    return nullptr;
  }
  return static_cast<unsigned*>(p);
}

namespace {

int fail(int status, const std::string& why) {
  t_last_error = why;
  return status;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || !na || !nb) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Shared checks of the dual-form and associative entry points.
int check_state_args(const char* fn, const StateArgs& a, size_t need_ws) {
  const std::string f(fn);
  if (!a.Q || !a.K || !a.V || !a.O || !a.S_out)
    return fail(TTT_ERR_INVALID_ARG, f + ": Q, K, V, O and the output state must be non-null");
  if (a.B <= 0 || a.H <= 0 || a.T <= 0 || a.d <= 0 || a.C <= 0)
    return fail(TTT_ERR_INVALID_ARG, f + ": B, H, T, d and C must be positive");
  if (a.T % a.C != 0) return fail(TTT_ERR_INVALID_ARG, f + ": T must be a multiple of C");
  if (a.dt != TTT_DTYPE_F32 && a.dt != TTT_DTYPE_BF16)
    return fail(TTT_ERR_INVALID_ARG, f + ": dtype must be TTT_DTYPE_F32 or TTT_DTYPE_BF16");
  const void* ptrs[] = {a.Q, a.K, a.V, a.O, a.S_out, a.eta, a.S0};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, f + ": every device pointer must be 16-byte aligned");
  if ((uint64_t)a.B * a.H * a.T * a.d >= (1ull << 40))
    return fail(TTT_ERR_UNSUPPORTED, f + ": tensor too large");
  const size_t esz = a.dt == TTT_DTYPE_F32 ? 4 : 2;
  const size_t nx = (size_t)a.B * a.H * a.T * a.d * esz;
  const size_t ns = (size_t)a.B * a.H * a.d * a.d * 4;
  const size_t ne = (size_t)a.B * a.H * a.T * 4;
  const void* ins[] = {a.Q, a.K, a.V};
  for (const void* p : ins)
    if (overlap(a.O, nx, p, nx) || overlap(a.S_out, ns, p, nx))
      return fail(TTT_ERR_INVALID_ARG, f + ": outputs must not overlap Q, K or V");
  if (overlap(a.O, nx, a.S_out, ns) || overlap(a.O, nx, a.eta, ne) ||
      overlap(a.S_out, ns, a.eta, ne) || overlap(a.O, nx, a.S0, ns))
    return fail(TTT_ERR_INVALID_ARG, f + ": outputs must not overlap eta, the initial state or "
                                         "each other");
  if (a.S0 && a.S0 != a.S_out && overlap(a.S0, ns, a.S_out, ns))
    return fail(TTT_ERR_INVALID_ARG,
                f + ": the output state may equal the initial state but not partly overlap it");
  if (need_ws && (!a.ws || a.ws_bytes < need_ws))
    return fail(TTT_ERR_WORKSPACE,
                f + ": workspace of at least " + std::to_string(need_ws) + " bytes required");
  if (need_ws && !aligned16(a.ws))
    return fail(TTT_ERR_INVALID_ARG, f + ": workspace must be 16-byte aligned");
  return TTT_OK;
}

int finish(int st, const std::string& msg) {
  if (st != TTT_OK) t_last_error = msg;
  return st;
}

}  // namespace
}  // namespace ttt

using namespace ttt;

extern "C" {

const char* ttt_status_string(int s) {
  switch (s) {
    case TTT_OK: return "TTT_OK";
    case TTT_ERR_INVALID_ARG: return "TTT_ERR_INVALID_ARG";
    case TTT_ERR_UNSUPPORTED: return "TTT_ERR_UNSUPPORTED";
    case TTT_ERR_WORKSPACE: return "TTT_ERR_WORKSPACE";
    case TTT_ERR_CUDA: return "TTT_ERR_CUDA";
    case TTT_ERR_TIMEOUT: return "TTT_ERR_TIMEOUT";
  }
  return "TTT_ERR_UNKNOWN";
}

const char* ttt_last_error_message(void) { return t_last_error.c_str(); }

int ttt_version(void) { return 10000; }

uint64_t ttt_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int ttt_set_tuning(const char* key, int value) {
  const int k = ttt::tune_key(key);
  if (k < 0)
    return fail(TTT_ERR_INVALID_ARG,
                std::string("ttt_set_tuning: unknown key ") + (key ? key : "(null)"));
  if (value < 0) return fail(TTT_ERR_INVALID_ARG, "ttt_set_tuning: value must be >= 0");
  ttt::g_tuning[k].store(value, std::memory_order_relaxed);
  return TTT_OK;
}

int ttt_get_tuning(const char* key) {
  const int k = ttt::tune_key(key);
  return k < 0 ? -1 : ttt::g_tuning[k].load(std::memory_order_relaxed);
}

void ttt_reset_tuning(void) {
  for (auto& t : ttt::g_tuning) t.store(0, std::memory_order_relaxed);
}

int ttt_read_device_error(unsigned* value) {
  if (!value) return fail(TTT_ERR_INVALID_ARG, "ttt_read_device_error: null output");
  unsigned v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess)
    return fail(TTT_ERR_CUDA, std::string("ttt_read_device_error: ") + cudaGetErrorString(e));
  *value = v;
  return TTT_OK;
}

size_t ttt_linear_dual_workspace_size(int, int, int, int, int, int) { return 0; }

int ttt_linear_dual_fwd(const void* Q, const void* K, const void* V, const float* eta,
                        float eta_scalar, const float* W0, void* O, float* W_out, int B, int H,
                        int T, int d, int C, int dt, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  StateArgs a{Q, K, V, eta, eta_scalar, W0, O, W_out, B, H, T, d, C, dt, workspace,
              workspace_bytes};
  int st = check_state_args("ttt_linear_dual_fwd", a, 0);
  if (st != TTT_OK) return st;
  if (!(d == 32 || d == 64 || d == 128) || C > 64)
    return fail(TTT_ERR_UNSUPPORTED,
                "ttt_linear_dual_fwd: supported d in {32, 64, 128} and 1 <= C <= 64");
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  st = dual_mma_supported(d, C, dt) ? launch_dual_mma(a, ctx) : launch_dual_simt(a, ctx);
  return finish(st, msg);
}

size_t ttt_linear_dual_seg_workspace_size(int B, int H, int T, int d, int C, int dt,
                                          int segments) {
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0 || T % C != 0 || segments < 0) return 0;
  (void)dt;
  const int S = dual_seg_choose_segments(B, H, T, C, segments);
  return S < 1 ? 0 : dual_seg_workspace_bytes(B, H, d, S);
}

int ttt_linear_dual_seg_fwd(const void* Q, const void* K, const void* V, const float* eta,
                            float eta_scalar, const float* W0, void* O, float* W_out, int B,
                            int H, int T, int d, int C, int dt, int segments, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream) {
  const char* fn = "ttt_linear_dual_seg_fwd";
  StateArgs a{Q, K, V, eta, eta_scalar, W0, O, W_out, B, H, T, d, C, dt, workspace,
              workspace_bytes};
  int st = check_state_args(fn, a, 0);
  if (st != TTT_OK) return st;
  if (!(d == 32 || d == 64 || d == 128) || C > 64)
    return fail(TTT_ERR_UNSUPPORTED, std::string(fn) + ": supported d in {32, 64, 128} and "
                                                       "1 <= C <= 64");
  if (segments < 0) return fail(TTT_ERR_INVALID_ARG, std::string(fn) + ": segments must be >= 0");
  const int S = dual_seg_choose_segments(B, H, T, C, segments);
  if (S < 1)
    return fail(TTT_ERR_INVALID_ARG,
                std::string(fn) + ": segments must divide the number of chunks T / C");
  const size_t need = dual_seg_workspace_bytes(B, H, d, S);
  st = check_state_args(fn, a, need);
  if (st != TTT_OK) return st;
  if (need && overlap(workspace, workspace_bytes, O, (size_t)B * H * T * d * (dt ? 2 : 4)))
    return fail(TTT_ERR_INVALID_ARG, std::string(fn) + ": workspace overlaps O");
  if (need && (overlap(workspace, workspace_bytes, W_out, (size_t)B * H * d * d * 4) ||
               overlap(workspace, workspace_bytes, W0, (size_t)B * H * d * d * 4)))
    return fail(TTT_ERR_INVALID_ARG, std::string(fn) + ": workspace overlaps a state");
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_dual_seg(a, S, ctx), msg);
}

size_t ttt_linear_dual_slice_maps_workspace_size(int B, int H, int T, int d, int C, int dt) {
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0 || T % C != 0) return 0;
  return dual_slice_maps_workspace_bytes(B, H, T, d, dt);
}

int ttt_linear_dual_slice_maps(const void* K, const void* V, const float* eta, float eta_scalar,
                               float* A_out, float* B_out, int B, int H, int T, int d, int C,
                               int dt, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  const std::string f("ttt_linear_dual_slice_maps");
  if (!K || !V || !A_out || !B_out)
    return fail(TTT_ERR_INVALID_ARG, f + ": K, V, A_out and B_out must be non-null");
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0)
    return fail(TTT_ERR_INVALID_ARG, f + ": B, H, T, d and C must be positive");
  if (T % C != 0) return fail(TTT_ERR_INVALID_ARG, f + ": T must be a multiple of C");
  if (dt != TTT_DTYPE_F32 && dt != TTT_DTYPE_BF16)
    return fail(TTT_ERR_INVALID_ARG, f + ": dtype must be TTT_DTYPE_F32 or TTT_DTYPE_BF16");
  const void* ptrs[] = {K, V, eta, A_out, B_out, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, f + ": every device pointer must be 16-byte aligned");
  if (!(d == 32 || d == 64 || d == 128) || C > 64)
    return fail(TTT_ERR_UNSUPPORTED, f + ": supported d in {32, 64, 128} and 1 <= C <= 64");
  const size_t need = dual_slice_maps_workspace_bytes(B, H, T, d, dt);
  if (!workspace || workspace_bytes < need)
    return fail(TTT_ERR_WORKSPACE, f + ": workspace smaller than the size query returns");
  const size_t nx = (size_t)B * H * T * d * (dt ? 2 : 4), ns = (size_t)B * H * d * d * 4;
  const size_t ne = (size_t)B * H * T * 4;
  struct R { const void* p; size_t n; };
  const R ins[] = {{K, nx}, {V, nx}, {eta, ne}};
  const R outs[] = {{A_out, ns}, {B_out, ns}, {workspace, workspace_bytes}};
  for (size_t i = 0; i < 3; ++i) {
    for (const R& in : ins)
      if (in.p && overlap(outs[i].p, outs[i].n, in.p, in.n))
        return fail(TTT_ERR_INVALID_ARG, f + ": outputs and workspace must not overlap inputs");
    for (size_t j = i + 1; j < 3; ++j)
      if (overlap(outs[i].p, outs[i].n, outs[j].p, outs[j].n))
        return fail(TTT_ERR_INVALID_ARG, f + ": outputs and workspace must not overlap");
  }
  StateArgs a{K, K, V, eta, eta_scalar, nullptr, nullptr, nullptr, B, H, T, d, C, dt, workspace,
              workspace_bytes};
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_dual_slice_maps(a, A_out, B_out, ctx), msg);
}

int ttt_dual_state_fold(const float* W0, const float* A_maps, const float* B_maps, int n_maps,
                        int upto, float* W_out, int B, int H, int d, cudaStream_t stream) {
  const std::string f("ttt_dual_state_fold");
  if (!A_maps || !B_maps || !W_out)
    return fail(TTT_ERR_INVALID_ARG, f + ": A_maps, B_maps and W_out must be non-null");
  if (B <= 0 || H <= 0 || d <= 0 || n_maps <= 0 || upto < 0 || upto > n_maps)
    return fail(TTT_ERR_INVALID_ARG, f + ": B, H, d, n_maps must be positive, 0 <= upto <= n_maps");
  const void* ptrs[] = {W0, A_maps, B_maps, W_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, f + ": every device pointer must be 16-byte aligned");
  if (!(d == 32 || d == 64 || d == 128))
    return fail(TTT_ERR_UNSUPPORTED, f + ": supported d in {32, 64, 128}");
  const size_t ns = (size_t)B * H * d * d * 4, nm = ns * n_maps;
  if (overlap(W_out, ns, A_maps, nm) || overlap(W_out, ns, B_maps, nm))
    return fail(TTT_ERR_INVALID_ARG, f + ": W_out must not overlap the maps");
  if (W0 && W0 != W_out && overlap(W0, ns, W_out, ns))
    return fail(TTT_ERR_INVALID_ARG, f + ": W_out may equal W0 but not partly overlap it");
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_dual_state_fold(W0, A_maps, B_maps, upto, B * H, d, W_out, ctx), msg);
}

size_t ttt_assoc_scan_workspace_size(int B, int H, int T, int d, int C, int dt) {
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0 || !assoc_supported(d, C, T, dt))
    return 0;
  return assoc_workspace_bytes(B, H, T, d, C);
}

int ttt_assoc_scan_fwd(const void* Q, const void* K, const void* V, const float* eta,
                       float eta_scalar, const float* S0, void* O, float* S_out, int B, int H,
                       int T, int d, int C, int dt, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
  StateArgs a{Q, K, V, eta, eta_scalar, S0, O, S_out, B, H, T, d, C, dt, workspace,
              workspace_bytes};
  int st = check_state_args("ttt_assoc_scan_fwd", a, 0);
  if (st != TTT_OK) return st;
  if (!assoc_supported(d, C, T, dt))
    return fail(TTT_ERR_UNSUPPORTED, "ttt_assoc_scan_fwd: supported bf16, d == 64 or 128, "
                                     "C == 16, 32 or 64, T % 64 == 0");
  st = check_state_args("ttt_assoc_scan_fwd", a, assoc_workspace_bytes(B, H, T, d, C));
  if (st != TTT_OK) return st;
  if (overlap(workspace, workspace_bytes, O, (size_t)B * H * T * d * 2) ||
      overlap(workspace, workspace_bytes, S_out, (size_t)B * H * d * d * 4))
    return fail(TTT_ERR_INVALID_ARG, "ttt_assoc_scan_fwd: workspace overlaps an output");
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_assoc(a, ctx), msg);
}

size_t ttt_assoc_momentum_workspace_size(int B, int H, int T, int d, int C, int dt) {
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0 || T % C != 0 ||
      !assoc_supported(d, C, T, dt))
    return 0;
  return assoc_momentum_workspace_bytes(B, H, T, d, C);
}

int ttt_assoc_momentum_fwd(const void* Q, const void* K, const void* V, const float* eta,
                           float eta_scalar, float beta, const float* S0, const float* M0,
                           void* O, float* S_out, float* M_out, int B, int H, int T, int d,
                           int C, int dt, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
  const char* fn = "ttt_assoc_momentum_fwd";
  const std::string f(fn);
  StateArgs a{Q, K, V, eta, eta_scalar, S0, O, S_out, B, H, T, d, C, dt, workspace,
              workspace_bytes};
  int st = check_state_args(fn, a, 0);
  if (st != TTT_OK) return st;
  if (!M_out) return fail(TTT_ERR_INVALID_ARG, f + ": M_out must be non-null");
  // The one-pass form weights every term by a sum of non-negative powers of beta: any beta in
  // [0, 1]. The two-pass form (a comparison variant) subtracts two bf16 outputs of size
  // ~1/(1 - beta) times the result early in a sequence; up to beta = 0.9 that stays within the
  // bf16 accuracy bar.
  if (tuning(kTuneMomentumForm) == 1) {
    if (!(beta >= 0.25f && beta <= 0.9f))
      return fail(TTT_ERR_UNSUPPORTED, f + ": the two-pass momentum form (momentum_form 1) needs "
                                           "a coefficient in [0.25, 0.9]");
  } else if (!(beta >= 0.f && beta <= 1.f)) {
    return fail(TTT_ERR_UNSUPPORTED, f + ": momentum coefficient must lie in [0, 1]");
  }
  if (!assoc_supported(d, C, T, dt))
    return fail(TTT_ERR_UNSUPPORTED,
                f + ": supported bf16, d == 64 or 128, C == 16, 32 or 64, T % 64 == 0");
  st = check_state_args(fn, a, assoc_momentum_workspace_bytes(B, H, T, d, C));
  if (st != TTT_OK) return st;
  const void* extra[] = {M0, M_out};
  for (const void* p : extra)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, f + ": every device pointer must be 16-byte aligned");
  const size_t nx = (size_t)B * H * T * d * 2, ns = (size_t)B * H * d * d * 4;
  const size_t ne = (size_t)B * H * T * 4;
  struct R { const void* p; size_t n; };
  const R others[] = {{Q, nx}, {K, nx}, {V, nx}, {eta, ne}, {O, nx}, {S_out, ns}, {S0, ns},
                      {workspace, workspace_bytes}};
  for (const R& o : others)
    if (o.p && overlap(M_out, ns, o.p, o.n))
      return fail(TTT_ERR_INVALID_ARG, f + ": M_out must not overlap another argument");
  if (M0 && M0 != M_out) {
    const R outs[] = {{O, nx}, {S_out, ns}, {workspace, workspace_bytes}};
    for (const R& o : outs)
      if (overlap(M0, ns, o.p, o.n))
        return fail(TTT_ERR_INVALID_ARG, f + ": M0 must not overlap O, S_out or the workspace");
  }
  if (overlap(workspace, workspace_bytes, O, nx) ||
      overlap(workspace, workspace_bytes, S_out, ns))
    return fail(TTT_ERR_INVALID_ARG, f + ": workspace overlaps an output");
  AssocMomentumArgs m{Q, K, V, eta, eta_scalar, beta, S0, M0, O, S_out, M_out, B, H, T, d, C,
                      workspace, workspace_bytes};
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_assoc_momentum(m, ctx), msg);
}

size_t ttt_assoc_scan_bwd_workspace_size(int B, int H, int T, int d, int C, int dt) {
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0 || T % C != 0 ||
      !assoc_supported(d, C, T, dt))
    return 0;
  return assoc_bwd_workspace_bytes(B, H, T, d, C);
}

int ttt_assoc_scan_bwd(const void* Q, const void* K, const void* V, const float* eta,
                       float eta_scalar, const float* S0, const void* dO, const float* dS_out,
                       void* dQ, void* dK, void* dV, float* deta, float* dS0, int B, int H,
                       int T, int d, int C, int dt, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
  const std::string f("ttt_assoc_scan_bwd");
  if (!Q || !K || !V || !dO || !dQ || !dK || !dV || !deta || !dS0)
    return fail(TTT_ERR_INVALID_ARG, f + ": Q, K, V, dO and every output must be non-null");
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0)
    return fail(TTT_ERR_INVALID_ARG, f + ": B, H, T, d and C must be positive");
  if (T % C != 0) return fail(TTT_ERR_INVALID_ARG, f + ": T must be a multiple of C");
  if (dt != TTT_DTYPE_F32 && dt != TTT_DTYPE_BF16)
    return fail(TTT_ERR_INVALID_ARG, f + ": dtype must be TTT_DTYPE_F32 or TTT_DTYPE_BF16");
  const void* ptrs[] = {Q, K, V, eta, S0, dO, dS_out, dQ, dK, dV, deta, dS0, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, f + ": every device pointer must be 16-byte aligned");
  if (!assoc_supported(d, C, T, dt))
    return fail(TTT_ERR_UNSUPPORTED,
                f + ": supported bf16, d == 64 or 128, C == 16, 32 or 64, T % 64 == 0");
  const size_t need = assoc_bwd_workspace_bytes(B, H, T, d, C);
  if (!workspace || workspace_bytes < need)
    return fail(TTT_ERR_WORKSPACE, f + ": workspace smaller than ttt_assoc_scan_bwd_workspace_size()");
  const size_t nx = (size_t)B * H * T * d * 2, ns = (size_t)B * H * d * d * 4;
  const size_t ne = (size_t)B * H * T * 4;
  struct R { const void* p; size_t n; };
  const R ins[] = {{Q, nx}, {K, nx}, {V, nx}, {dO, nx}, {eta, ne}, {S0, ns}, {dS_out, ns}};
  const R outs[] = {{dQ, nx}, {dK, nx}, {dV, nx}, {deta, ne}, {dS0, ns},
                    {workspace, workspace_bytes}};
  for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
    for (const R& in : ins)
      if (in.p && overlap(outs[i].p, outs[i].n, in.p, in.n))
        return fail(TTT_ERR_INVALID_ARG, f + ": outputs and workspace must not overlap inputs");
    for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
      if (overlap(outs[i].p, outs[i].n, outs[j].p, outs[j].n))
        return fail(TTT_ERR_INVALID_ARG, f + ": outputs and workspace must not overlap");
  }
  AssocBwdArgs a{Q, K, V, eta, eta_scalar, S0, dO, dS_out, dQ, dK, dV, deta, dS0, B, H, T, d, C,
                 workspace, workspace_bytes};
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_assoc_bwd(a, ctx), msg);
}

namespace {
// Host-side checks shared by the dual-form backward entry points (before any CUDA call):
// pointers, sizes, dtype, alignment, support, workspace and overlaps.
int check_dual_bwd_args(const std::string& f, const void* Q, const void* K, const void* V,
                        const float* eta, const float* W0, const void* dO, const float* dW_out,
                        void* dQ, void* dK, void* dV, float* deta, float* dW0, int B, int H,
                        int T, int d, int C, int dt, void* workspace, size_t workspace_bytes,
                        size_t need) {
  if (!Q || !K || !V || !dO || !dQ || !dK || !dV || !deta || !dW0)
    return fail(TTT_ERR_INVALID_ARG, f + ": Q, K, V, dO and every output must be non-null");
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0)
    return fail(TTT_ERR_INVALID_ARG, f + ": B, H, T, d and C must be positive");
  if (T % C != 0) return fail(TTT_ERR_INVALID_ARG, f + ": T must be a multiple of C");
  if (dt != TTT_DTYPE_F32 && dt != TTT_DTYPE_BF16)
    return fail(TTT_ERR_INVALID_ARG, f + ": dtype must be TTT_DTYPE_F32 or TTT_DTYPE_BF16");
  const void* ptrs[] = {Q, K, V, eta, W0, dO, dW_out, dQ, dK, dV, deta, dW0, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, f + ": every device pointer must be 16-byte aligned");
  if (!dual_bwd_supported(d, C, dt))
    return fail(TTT_ERR_UNSUPPORTED, f + ": supported bf16, C == 16, d in {32, 64, 128}");
  if (need == 0) return TTT_OK;   // caller signals an invalid segment count separately
  if (!workspace || workspace_bytes < need)
    return fail(TTT_ERR_WORKSPACE, f + ": workspace smaller than the size query returns");
  const size_t nx = (size_t)B * H * T * d * 2, ns = (size_t)B * H * d * d * 4;
  const size_t ne = (size_t)B * H * T * 4;
  struct R { const void* p; size_t n; };
  const R ins[] = {{Q, nx}, {K, nx}, {V, nx}, {dO, nx}, {eta, ne}, {W0, ns}, {dW_out, ns}};
  const R outs[] = {{dQ, nx}, {dK, nx}, {dV, nx}, {deta, ne}, {dW0, ns},
                    {workspace, workspace_bytes}};
  for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
    for (const R& in : ins)
      if (in.p && overlap(outs[i].p, outs[i].n, in.p, in.n))
        return fail(TTT_ERR_INVALID_ARG, f + ": outputs and workspace must not overlap inputs");
    for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
      if (overlap(outs[i].p, outs[i].n, outs[j].p, outs[j].n))
        return fail(TTT_ERR_INVALID_ARG, f + ": outputs and workspace must not overlap");
  }
  return TTT_OK;
}
}  // namespace

size_t ttt_linear_dual_bwd_workspace_size(int B, int H, int T, int d, int C, int dt) {
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0 || T % C != 0 ||
      !dual_bwd_supported(d, C, dt))
    return 0;
  return dual_bwd_workspace_bytes(B, H, T, d);
}

int ttt_linear_dual_bwd(const void* Q, const void* K, const void* V, const float* eta,
                        float eta_scalar, const float* W0, const void* dO, const float* dW_out,
                        void* dQ, void* dK, void* dV, float* deta, float* dW0, int B, int H,
                        int T, int d, int C, int dt, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  const std::string f("ttt_linear_dual_bwd");
  const size_t need = (B > 0 && H > 0 && T > 0 && d > 0) ? dual_bwd_workspace_bytes(B, H, T, d)
                                                          : 1;
  int st = check_dual_bwd_args(f, Q, K, V, eta, W0, dO, dW_out, dQ, dK, dV, deta, dW0, B, H, T,
                               d, C, dt, workspace, workspace_bytes, need);
  if (st != TTT_OK) return st;
  AssocBwdArgs a{Q, K, V, eta, eta_scalar, W0, dO, dW_out, dQ, dK, dV, deta, dW0, B, H, T, d, C,
                 workspace, workspace_bytes};
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_dual_bwd(a, ctx), msg);
}

size_t ttt_linear_dual_seg_bwd_workspace_size(int B, int H, int T, int d, int C, int dt,
                                              int segments) {
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0 || T % C != 0 || segments < 0 ||
      !dual_bwd_supported(d, C, dt))
    return 0;
  const int S = dual_seg_choose_segments(B, H, T, C, segments);
  return S < 1 ? 0 : dual_seg_bwd_workspace_bytes(B, H, T, d, S);
}

int ttt_linear_dual_seg_bwd(const void* Q, const void* K, const void* V, const float* eta,
                            float eta_scalar, const float* W0, const void* dO,
                            const float* dW_out, void* dQ, void* dK, void* dV, float* deta,
                            float* dW0, int B, int H, int T, int d, int C, int dt, int segments,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const std::string f("ttt_linear_dual_seg_bwd");
  int st = check_dual_bwd_args(f, Q, K, V, eta, W0, dO, dW_out, dQ, dK, dV, deta, dW0, B, H, T,
                               d, C, dt, workspace, workspace_bytes, 0);
  if (st != TTT_OK) return st;
  if (segments < 0) return fail(TTT_ERR_INVALID_ARG, f + ": segments must be >= 0");
  const int S = dual_seg_choose_segments(B, H, T, C, segments);
  if (S < 1)
    return fail(TTT_ERR_INVALID_ARG, f + ": segments must divide the number of chunks T / C");
  st = check_dual_bwd_args(f, Q, K, V, eta, W0, dO, dW_out, dQ, dK, dV, deta, dW0, B, H, T, d,
                           C, dt, workspace, workspace_bytes,
                           dual_seg_bwd_workspace_bytes(B, H, T, d, S));
  if (st != TTT_OK) return st;
  AssocBwdArgs a{Q, K, V, eta, eta_scalar, W0, dO, dW_out, dQ, dK, dV, deta, dW0, B, H, T, d, C,
                 workspace, workspace_bytes};
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_dual_seg_bwd(a, S, ctx), msg);
}

int ttt_assoc_state_fwd(const void* K, const void* V, const float* eta, float eta_scalar,
                        float* dS, int B, int H, int T, int d, int C, int dt,
                        cudaStream_t stream) {
  const std::string f("ttt_assoc_state_fwd");
  if (!K || !V || !dS) return fail(TTT_ERR_INVALID_ARG, f + ": K, V and dS must be non-null");
  if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || C <= 0)
    return fail(TTT_ERR_INVALID_ARG, f + ": B, H, T, d and C must be positive");
  if (T % C != 0) return fail(TTT_ERR_INVALID_ARG, f + ": T must be a multiple of C");
  if (dt != TTT_DTYPE_F32 && dt != TTT_DTYPE_BF16)
    return fail(TTT_ERR_INVALID_ARG, f + ": dtype must be TTT_DTYPE_F32 or TTT_DTYPE_BF16");
  const void* ptrs[] = {K, V, eta, dS};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, f + ": every device pointer must be 16-byte aligned");
  if (!assoc_supported(d, C, T, dt))
    return fail(TTT_ERR_UNSUPPORTED,
                f + ": supported bf16, d == 64 or 128, C == 16, 32 or 64, T % 64 == 0");
  const size_t nx = (size_t)B * H * T * d * 2, ns = (size_t)B * H * d * d * 4;
  const size_t ne = (size_t)B * H * T * 4;
  if (overlap(dS, ns, K, nx) || overlap(dS, ns, V, nx) || overlap(dS, ns, eta, ne))
    return fail(TTT_ERR_INVALID_ARG, f + ": dS must not overlap K, V or eta");
  StateArgs a{nullptr, K, V, eta, eta_scalar, nullptr, nullptr, dS, B, H, T, d, C, dt,
              nullptr, 0};
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_assoc_state(a, ctx), msg);
}

size_t inplace_ttt_workspace_size(int T, int Dff, int D, int C) {
  if (T <= 0 || Dff <= 0 || D <= 0 || C <= 0) return 0;
  return inplace_workspace_bytes(T, Dff, D, C);
}

int inplace_ttt_chunk_fwd(const void* Z, const void* Vhat, const void* W0, float eta, void* O,
                          float* W_out, int T, int Dff, int D, int C, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
  const char* f = "inplace_ttt_chunk_fwd";
  if (!Z || !Vhat || !W0 || !O || !W_out)
    return fail(TTT_ERR_INVALID_ARG, std::string(f) + ": Z, Vhat, W0, O, W_out must be non-null");
  if (T <= 0 || Dff <= 0 || D <= 0 || C <= 0)
    return fail(TTT_ERR_INVALID_ARG, std::string(f) + ": T, Dff, D and C must be positive");
  if (T % C != 0) return fail(TTT_ERR_INVALID_ARG, std::string(f) + ": T must be a multiple of C");
  const void* ptrs[] = {Z, Vhat, W0, O, W_out, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, std::string(f) + ": pointers must be 16-byte aligned");
  std::string why;
  if (!inplace_supported(T, Dff, D, C, &why))
    return fail(TTT_ERR_UNSUPPORTED, std::string(f) + ": " + why);
  const size_t nz = (size_t)T * Dff * 2, nv = (size_t)T * D * 2, nw = (size_t)Dff * D * 2;
  const size_t no = (size_t)T * D * 2, nwo = (size_t)Dff * D * 4;
  const void* ins[] = {Z, Vhat, W0};
  const size_t nin[] = {nz, nv, nw};
  for (int i = 0; i < 3; ++i)
    if (overlap(O, no, ins[i], nin[i]) || overlap(W_out, nwo, ins[i], nin[i]) ||
        overlap(workspace, workspace_bytes, ins[i], nin[i]))
      return fail(TTT_ERR_INVALID_ARG, std::string(f) + ": outputs/workspace overlap an input");
  if (overlap(O, no, W_out, nwo) || overlap(workspace, workspace_bytes, O, no) ||
      overlap(workspace, workspace_bytes, W_out, nwo))
    return fail(TTT_ERR_INVALID_ARG, std::string(f) + ": outputs/workspace overlap");
  const size_t need = inplace_workspace_bytes(T, Dff, D, C);
  if (need && (!workspace || workspace_bytes < need))
    return fail(TTT_ERR_WORKSPACE, std::string(f) + ": workspace of at least " +
                                       std::to_string(need) + " bytes required");
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  InplaceArgs a{Z, Vhat, W0, eta, O, W_out, T, Dff, D, C, workspace, workspace_bytes};
  return finish(launch_inplace(a, ctx), msg);
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static int check_lm_shapes(const std::string& f, int T, int Dm, int D, int k) {
  if (T <= 0 || Dm <= 0 || D <= 0 || k <= 0)
    return fail(TTT_ERR_INVALID_ARG, f + ": T, Dm, D and k must be positive");
  if (T % 128 != 0 || Dm % 128 != 0 || D % 64 != 0 || k > 8)
    return fail(TTT_ERR_UNSUPPORTED,
                f + ": supported T % 128 == 0, Dm % 128 == 0, D % 64 == 0, 1 <= k <= 8");
  if ((long long)T * std::max(Dm, D) >= (1ll << 40))
    return fail(TTT_ERR_UNSUPPORTED, f + ": too large");
  return TTT_OK;
}

size_t ttt_lm_target_workspace_size(int T, int Dm, int D, int k) {
  if (T <= 0 || Dm <= 0 || D <= 0 || k <= 0) return 0;
  return lm_target_workspace_bytes(T, Dm, D, k);
}

int ttt_lm_target_fwd(const void* X, const float* Wc, const void* Wp, void* Vhat, int T, int Dm,
                      int D, int k, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream) {
  const std::string f("ttt_lm_target_fwd");
  if (!X || !Wc || !Wp || !Vhat)
    return fail(TTT_ERR_INVALID_ARG, f + ": X, Wc, Wp and Vhat must be non-null");
  int st = check_lm_shapes(f, T, Dm, D, k);
  if (st != TTT_OK) return st;
  const void* ptrs[] = {X, Wc, Wp, Vhat, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, f + ": pointers must be 16-byte aligned");
  const size_t need = lm_target_workspace_bytes(T, Dm, D, k);
  if (!workspace || workspace_bytes < need)
    return fail(TTT_ERR_WORKSPACE, f + ": workspace of at least " + std::to_string(need) +
                                       " bytes required");
  const size_t nx = (size_t)T * Dm * 2, nc = (size_t)k * Dm * 4, np = (size_t)Dm * D * 2;
  const size_t nv = (size_t)T * D * 2;
  const void* ins[] = {X, Wc, Wp};
  const size_t nin[] = {nx, nc, np};
  for (int i = 0; i < 3; ++i)
    if (overlap(Vhat, nv, ins[i], nin[i]) || overlap(workspace, workspace_bytes, ins[i], nin[i]))
      return fail(TTT_ERR_INVALID_ARG, f + ": output/workspace overlap an input");
  if (overlap(Vhat, nv, workspace, workspace_bytes))
    return fail(TTT_ERR_INVALID_ARG, f + ": output overlaps the workspace");
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  return finish(launch_lm_target(X, Wc, Wp, Vhat, T, Dm, D, k, workspace, workspace_bytes, ctx),
                msg);
}

size_t inplace_ttt_lm_workspace_size(int T, int Dff, int D, int Dm, int C, int k) {
  if (T <= 0 || Dff <= 0 || D <= 0 || Dm <= 0 || C <= 0 || k <= 0 || T % C != 0) return 0;
  return align256(lm_target_workspace_bytes(T, Dm, D, k)) + align256((size_t)T * D * 2) +
         inplace_workspace_bytes(T, Dff, D, C);
}

int inplace_ttt_lm_chunk_fwd(const void* Z, const void* X, const float* Wc, const void* Wp,
                             const void* W0, float eta, void* O, float* W_out, int T, int Dff,
                             int D, int Dm, int C, int k, void* workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
  const std::string f("inplace_ttt_lm_chunk_fwd");
  if (!Z || !X || !Wc || !Wp || !W0 || !O || !W_out)
    return fail(TTT_ERR_INVALID_ARG, f + ": every pointer but the workspace must be non-null");
  int st = check_lm_shapes(f, T, Dm, D, k);
  if (st != TTT_OK) return st;
  if (Dff <= 0 || C <= 0 || T % C != 0)
    return fail(TTT_ERR_INVALID_ARG, f + ": Dff and C must be positive, T a multiple of C");
  std::string why;
  if (!inplace_supported(T, Dff, D, C, &why)) return fail(TTT_ERR_UNSUPPORTED, f + ": " + why);
  const void* ptrs[] = {Z, X, Wc, Wp, W0, O, W_out, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(TTT_ERR_INVALID_ARG, f + ": pointers must be 16-byte aligned");
  const size_t need = inplace_ttt_lm_workspace_size(T, Dff, D, Dm, C, k);
  if (!workspace || workspace_bytes < need)
    return fail(TTT_ERR_WORKSPACE, f + ": workspace of at least " + std::to_string(need) +
                                       " bytes required");
  const size_t sizes_in[] = {(size_t)T * Dff * 2, (size_t)T * Dm * 2, (size_t)k * Dm * 4,
                             (size_t)Dm * D * 2, (size_t)Dff * D * 2};
  const void* ins[] = {Z, X, Wc, Wp, W0};
  const size_t no = (size_t)T * D * 2, nwo = (size_t)Dff * D * 4;
  for (int i = 0; i < 5; ++i)
    if (overlap(O, no, ins[i], sizes_in[i]) || overlap(W_out, nwo, ins[i], sizes_in[i]) ||
        overlap(workspace, workspace_bytes, ins[i], sizes_in[i]))
      return fail(TTT_ERR_INVALID_ARG, f + ": outputs/workspace overlap an input");
  if (overlap(O, no, W_out, nwo) || overlap(workspace, workspace_bytes, O, no) ||
      overlap(workspace, workspace_bytes, W_out, nwo))
    return fail(TTT_ERR_INVALID_ARG, f + ": outputs/workspace overlap");
  std::string msg;
  unsigned* err = device_error_word(&msg);
  if (!err) return fail(TTT_ERR_CUDA, msg);
  LaunchCtx ctx{stream, err, &msg};
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t lm = align256(lm_target_workspace_bytes(T, Dm, D, k));
  void* Vhat = ws + lm;
  const size_t vb = align256((size_t)T * D * 2);
  int r = launch_lm_target(X, Wc, Wp, Vhat, T, Dm, D, k, ws, lm, ctx);
  if (r != kOk) return finish(r, msg);
  InplaceArgs a{Z, Vhat, W0, eta, O, W_out, T, Dff, D, C, ws + lm + vb,
                workspace_bytes - lm - vb};
  return finish(launch_inplace(a, ctx), msg);
}

}  // extern "C"
