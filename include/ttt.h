/*
 * ttt.h - C ABI of the B200 (sm_100a) fast-weight update-and-read library (libttt_b200.so).
 *
 * Three operations, each the chunked update-and-read of a fast-weight state whose inner model is
 * linear and bias-free:
 *
 *   ttt_linear_dual_fwd    TTT-Linear, mini-batch dual form.
 *                          Source: "RNN의 기억을 작은 모델로 바꾼다면: Test-Time Training 읽기"
 *                          (a reading of "Learning to (Learn at Test Time)"), section
 *                          "gradient를 효율적인 layer로 만드는 작업" (mini-batch TTT and its dual
 *                          form) and section "읽는 동안 문제를 하나 더 푼다" (per-token rule, output
 *                          read from the updated model).
 *   ttt_assoc_scan_fwd     weight-norm-free, gradient-ascent linear-attention form, computed
 *                          chunk-parallel with a prefix scan over chunk states.
 *                          Source: "KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다"
 *                          (one-step closed form o = q(S0 + k^T v); removing weight normalisation
 *                          restores associativity and allows a parallel prefix scan; per-token
 *                          learning rates fold into the values; gradient ascent).
 *   inplace_ttt_chunk_fwd  In-Place TTT: W_down of a gated MLP as the fast weight, one step per
 *                          chunk, deltas combined by a prefix sum.
 *                          Source: "In-Place 테스트 시점 학습: LLM을 위한 원활한 동적 적응 프레임워크"
 *                          (gated-MLP paragraph, chunk-update paragraph, associative-scan
 *                          paragraph).
 *
 * Around them, declared below in this order: the dual form evaluated sequence-parallel
 * (ttt_linear_dual_seg_fwd), the associative mode with a momentum inner loop, the backwards of
 * both modes (and of the sequence-parallel dual form), the context-parallel pieces (a slice's
 * state increment and their prefix for the associative mode; a slice's affine maps and their
 * ordered fold for the dual form), an allocation-free In-Place entry point, and the LM-aligned
 * target of the In-Place update.
 *
 * Conventions shared by every entry point
 *   - Row vectors: q_t, k_t, v_t are 1 x d; the state W (or S) is d x d laid out [d_in][d_out]
 *     (row-major), and a token reads o_t = q_t W.
 *   - Tensors [B,H,T,d] are contiguous row-major; stream (b,h) owns rows (b*H+h)*T .. +T-1.
 *   - All pointers except host-side scalars are DEVICE pointers owned by the caller. The library
 *     allocates no device memory of its own and never synchronises: all work is enqueued on
 *     `stream` (0 = the legacy default stream) in order. Scratch memory is the caller's
 *     `workspace` of at least the size the matching *_workspace_size() returns.
 *   - Errors that the host can detect (null or misaligned pointers, bad sizes, unsupported
 *     shapes, short workspace) return a status BEFORE anything is launched; outputs are then
 *     untouched. A failed launch returns TTT_ERR_CUDA. Details of the last error of the calling
 *     thread are in ttt_last_error_message().
 *   - Every device pointer must be 16-byte aligned.
 *   - Outputs must not overlap inputs, except the documented state aliasing (W_out == W0,
 *     S_out == S0 is allowed: the state is read before it is written).
 *   - Numerics: bf16 operands go through the tensor cores with fp32 accumulation; the state is
 *     kept in fp32; outputs O are rounded (nearest-even) to the input dtype; final states are
 *     fp32. fp32 inputs use an exact-fp32 CUDA-core path (no TF32).
 */
#ifndef TTT_B200_TTT_H
#define TTT_B200_TTT_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTT_OK = 0,
  TTT_ERR_INVALID_ARG = 1, /* null/misaligned pointer, non-positive size, T % C != 0, bad dtype */
  TTT_ERR_UNSUPPORTED = 2, /* valid but not implemented: head dim, chunk size, dtype combination */
  TTT_ERR_WORKSPACE = 3,   /* workspace pointer null or smaller than *_workspace_size() */
  TTT_ERR_CUDA = 4,        /* a CUDA call or kernel launch failed */
  TTT_ERR_TIMEOUT = 5      /* reserved; a bounded device-side wait that gives up is reported
                              through ttt_read_device_error(), not as a status */
} ttt_status_t;

typedef enum { TTT_DTYPE_F32 = 0, TTT_DTYPE_BF16 = 1 } ttt_dtype_t;

/* Static, human-readable name of a status code. */
const char* ttt_status_string(int status);

/* Detail of the last non-OK status returned on the calling thread ("" if none). */
const char* ttt_last_error_message(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int ttt_version(void);

/* Number of kernels this library has launched in this process (all entry points, all devices). */
uint64_t ttt_launch_count(void);

/* Kernel-variant choices, process-wide, for comparing variants (0 = the library's automatic
 * choice, the default). Keys:
 *   "dual_column_split"  CTAs per stream of the dual form: 1, 2 or 4 (4 only for d = 64).
 *   "dual_kernel"        dual form with bf16 inputs and C = 16: 1 = all products on warp MMAs
 *                        (one warp per 16 columns), 2 = the same on chain/output warp pairs,
 *                        3 = chain on warp MMAs with the outputs per 128-token stage on the
 *                        tcgen05 tensor cores (d = 64 only; what 0 picks for d = 64),
 *                        4 = the same with the chain and the outputs on separate SMs of a
 *                        thread-block cluster (d = 64, C = 16, where the streams leave one
 *                        more SM per one or two streams; measured slower than 3),
 *                        5 = the state resident in TMEM, updated once per 128-token stage on
 *                        tcgen05, with the chain reduced to 16 x 16 key-Gram-block updates
 *                        (d = 64, C = 16, 32 or 64), 6 = the same substitution with the state
 *                        in registers and its products on warp MMAs, the data-only products
 *                        on tcgen05 (d = 64, C = 16, 32 or 64).
 *   "dual_cluster_streams"  dual_kernel 4: streams per cluster, 1 or 2 (each cluster adds one
 *                        output CTA).
 *   "dual_warp_cols"     d = 64 with C = 16: 8 or 16 output columns per warp, for dual_kernel
 *                        1 and for the stage kernel (dual_kernel 3; by default 16 with one CTA
 *                        per stream, 8 when a stream is split over several CTAs).
 *   "dual_stage_chunks"  dual_kernel 1 with d = 64 and 8 columns per warp: 4 or 8 chunks per
 *                        pipeline stage.
 *   "assoc_parts"        superchunks per stream of the associative mode (must divide T / C).
 *   "wait_limit_ns"      limit, in ns, of every pipeline wait of the dual form's d = 64
 *                        kernels (dual_kernel 2 and 3; 0 = 4 s). A wait that runs out sets bit 0 of the
 *                        device error word and the kernel returns early with incomplete outputs
 *                        (see ttt_read_device_error); waits for copies already in flight keep
 *                        a fixed one-second limit, so nothing is left running.
 *   "inplace_chunks_per_launch"  In-Place update: 1 = one chunk per launch; 0 or 2 = two
 *                        chunks per launch where the shape allows it (D % 256 == 0, C % 256 == 0),
 *                        chunk i+1's read corrected by eta (Z_(i+1) Z_i^T) Vhat_i.
 *   "momentum_form"      ttt_assoc_momentum_fwd: 0 = one pass carrying (S, M) (every beta in
 *                        [0, 1]); 1 = plain + decayed associative passes (beta in [0.25, 0.9]).
 *   "assoc_bwd_form"     ttt_assoc_scan_bwd: 0 = dV and dK in one reverse pass; 1 = two
 *                        separate reverse passes.
 *   "dual_bwd_form"      ttt_linear_dual_bwd, d = 64: 0 = stage form (the forward's residuals
 *                        and stage-start states from the stage kernel's state-only chain, then
 *                        the state gradient's chain on warp MMAs and every product that needs
 *                        the forward states on tcgen05, per 128-token stage); 1 = one kernel
 *                        that recomputes every chunk-start state in a forward sweep, then runs
 *                        the reverse sweep on warp MMAs; 2 = the chunk-start states from the
 *                        stage kernel's chain, then that reverse sweep.
 * Every variant computes the same operation within the same tolerance. ttt_set_tuning returns
 * TTT_ERR_INVALID_ARG for an unknown key or a negative value; ttt_get_tuning returns -1 for an
 * unknown key; ttt_reset_tuning restores every key to 0. Not synchronised with calls in flight
 * on other threads: set choices before the calls they should affect. */
int ttt_set_tuning(const char* key, int value);
int ttt_get_tuning(const char* key);
void ttt_reset_tuning(void);

/* Reads and clears the current device's error word. Bit 0 set means a bounded device-side wait
 * gave up (a kernel stopped early; its outputs are incomplete). SYNCHRONOUS: waits for all work
 * on the device to finish. Returns TTT_OK or TTT_ERR_CUDA. */
int ttt_read_device_error(unsigned* value);

/* --------------------------------------------------------------------------------------------
 * TTT-Linear, mini-batch dual form (per stream (b,h), W = W0, for each chunk c of C tokens):
 *     G   = K_c W - V_c                                  residual of 1/2||k W - v||^2
 *     O_c = Q_c W - (tril(Q_c K_c^T) diag(eta_c)) G      tril includes the diagonal
 *     W   = W - K_c^T diag(eta_c) G
 *
 *  Q, K, V   [B,H,T,d] of dtype `dt` (fp32 or bf16).
 *  eta       [B,H,T] fp32 per-token learning rates, or NULL to use `eta_scalar` for every token.
 *            A learning rate scales its own (source) token's gradient.
 *  W0        [B,H,d,d] fp32 initial state, or NULL for zeros.
 *  O         [B,H,T,d] of dtype `dt` (output).
 *  W_out     [B,H,d,d] fp32 final state (output); may be the same pointer as W0.
 *  Supported: d in {32, 64, 128}; 1 <= C <= 64; T % C == 0. bf16 runs on tensor cores for
 *  C == 16 with d in {32, 64, 128} and for C in {32, 64} with d == 64 (d == 64: the chain on
 *  warp MMAs, the outputs per 128-token stage on tcgen05); other supported shapes run the
 *  CUDA-core path.
 *  Workspace: none (ttt_linear_dual_workspace_size returns 0; `workspace` may be NULL).
 * ------------------------------------------------------------------------------------------ */
size_t ttt_linear_dual_workspace_size(int B, int H, int T, int d, int C, int dt);
int ttt_linear_dual_fwd(const void* Q, const void* K, const void* V, const float* eta,
                        float eta_scalar, const float* W0, void* O, float* W_out, int B, int H,
                        int T, int d, int C, int dt, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * Sequence-parallel dual form (the segment-affine scan). Same operation, arguments, layouts
 * and results as ttt_linear_dual_fwd, evaluated differently: without weight normalisation the
 * chunk update W' = (I - K^T diag(eta) K) W + K^T diag(eta) V is affine in W ("KV 바인딩 기반
 * 테스트 시간 학습은 사실상 선형 어텐션이다", associativity paragraph), so each stream is cut
 * into `segments` segments of T / segments tokens whose maps W_end = A_s W_start + B_s are
 * computed in parallel (two dual-form passes over the segments, from W = 0 and W = I), folded in
 * order in fp32 to give every segment's start state, and a third pass produces O and W_out.
 * Three passes of work over segments-times as many chains: for few streams (B*H well below
 * the SM count) and long sequences.
 *  segments: 0 picks the count (the most segments that keep B*H*segments chains within the SM
 *  count, at least 4, else 1 = the sequential kernel); otherwise it must divide T / C.
 *  Workspace: ttt_linear_dual_seg_workspace_size() bytes (5 fp32 d x d states per segment;
 *  0 when the choice is 1). Returns TTT_ERR_INVALID_ARG when segments does not divide T / C.
 * ------------------------------------------------------------------------------------------ */
size_t ttt_linear_dual_seg_workspace_size(int B, int H, int T, int d, int C, int dt,
                                          int segments);
int ttt_linear_dual_seg_fwd(const void* Q, const void* K, const void* V, const float* eta,
                            float eta_scalar, const float* W0, void* O, float* W_out, int B,
                            int H, int T, int d, int C, int dt, int segments, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * Associative (gradient-ascent, weight-norm-free) linear-attention mode, per stream:
 *     S_t = S_(t-1) + eta_t k_t^T v_t,   o_t = q_t S_t      (S_0 = S0)
 *  computed per chunk of C tokens as O_c = Q_c S + (tril(Q_c K_c^T) diag(eta_c)) V_c,
 *  S += K_c^T diag(eta_c) V_c, with a two-pass prefix scan over superchunk states.
 *
 *  Q, K, V, O [B,H,T,d]; eta [B,H,T] fp32 or NULL (eta_scalar); S0 [B,H,d,d] fp32 or NULL
 *  (zeros); S_out [B,H,d,d] fp32, may equal S0.
 *  Supported: bf16, d == 64 or 128, C == 16, 32 or 64, T % 64 == 0 (tensor-core path). The
 *  result does not depend on C (the recurrence is per token; C only sets the evaluation
 *  granularity): every C is evaluated in 64-token tiles, and d = 64 runs zero-padded to 128
 *  inside the kernel, at the cost of d = 128 arithmetic for half the bytes.
 *  Workspace: ttt_assoc_scan_workspace_size() bytes (superchunk states, fp32).
 * ------------------------------------------------------------------------------------------ */
size_t ttt_assoc_scan_workspace_size(int B, int H, int T, int d, int C, int dt);
int ttt_assoc_scan_fwd(const void* Q, const void* K, const void* V, const float* eta,
                       float eta_scalar, const float* S0, void* O, float* S_out, int B, int H,
                       int T, int d, int C, int dt, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * Associative mode with a momentum inner loop ("KV 바인딩 기반 테스트 시간 학습은 사실상 선형
 * 어텐션이다", momentum paragraph: with momentum SGD the layer remains a weighted sum of
 * linear-attention terms), per stream:
 *     M_t = beta M_(t-1) + eta_t k_t^T v_t,   S_t = S_(t-1) + M_t,   o_t = q_t S_t
 *  (M_0 = M0, S_0 = S0; the rate scales each token's gradient before it enters the momentum).
 *  Q, K, V, O [B,H,T,d] bf16; eta [B,H,T] fp32 or NULL (eta_scalar); S0, M0 [B,H,d,d] fp32 or
 *  NULL (zeros); S_out, M_out [B,H,d,d] fp32 (S_out may equal S0, M_out may equal M0).
 *  beta in [0, 1] (beta = 0 is ttt_assoc_scan_fwd; beta = 1 makes M the running sum of the
 *  updates). Supported: as ttt_assoc_scan_fwd (bf16, d == 64 or 128, C == 16, 32 or 64,
 *  T % 64 == 0). Workspace: ttt_assoc_momentum_workspace_size() bytes (enough for either form).
 *  Runs as one pass that carries both states through 64-token chunks: inside a chunk every
 *  token pair is weighted by w(n) = sum_{r<=n} beta^r, formed directly, so the accuracy does not
 *  depend on beta; long sequences are cut into superchunks whose (S, M) maps are composed in
 *  sequence order (see assoc_mom.cu). The tuning key "momentum_form" = 1 selects the two-pass
 *  comparison form instead (a plain and a decayed associative pass combined in the output
 *  stage; beta in [0.25, 0.9], since it subtracts outputs of size ~1/(1 - beta)).
 * ------------------------------------------------------------------------------------------ */
size_t ttt_assoc_momentum_workspace_size(int B, int H, int T, int d, int C, int dt);
int ttt_assoc_momentum_fwd(const void* Q, const void* K, const void* V, const float* eta,
                           float eta_scalar, float beta, const float* S0, const float* M0,
                           void* O, float* S_out, float* M_out, int B, int H, int T, int d,
                           int C, int dt, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * Backward of the associative mode (the gradients that outer-loop training of the layer needs,
 * "KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다": the layer is trained end to end
 * through its inner updates). For the forward above and a scalar loss L with
 *     dL/dO = dO,   dL/dS_out = dS_out,
 *  returns dQ = dL/dQ, dK, dV, deta (per token) and dS0. With A_t = dS_out + sum_{u>=t} q_u^T dO_u:
 *     dq_t = dO_t S_t^T,  dv_t = eta_t k_t A_t,  dk_t = eta_t v_t A_t^T,  deta_t = k_t A_t v_t^T,
 *     dS0 = A_0.
 *  Q, K, V, dO [B,H,T,d] bf16; eta [B,H,T] fp32 or NULL (eta_scalar for every token); S0 and
 *  dS_out [B,H,d,d] fp32 or NULL (zeros). Outputs: dQ, dK, dV [B,H,T,d] bf16; deta [B,H,T]
 *  fp32 (per token also when eta is NULL: the scalar's gradient is their sum); dS0 [B,H,d,d]
 *  fp32. Outputs must not overlap the inputs or each other.
 *  Supported: as ttt_assoc_scan_fwd (bf16, d == 64 or 128, C == 16, 32 or 64, T % 64 == 0).
 *  C is the evaluation granularity; the gradients do not depend on it beyond rounding.
 *  Workspace: ttt_assoc_scan_bwd_workspace_size() bytes.
 *  Runs as one pass of the forward kernel for dQ (forward order), one reverse-order pass that
 *  carries the state gradient and writes dK and the unscaled dV (see assoc_yz.cu), and one
 *  elementwise pass (dV = eta Y, deta). The tuning key "assoc_bwd_form" = 1 runs dV and dK as
 *  two separate reverse passes of the forward kernel instead.
 * ------------------------------------------------------------------------------------------ */
size_t ttt_assoc_scan_bwd_workspace_size(int B, int H, int T, int d, int C, int dt);
int ttt_assoc_scan_bwd(const void* Q, const void* K, const void* V, const float* eta,
                       float eta_scalar, const float* S0, const void* dO, const float* dS_out,
                       void* dQ, void* dK, void* dV, float* deta, float* dS0, int B, int H,
                       int T, int d, int C, int dt, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * Backward of the TTT-Linear dual form ("RNN의 기억을 작은 모델로 바꾼다면: Test-Time Training
 * 읽기", section "gradient를 효율적인 layer로 만드는 작업": the mini-batch inner updates are part
 * of the layer and are differentiated with it in outer-loop training). For ttt_linear_dual_fwd
 * and a scalar loss L with dL/dO = dO and dL/dW_out = dW_out, returns dQ, dK, dV, deta (per
 * token) and dW0. Per chunk, with X the gradient of the state after the chunk (dW_out after the
 * last), W the chunk-start state, G = K W - V and A = tril(Q K^T) diag(eta):
 *     dG = -A^T dO - diag(eta) K X,   dV = -dG,   dA = -tril(dO G^T),   dS = dA diag(eta),
 *     dQ = dO W^T + dS K,   dK = dS^T Q - diag(eta) G X^T + dG W^T,
 *     deta_s = sum_t dA[t,s] (Q K^T)[t,s] - (K X)_s . G_s,   X <- X + Q^T dO + K^T dG;
 *  dW0 is X after the first chunk.
 *  Q, K, V, dO [B,H,T,d] bf16; eta [B,H,T] fp32 or NULL (eta_scalar for every token); W0 and
 *  dW_out [B,H,d,d] fp32 or NULL (zeros). Outputs: dQ, dK, dV [B,H,T,d] bf16; deta [B,H,T]
 *  fp32 (per token also when eta is NULL); dW0 [B,H,d,d] fp32. Outputs and workspace must not
 *  overlap the inputs or each other.
 *  Supported: bf16, C == 16, d in {32, 64, 128}, T % C == 0 (C changes the result: it is the
 *  mini-batch size of the forward).
 *  Workspace: ttt_linear_dual_bwd_workspace_size() bytes (d = 32, 128: one bf16 d x d state per
 *  chunk, B*H*(T/16)*d*d*2; d = 64: the larger of that and the stage form's G and -diag(eta) G
 *  rows plus one bf16 d x d state per 128 tokens, B*H*(4*T*d + ceil(T/128)*2*d*d)). A forward
 *  recompute fills the workspace, then the reverse pass forms the gradients. d = 64 (stage form,
 *  dual_bwd_tc.cu): the forward stage kernel's state-only chain writes G, -diag(eta) G and the
 *  stage-start states; the reverse pass keeps the state gradient's chain on warp MMAs and forms
 *  every product that needs the forward states per 128-token stage on tcgen05. d = 32, 128
 *  (dual_bwd.cu): one kernel, a forward sweep of chunk-start states then a reverse sweep of the
 *  chunk adjoint. The tuning key "dual_bwd_form" selects the other d = 64 forms.
 * ------------------------------------------------------------------------------------------ */
size_t ttt_linear_dual_bwd_workspace_size(int B, int H, int T, int d, int C, int dt);
int ttt_linear_dual_bwd(const void* Q, const void* K, const void* V, const float* eta,
                        float eta_scalar, const float* W0, const void* dO, const float* dW_out,
                        void* dQ, void* dK, void* dV, float* deta, float* dW0, int B, int H,
                        int T, int d, int C, int dt, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * Backward of the sequence-parallel dual form: the gradients of ttt_linear_dual_bwd (same
 * arguments, layouts, results up to rounding, support and errors) evaluated over `segments`
 * segments per stream. The state gradient X follows its own affine recurrence, in reverse and
 * free of W: X_before = (I - K^T diag(eta) K) X_after + Q^T dO - K^T A^T dO per chunk, so a
 * segment maps X_before = A_s^T X_after + N_s with the forward's A_s. The library computes the
 * forward maps and segment start states (as ttt_linear_dual_seg_fwd), the offsets N_s (a
 * backward pass over the segments from X_after = 0), every segment's X_after (a reverse fold),
 * and then the gradients (a second backward pass over the segments).
 *  segments: 0 picks the count as ttt_linear_dual_seg_fwd does (1 = ttt_linear_dual_bwd);
 *  otherwise it must divide T / C (else TTT_ERR_INVALID_ARG).
 *  Workspace: ttt_linear_dual_seg_bwd_workspace_size() bytes.
 * ------------------------------------------------------------------------------------------ */
size_t ttt_linear_dual_seg_bwd_workspace_size(int B, int H, int T, int d, int C, int dt,
                                              int segments);
int ttt_linear_dual_seg_bwd(const void* Q, const void* K, const void* V, const float* eta,
                            float eta_scalar, const float* W0, const void* dO,
                            const float* dW_out, void* dQ, void* dK, void* dV, float* deta,
                            float* dW0, int B, int H, int T, int d, int C, int dt, int segments,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * Context parallelism of the dual form (the segment-affine maps of ttt_linear_dual_seg_fwd, one
 * segment per rank; orchestration in weight_linear_attention_ttt_b200/context_parallel.py):
 *
 * ttt_linear_dual_slice_maps: for a token slice of every stream (K, V [B,H,T,d], eta [B,H,T]
 *  or NULL with eta_scalar), the affine map of its chunk updates, W_end = A W_start + B:
 *  B_out = the end state from W = 0, A_out = the end state from W = I minus B_out
 *  ([B,H,d,d] fp32 each). Workspace: ttt_linear_dual_slice_maps_workspace_size() bytes. Same
 *  support as ttt_linear_dual_fwd (d in {32, 64, 128}, C <= 64, fp32 or bf16).
 * ttt_dual_state_fold: W_out = the state after applying maps 0 .. upto-1 in order to W0 (NULL:
 *  zeros): W <- A_m W + B_m, with A_maps and B_maps [n_maps][B,H,d,d] fp32 (the all-gathered
 *  layout). 0 <= upto <= n_maps; W_out may equal W0. fp32 throughout.
 * ------------------------------------------------------------------------------------------ */
size_t ttt_linear_dual_slice_maps_workspace_size(int B, int H, int T, int d, int C, int dt);
int ttt_linear_dual_slice_maps(const void* K, const void* V, const float* eta, float eta_scalar,
                               float* A_out, float* B_out, int B, int H, int T, int d, int C,
                               int dt, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);
int ttt_dual_state_fold(const float* W0, const float* A_maps, const float* B_maps, int n_maps,
                        int upto, float* W_out, int B, int H, int d, cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * State increment of a sequence slice in the associative mode (the first pass of the prefix
 * scan over states, "KV 바인딩 기반 테스트 시간 학습은 사실상 선형 어텐션이다", associativity
 * paragraph; per-chunk deltas combined by a prefix sum for context parallelism, "In-Place
 * 테스트 시점 학습", associative-scan paragraph):
 *     dS = sum_t eta_t k_t^T v_t  over the T tokens given
 *  K, V [B,H,T,d]; eta [B,H,T] fp32 or NULL (eta_scalar); dS [B,H,d,d] fp32 output.
 *  A context-parallel caller gives each device a slice of the sequence, exchanges the slices'
 *  increments, and starts ttt_assoc_scan_fwd on its slice from S0 plus the earlier slices'
 *  increments. Supported: as ttt_assoc_scan_fwd. No workspace.
 * ------------------------------------------------------------------------------------------ */
int ttt_assoc_state_fwd(const void* K, const void* V, const float* eta, float eta_scalar,
                        float* dS, int B, int H, int T, int d, int C, int dt,
                        cudaStream_t stream);

/* Prefix combination of per-slice state increments: out = S0 + sum_{r < upto} increments[r].
 *  S0 [B,H,d,d] fp32 or NULL (zeros); increments [n_increments][B,H,d,d] fp32 (e.g. gathered
 *  from all devices); out [B,H,d,d] fp32, may equal S0, must not overlap the increments.
 *  With upto = this device's slice index it gives the slice's starting state; with
 *  upto = n_increments, the state after the whole sequence. */
int ttt_state_prefix_sum(const float* S0, const float* increments, int n_increments, int upto,
                         int B, int H, int d, float* out, cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * In-Place TTT, W_down chunk update (W = W0; for each chunk i of C tokens, in order):
 *     O_i = Z_i W                  (W holds W0 plus the deltas of the chunks before i)
 *     W   = W + eta Z_i^T Vhat_i
 *
 *  Z     [T,Dff] bf16 activations (the gated-MLP hidden state).
 *  Vhat  [T,D]  bf16 targets.
 *  W0    [Dff,D] bf16 initial W_down.
 *  O     [T,D]  bf16 output.
 *  W_out [Dff,D] fp32 final W_down (the running fp32 master).
 *  Supported: T % C == 0; C % 128 == 0; Dff % 128 == 0; D % 64 == 0.
 *  Workspace: inplace_ttt_workspace_size() bytes (two bf16 copies of the running W, per-launch
 *  tile counters and, with two chunks per launch, the C x C bf16 correction eta Z_(i+1) Z_i^T).
 * ------------------------------------------------------------------------------------------ */
size_t inplace_ttt_workspace_size(int T, int Dff, int D, int C);
int inplace_ttt_chunk_fwd(const void* Z, const void* Vhat, const void* W0, float eta, void* O,
                          float* W_out, int T, int Dff, int D, int C, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * Allocation-free In-Place W_down update. The pages have no counterpart: this is an interface
 * for callers that cannot provide a workspace, such as host runtimes that plan all device
 * memory up front and refuse allocations while serving, or plugin interfaces that pass only
 * input and output pointers.
 *
 *  Same computation, arguments and validation as inplace_ttt_chunk_fwd, minus the workspace:
 *  the scratch (two bf16 copies of W_down and one tile counter per chunk) is a static device
 *  array of inplace_ttt_noalloc_max_scratch_bytes() bytes (32 MiB) inside the library. Every
 *  GPU that loads the library holds that array until the process exits (with CUDA's lazy
 *  module loading, from this entry point's first call on that GPU).
 *  - Calls allocate nothing: no cudaMalloc, no cudaFree, no allocating library routine. The
 *    caller still provides Z, Vhat, W0, O and W_out.
 *  - Shapes whose scratch (inplace_ttt_workspace_size) exceeds the maximum return
 *    TTT_ERR_UNSUPPORTED before anything is launched, with the reason in
 *    ttt_last_error_message(). With T > C the need is about 4 * Dff * D + 2 * C * C bytes.
 *  - All calls share the one array and it keeps the previous call's contents; the tile counters
 *    are zeroed on `stream` at the start of every call, and the W copies are always written
 *    before they are read. Calls whose work overlaps on the GPU (different streams, or threads
 *    racing on one device) race on the array: serialise them.
 *  - The first call on each device looks up the array's device address (a one-time runtime
 *    query for the current device and its context; it is made again after a device reset,
 *    which gives the device a new context). Make that first call before any stream capture
 *    begins.
 *  - Errors name this function in ttt_last_error_message(); the shape, pointer and alignment
 *    checks are those of inplace_ttt_chunk_fwd.
 * ------------------------------------------------------------------------------------------ */
size_t inplace_ttt_noalloc_max_scratch_bytes(void);
int inplace_ttt_chunk_fwd_noalloc(const void* Z, const void* Vhat, const void* W0, float eta,
                                  void* O, float* W_out, int T, int Dff, int D, int C,
                                  cudaStream_t stream);

/* --------------------------------------------------------------------------------------------
 * LM-aligned target of the In-Place update ("In-Place 테스트 시점 학습", LM-aligned objective
 * paragraph: the target is made from the token embeddings by a 1D convolution and a projection
 * and carries the next token's information). Reading: a depthwise convolution over tokens whose
 * tap i multiplies token t + 1 - i (tokens outside [0, T) are zero), then a bias-free projection:
 *     Vhat[t, :] = (sum_i Wc[i, :] * X[t + 1 - i, :]) Wp
 *  X [T, Dm] bf16; Wc [k, Dm] fp32; Wp [Dm, D] bf16; Vhat [T, D] bf16 (output).
 *  Supported: T % 128 == 0, Dm % 128 == 0, D % 64 == 0, 1 <= k <= 8.
 *  Workspace: ttt_lm_target_workspace_size() bytes (the convolved embeddings, bf16).
 *  Errors: TTT_ERR_INVALID_ARG (null/misaligned/overlapping pointers), TTT_ERR_UNSUPPORTED
 *  (shape), TTT_ERR_WORKSPACE, TTT_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
size_t ttt_lm_target_workspace_size(int T, int Dm, int D, int k);
int ttt_lm_target_fwd(const void* X, const float* Wc, const void* Wp, void* Vhat, int T, int Dm,
                      int D, int k, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream);

/* The In-Place chunk update with its LM-aligned target formed in front of it: Vhat as above
 *  (into the workspace), then inplace_ttt_chunk_fwd(Z, Vhat, W0, eta, O, W_out, T, Dff, D, C).
 *  Arguments as for the two calls; workspace: inplace_ttt_lm_workspace_size() bytes. */
size_t inplace_ttt_lm_workspace_size(int T, int Dff, int D, int Dm, int C, int k);
int inplace_ttt_lm_chunk_fwd(const void* Z, const void* X, const float* Wc, const void* Wp,
                             const void* W0, float eta, void* O, float* W_out, int T, int Dff,
                             int D, int Dm, int C, int k, void* workspace, size_t workspace_bytes,
                             cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TTT_B200_TTT_H */
