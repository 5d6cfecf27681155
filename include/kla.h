/*
 * kla.h -- C ABI of the Kaczmarz Linear Attention (KLA) hot path on NVIDIA
 * B200 (sm_100a).  Library: libkla.so (delta_rule_linear_kla_b200/).
 *
 * The method (h = S^T is stored, one [dk][dv] fp32 matrix per head):
 *
 *   beta_t = eta_t / (||k_t||_2^2 + eps)
 *       -- "Kaczmarz Linear Attention" (arXiv 2605.08587 summary), Abstract:
 *          the key-norm-normalised step size of the Kaczmarz projection.
 *   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *   alpha_t = exp(g_t),   o_t = S_t q_t
 *       -- "Deep Dive into KDA", section 2.2 (Gated DeltaNet), which the KLA
 *          Abstract keeps except for beta; the erase factor is placed where
 *          S (dv x dk) type-checks, and o reads the updated state.
 *
 * Conventions shared by every call:
 *   * All tensors are device pointers, contiguous, row-major, 16-byte
 *     aligned, on the current device, in the layouts stated per argument
 *     (kla_chunk_fwd_host alone takes host pointers).
 *   * The caller owns every buffer (including any workspace).  The library
 *     allocates no device memory and never synchronises the stream: work is
 *     queued on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream) and returns immediately.
 *   * Arguments are validated on the host before anything is launched; a
 *     bad argument returns KLA_ERR_INVALID_ARG or KLA_ERR_UNSUPPORTED and
 *     leaves every buffer untouched.  A failed launch returns KLA_ERR_CUDA.
 *     No call aborts, throws or prints.
 *   * dtype selects the element type of q, k, v and o (KLA_BF16 or
 *     KLA_FP32); g, eta, states are always fp32.  Arithmetic is fp32
 *     (tensor-core products take bf16 operands with fp32 accumulation).
 */
#ifndef KLA_H_
#define KLA_H_

#include <stddef.h>

/* Every entry point below is exported from libkla.so; the rest is hidden. */
#if defined(__GNUC__)
#define KLA_API __attribute__((visibility("default")))
#else
#define KLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KLA_OK = 0,
    KLA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment, aliasing */
    KLA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d not 64/128) */
    KLA_ERR_CUDA = 3,         /* a CUDA runtime/driver call or launch failed   */
    KLA_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up            */
    KLA_ERR_BOUND = 5         /* a debug bound check found a violation         */
} kla_status;

typedef enum { KLA_BF16 = 0, KLA_FP32 = 1 } kla_dtype;

/* Chunk length of the chunkwise prefill ("Deep Dive into KDA", section 3:
 * the sequence is cut into chunks of C tokens).  Fixed at compile time. */
#define KLA_CHUNK 64

/*
 * Prefill forward (chunkwise parallel form, "Deep Dive into KDA", section 3).
 *
 *   q, k    [B][T][H][dk]  dtype       queries, keys (keys are NOT normalised;
 *                                      beta carries the key norm)
 *   v       [B][T][H][dv]  dtype       values
 *   g       [B][T][H]      fp32        log gate, alpha_t = exp(g_t)
 *   eta     [B][T][H]      fp32        relaxation eta_t of the Kaczmarz step
 *   eps                    fp32        added to ||k_t||^2 (KLA Abstract)
 *   h0      [B][H][dk][dv] fp32        initial state h = S^T; NULL = zeros
 *   o       [B][T][H][dv]  dtype       output, o_t = S_t q_t (written)
 *   hT      [B][H][dk][dv] fp32        final state (written); NULL = not
 *                                      returned.  hT may alias h0 exactly.
 *   chunk   must equal KLA_CHUNK (else KLA_ERR_UNSUPPORTED)
 *   workspace / ws_bytes: caller-owned device scratch of
 *     kla_chunk_fwd_workspace_size(...) bytes (NULL allowed when that is 0):
 *     the per-chunk factors (B * H * ceil(T / KLA_CHUNK) * 16384 bytes, the
 *     least accepted, else KLA_ERR_INVALID_ARG) followed either, for few
 *     heads and long sequences, by the states of the sequence segments the
 *     state chain is cut into (run in parallel).  A workspace smaller than
 *     the full size but holding the factors runs the chain uncut.  The
 *     factors are formed by a launch of their own before the chain.
 *     It must not overlap any other argument.
 *
 * Supported: B, H >= 1; T >= 0 (T = 0 copies h0 to hT); dk = dv in {64, 128}.
 * A ragged tail (T not a multiple of the chunk) is processed as if padded
 * with g = 0, eta = 0, which is an exact identity step.
 * o must not overlap any input.  bf16 runs the tcgen05 chunk kernel; fp32
 * runs the token-serial CUDA-core kernel (kla_recurrent_fwd).
 */
KLA_API size_t kla_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int dtype);

/*
 * Number of sequence segments the bf16 state chain of kla_chunk_fwd (and of
 * kla_chunk_state_fwd, kla_gdn_chunk_fwd) runs in for these sizes and a
 * workspace of ws_bytes: 1 = one pass over the whole sequence (one chain
 * kernel launch); S > 1 = the segment transitions of segments 0 .. S-2, a
 * start-state kernel, then the outputs of all S segments (three launches).
 * 0 when the bf16 chunk path does not apply (fp32 I/O, bad sizes).
 * Informational: the entry points choose by themselves.
 */
KLA_API int kla_chunk_fwd_segments(int B, int T, int H, int dk, int dv, int dtype,
                                   size_t ws_bytes);

/*
 * 1 when the bf16 kla_chunk_fwd of this shape would run as a single kernel
 * launch with a workspace of ws_bytes (the per-chunk factors formed beside
 * the state CTAs in one cooperative launch).  At present 0 for every shape:
 * that launch is built but not taken, after an intermittent launch failure
 * whose cause has not been found, so the factors are always formed by a
 * launch of their own first.  Host-only query.
 */
KLA_API int kla_chunk_fwd_single_launch(int B, int T, int H, int dk, int dv, int dtype,
                                        size_t ws_bytes);

KLA_API kla_status kla_chunk_fwd(const void *q, const void *k, const void *v,
                         const float *g, const float *eta, float eps,
                         const float *h0, void *o, float *hT,
                         int B, int T, int H, int dk, int dv, int chunk, int dtype,
                         void *workspace, size_t ws_bytes, void *stream);

/*
 * kla_chunk_fwd (bf16, same arguments, layouts and workspace) that also
 * writes the state at the start of every chunk: hs [B][H][ceil(T/64)]
 * [dk][dv] fp32, hs[b][h][n] = h after the first 64 n tokens (n = 0: h0, or
 * zeros), as the state kernel carries it (fp32 sums of bf16 products) -- the
 * checkpoints a training framework needs for its own backward.  o and hT
 * may be NULL (not written).  hs must be 16-byte aligned and disjoint from
 * every other argument; dtype KLA_FP32 -> KLA_ERR_UNSUPPORTED; T >= 1.
 */
KLA_API kla_status kla_chunk_fwd_states(const void *q, const void *k, const void *v,
                                        const float *g, const float *eta, float eps,
                                        const float *h0, void *o, float *hT, float *hs,
                                        int B, int T, int H, int dk, int dv, int dtype,
                                        void *workspace, size_t ws_bytes, void *stream);

/*
 * The two stages of the bf16 kla_chunk_fwd, callable on their own (same
 * layouts and conventions; kla_chunk_fwd is exactly the first call followed
 * by the second on the same stream).  dtype must be KLA_BF16 (KLA_FP32 ->
 * KLA_ERR_UNSUPPORTED); T >= 1; workspace as for kla_chunk_fwd.
 *
 * kla_chunk_ut_transform -- per chunk of KLA_CHUNK tokens ("Deep Dive into
 *   KDA", section 3, with the KLA step size of the KLA Abstract):
 *   beta_r = eta_r / (||k_r||^2 + eps), G_r = in-chunk inclusive cumsum of
 *   g, A_rs = beta_r (k_r . k_s) e^{G_r - G_s} (s < r), T = (I + A)^{-1};
 *   writes T diag(beta) and T diag(beta e^G) of every chunk (bf16, opaque
 *   layout) into the workspace.  Reads k [B][T][H][dk], g, eta [B][T][H].
 *   The workspace must not overlap k, g or eta.
 *
 * kla_chunk_state_fwd -- the inter-chunk state recurrence and the
 *   intra-chunk outputs from those factors: per chunk U = T diag(beta) V,
 *   W = T diag(beta e^G) K, V' = U - W h, o = e^G Q h + P V' (P the causal
 *   decayed Q K^T, diagonal included), h <- e^{G_last} h + K^T diag(e^{G_last
 *   - G}) V'.  Reads q, k, v, g (the same k and g the workspace was made
 *   from), h0 (NULL = zeros) and the workspace; writes o and hT (NULL = not
 *   returned, may alias h0).  It writes the workspace past the factors
 *   (the segment states) when ws_bytes is kla_chunk_fwd_workspace_size's;
 *   the factors themselves are left as they are.  No other argument may
 *   overlap the workspace.
 */
KLA_API kla_status kla_chunk_ut_transform(const void *k, const float *g, const float *eta,
                                  float eps, int B, int T, int H, int dk, int dtype,
                                  void *workspace, size_t ws_bytes, void *stream);

KLA_API kla_status kla_chunk_state_fwd(const void *q, const void *k, const void *v,
                               const float *g, const float *h0, void *o, float *hT,
                               int B, int T, int H, int dk, int dv, int dtype,
                               void *workspace, size_t ws_bytes, void *stream);

/*
 * kla_chunk_ut_transform with a debug check of its factors (same arguments
 * and workspace, plus `ratio_max`: one device float, 16-byte aligned,
 * disjoint from the rest).  The bound follows from the recurrence: with
 * k_s = ||k_s|| khat_s, T_rs (r > s) is -eta'_r (||k_s|| / ||k_r||)
 * e^{G_r - G_s} khat_r^T P khat_s, P a product of erase factors
 * (I - beta_j k_j k_j^T) that each have norm <= 1 when eta_j is in [0, 2]
 * (the Kaczmarz step of the KLA Abstract, over-relaxed up to 2), and
 * eta'_r = beta_r ||k_r||^2, so |T_rs| ||k_r|| / ||k_s|| <= eta'_r
 * e^{G_r - G_s}.  The call writes the largest ratio of the left side to the
 * right side over every entry the kernel forms (entries below 1e-30 are
 * skipped) into *ratio_max, and when it exceeds 1.25 (the allowance for the
 * factors' own bf16 rounding) it sets the device error word, so the next
 * kla_check_device_error returns KLA_ERR_BOUND.  Nothing traps.  eta
 * outside [0, 2] voids the bound (a ratio above 1 is then not an error of
 * the kernel).
 */
KLA_API kla_status kla_chunk_ut_bound_check(const void *k, const float *g, const float *eta,
                                            float eps, int B, int T, int H, int dk, int dtype,
                                            void *workspace, size_t ws_bytes, float *ratio_max,
                                            void *stream);

/*
 * Token-serial prefill on CUDA cores: the recurrence evaluated one token at
 * a time in fp32 (same arguments and layouts as kla_chunk_fwd, no chunk and
 * no workspace).  Exact-order fp32 evaluation, used for the fp32 I/O mode.
 * Supported: dk, dv in {64, 128}.
 */
KLA_API kla_status kla_recurrent_fwd(const void *q, const void *k, const void *v,
                             const float *g, const float *eta, float eps,
                             const float *h0, void *o, float *hT,
                             int B, int T, int H, int dk, int dv, int dtype,
                             void *stream);

/*
 * One decode step for B sequences (one new token each), updating the state
 * in place -- the recurrence above for a single t.
 *
 *   q, k  [B][H][dk] dtype;  v [B][H][dv] dtype
 *   g, eta [B][H] fp32;  eps fp32
 *   S     [B][H][dk][dv] fp32   state h = S^T, read and overwritten
 *   o     [B][H][dv] dtype      o = S_t q (the updated state)
 * Supported: dk, dv in {64, 128}.  o must not overlap S or the inputs.
 */
KLA_API kla_status kla_decode_step(const void *q, const void *k, const void *v,
                           const float *g, const float *eta, float eps,
                           float *S, void *o, int B, int H, int dk, int dv,
                           int dtype, void *stream);

/*
 * Gated DeltaNet form: the same recurrence with the step size beta_t given
 * per token instead of derived from the key norm ("Deep Dive into KDA",
 * section 2.2; "Kaczmarz Linear Attention", Abstract, describes KLA as this
 * rule with beta_t = eta_t / (||k_t||^2 + eps)).  Arguments, layouts, limits
 * and errors are those of kla_chunk_fwd / kla_decode_step with `beta`
 * ([B][T][H] resp. [B][H] fp32, any real value) in place of eta and no eps;
 * the workspace size is kla_chunk_fwd_workspace_size's.  Runs the same
 * kernels.
 */
KLA_API kla_status kla_gdn_chunk_fwd(const void *q, const void *k, const void *v,
                             const float *g, const float *beta, const float *h0,
                             void *o, float *hT, int B, int T, int H, int dk, int dv,
                             int chunk, int dtype, void *workspace, size_t ws_bytes,
                             void *stream);

KLA_API kla_status kla_gdn_decode_step(const void *q, const void *k, const void *v,
                               const float *g, const float *beta, float *S, void *o,
                               int B, int H, int dk, int dv, int dtype, void *stream);

/*
 * Per-channel gate (KDA form, "Deep Dive into KDA", section 2.3; the
 * "Kaczmarz Linear Attention" Abstract lists its preconditioned variant):
 *
 *   h_t = (I - beta_t k_t k_t^T) Diag(a_t) h_{t-1} + beta_t k_t v_t^T,
 *   a_t = exp(g_t),  o_t = h_t^T q_t   (h = S^T, [dk][dv] per head)
 *
 * with one log-gate per key channel: g is [B][T][H][dk] fp32 for the
 * prefill and [B][H][dk] fp32 for the decode step (any value <= 0 is
 * meaningful; larger values grow the state).  Row i of the state decays by
 * a_{t,i} before the erase reads it.  beta_t = eta_t / (||k_t||^2 + eps) for
 * kla_kda_fwd / kla_kda_decode_step; given per token ([B][T][H] resp.
 * [B][H] fp32) for the _beta variants.  Every other argument, layout, limit
 * and error is that of kla_recurrent_fwd resp. kla_decode_step (dtype bf16
 * or fp32; dk = dv in {64, 128}; o and the written states must not overlap
 * any input, hT may alias h0).  The prefill runs the token-serial CUDA-core
 * kernel (fp32 arithmetic); the decode step the same one-pass state kernel
 * as kla_decode_step.
 */
/*
 * The per-channel-gate prefill as chunks (arguments as kla_kda_fwd plus
 * chunk = KLA_CHUNK and a workspace of kla_kda_chunk_fwd_workspace_size(...)
 * bytes, 16-byte aligned: the per-chunk factors, B * H * ceil(T / 64) *
 * (16 KiB + 24 KiB * dk / 64 + 1 KiB), validated but at present not used).
 * Both I/O types currently run the token-serial per-channel kernel (exact
 * fp32 evaluation): the chunk kernels of this form -- a CUDA-core kernel
 * forming every chunk's factors (A and P summed channel by channel with one
 * e^{G_ri - G_si} <= 1 per term, T = (I + A)^{-1}, W, Q o e^G,
 * K o e^{G_last - G}) and the tcgen05 chain kernel carrying the state --
 * raised intermittent faults whose cause has not been found, and stay
 * unused until it is.  The workspace must not overlap any other argument.
 */
KLA_API size_t kla_kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int dtype);
KLA_API kla_status kla_kda_chunk_fwd(const void *q, const void *k, const void *v,
                                     const float *g, const float *eta, float eps,
                                     const float *h0, void *o, float *hT,
                                     int B, int T, int H, int dk, int dv, int chunk, int dtype,
                                     void *workspace, size_t ws_bytes, void *stream);
KLA_API kla_status kla_kda_chunk_fwd_beta(const void *q, const void *k, const void *v,
                                          const float *g, const float *beta,
                                          const float *h0, void *o, float *hT,
                                          int B, int T, int H, int dk, int dv, int chunk,
                                          int dtype, void *workspace, size_t ws_bytes,
                                          void *stream);
KLA_API kla_status kla_kda_fwd(const void *q, const void *k, const void *v,
                               const float *g, const float *eta, float eps,
                               const float *h0, void *o, float *hT,
                               int B, int T, int H, int dk, int dv, int dtype,
                               void *stream);
KLA_API kla_status kla_kda_fwd_beta(const void *q, const void *k, const void *v,
                                    const float *g, const float *beta,
                                    const float *h0, void *o, float *hT,
                                    int B, int T, int H, int dk, int dv, int dtype,
                                    void *stream);
KLA_API kla_status kla_kda_decode_step(const void *q, const void *k, const void *v,
                                       const float *g, const float *eta, float eps,
                                       float *S, void *o, int B, int H, int dk, int dv,
                                       int dtype, void *stream);
KLA_API kla_status kla_kda_decode_step_beta(const void *q, const void *k, const void *v,
                                            const float *g, const float *beta, float *S,
                                            void *o, int B, int H, int dk, int dv,
                                            int dtype, void *stream);

/*
 * Backward of the prefill (kla_recurrent_fwd / kla_chunk_fwd), for training:
 * given dL/do (grad_o) and dL/dh_T (grad_hT, nullable = 0), the gradients of
 * a loss L with respect to q, k, v, g, eta (the _gdn variant: beta) and h0.
 * The pages print no backward; these are the exact adjoints of the token
 * recurrence above ("Kaczmarz Linear Attention", Abstract, for the step
 * size; "Deep Dive into KDA", section 2.2, for the gated delta rule), taken
 * token by token in reverse order:
 *   dH += q do^T;  dq = h_t do;  du = dH^T k;  dr = -alpha beta du;
 *   dk = dH u + h_{t-1} dr;  dv = beta du;  dbeta = du . (v - alpha r);
 *   dalpha = <dH, h_{t-1}> - beta du . r;  dH <- alpha dH + k dr^T;
 *   dg = alpha dalpha;  deta = dbeta / (||k||^2 + eps) and
 *   dk += -2 dbeta eta k / (||k||^2 + eps)^2 (KLA only).
 * Arithmetic in fp32 on CUDA cores (token-serial; states recomputed from
 * checkpoints every 64 tokens kept in the workspace).
 *
 *   q, k   [B][T][H][dk] dtype;  v, grad_o [B][T][H][dv] dtype
 *   g, eta (beta) [B][T][H] fp32;  h0, grad_hT [B][H][dk][dv] fp32, nullable
 *   grad_q, grad_k [B][T][H][dk] fp32;  grad_v [B][T][H][dv] fp32
 *   grad_g, grad_eta (grad_beta) [B][T][H] fp32;  grad_h0 [B][H][dk][dv]
 *   fp32, nullable (not computed)
 *   workspace: device memory of kla_recurrent_bwd_workspace_size(...) bytes
 *   (16-byte aligned; contents need no initialisation; about
 *   B*H*ceil(T/64)*dk*dv*4 + 2*(dv/32)*B*T*H*(dk+1)*4 bytes), NULL allowed
 *   when T == 0.
 * dk = dv in {64, 128} (else KLA_ERR_UNSUPPORTED); T >= 0 (T == 0: grad_h0 =
 * grad_hT).  Every gradient buffer and the workspace must be disjoint from
 * each other and from every input, else KLA_ERR_INVALID_ARG.  Deterministic:
 * no atomics.  Asynchronous on `stream`, no allocation.
 */
KLA_API size_t kla_recurrent_bwd_workspace_size(int B, int T, int H, int dk, int dv);
KLA_API kla_status kla_recurrent_bwd(const void *q, const void *k, const void *v,
                                     const float *g, const float *eta, float eps,
                                     const float *h0, const void *grad_o,
                                     const float *grad_hT, float *grad_q, float *grad_k,
                                     float *grad_v, float *grad_g, float *grad_eta,
                                     float *grad_h0, int B, int T, int H, int dk, int dv,
                                     int dtype, void *workspace, size_t ws_bytes,
                                     void *stream);
/*
 * Chunkwise backward: the same gradients, arguments, layouts and errors as
 * kla_recurrent_bwd / kla_gdn_recurrent_bwd, computed from the chunk form
 * of the forward (chunk C = 64; "Deep Dive into KDA", section 3).  Per chunk
 * n with start state h_n: dV'_n = P^T dO + Kt dH_{n+1} and
 * dH_n = gamma_C dH_{n+1} + (diag(gamma) Q)^T dO - W^T dV'_n form one
 * reverse chain over the chunks (per head and 64-column slab); every other
 * gradient is per-chunk work on warp-level tensor-core products (tf32
 * operands, fp32 sums): dQ, dK from P, W, U = T diag(beta) V and
 * T = (I + A)^{-1} (dA = -strict_lower(T^T dT T^T)), dg as the reverse
 * in-chunk cumsum of dG.  The states h_n come from the forward chunk
 * prefill (the kernels of kla_chunk_fwd, outputs off, its state chain
 * writing every h_n).  bf16 I/O runs these kernels (relative L2 of the
 * gradients about 1e-3: bf16 state chain, tf32 products); fp32 I/O runs the
 * token-serial kernels of kla_recurrent_bwd (fp32 accuracy).
 * Workspace: kla_chunk_bwd_workspace_size(...) bytes (for the chunk kernels
 * about B*H*ceil(T/64) * 224 KiB).
 */
KLA_API size_t kla_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int dtype);
KLA_API kla_status kla_chunk_bwd(const void *q, const void *k, const void *v,
                                 const float *g, const float *eta, float eps,
                                 const float *h0, const void *grad_o, const float *grad_hT,
                                 float *grad_q, float *grad_k, float *grad_v, float *grad_g,
                                 float *grad_eta, float *grad_h0, int B, int T, int H,
                                 int dk, int dv, int dtype, void *workspace, size_t ws_bytes,
                                 void *stream);
KLA_API kla_status kla_gdn_chunk_bwd(const void *q, const void *k, const void *v,
                                     const float *g, const float *beta, const float *h0,
                                     const void *grad_o, const float *grad_hT, float *grad_q,
                                     float *grad_k, float *grad_v, float *grad_g,
                                     float *grad_beta, float *grad_h0, int B, int T, int H,
                                     int dk, int dv, int dtype, void *workspace,
                                     size_t ws_bytes, void *stream);

/*
 * The same backward for the per-channel-gate form (kla_kda_fwd; "Deep Dive
 * into KDA", section 2.3): g and grad_g are [B][T][H][dk] (one log-gate per
 * key channel), the forward being hd = Diag(e^{g_t}) h_{t-1}; r = hd^T k;
 * u = beta (v - r); h_t = hd + k u^T.  Reverse per token: dH += q do^T;
 * dq = h_t do; du = dH^T k; dr = -beta du; dv = beta du;
 * dbeta = du . (v - r); dk = dH u + hd dr; Hd = dH + k dr^T;
 * dg_i = sum_j Hd_ij hd_ij; dH <- Diag(e^{g_t}) Hd; then the step size's
 * chain rule as above (the _beta form returns dbeta).  Workspace:
 * kla_kda_recurrent_bwd_workspace_size(...) bytes (about (dv/32)*dk*4 more
 * per head-token than the scalar gate's).  Everything else as
 * kla_recurrent_bwd.
 */
KLA_API size_t kla_kda_recurrent_bwd_workspace_size(int B, int T, int H, int dk, int dv);
KLA_API kla_status kla_kda_recurrent_bwd(const void *q, const void *k, const void *v,
                                         const float *g, const float *eta, float eps,
                                         const float *h0, const void *grad_o,
                                         const float *grad_hT, float *grad_q, float *grad_k,
                                         float *grad_v, float *grad_g, float *grad_eta,
                                         float *grad_h0, int B, int T, int H, int dk, int dv,
                                         int dtype, void *workspace, size_t ws_bytes,
                                         void *stream);
KLA_API kla_status kla_kda_recurrent_bwd_beta(const void *q, const void *k, const void *v,
                                              const float *g, const float *beta,
                                              const float *h0, const void *grad_o,
                                              const float *grad_hT, float *grad_q,
                                              float *grad_k, float *grad_v, float *grad_g,
                                              float *grad_beta, float *grad_h0, int B, int T,
                                              int H, int dk, int dv, int dtype,
                                              void *workspace, size_t ws_bytes, void *stream);
KLA_API kla_status kla_gdn_recurrent_bwd(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta,
                                         const float *h0, const void *grad_o,
                                         const float *grad_hT, float *grad_q, float *grad_k,
                                         float *grad_v, float *grad_g, float *grad_beta,
                                         float *grad_h0, int B, int T, int H, int dk, int dv,
                                         int dtype, void *workspace, size_t ws_bytes,
                                         void *stream);

/*
 * Prefill from HOST buffers, end to end: the same computation as
 * kla_chunk_fwd with q, k, v, g, eta, h0 (nullable), o and hT (nullable) in
 * host memory (same layouts; page-locked memory is needed for the copies to
 * run asynchronously and overlap).  T >= 1.
 *
 * The batch is cut into pieces of whole sequences; each piece is copied to a
 * staging slot in `staging` (caller-owned device memory of
 * kla_chunk_fwd_host_staging_size(...) bytes, 256-byte aligned, else
 * KLA_ERR_INVALID_ARG), its prefill runs on `stream`, and its outputs are
 * copied back, with the copy-in of the next piece and the copy-out of the
 * previous one overlapping the kernels (two copy streams per device, created
 * on first use and kept).  The call only enqueues work: the host buffers
 * must stay valid, and o / hT may be read only once `stream` has passed the
 * call (e.g. after cudaStreamSynchronize).  Calls that share a staging
 * buffer are ordered by `stream`.  Limits and errors otherwise as
 * kla_chunk_fwd.
 */
KLA_API size_t kla_chunk_fwd_host_staging_size(int B, int T, int H, int dk, int dv, int dtype);
KLA_API kla_status kla_chunk_fwd_host(const void *q, const void *k, const void *v,
                                      const float *g, const float *eta, float eps,
                                      const float *h0, void *o, float *hT,
                                      int B, int T, int H, int dk, int dv, int dtype,
                                      void *staging, size_t staging_bytes, void *stream);

/*
 * Chunkwise prefill without any caller-provided device memory.
 *
 * No counterpart in the paper: this is a deployment convenience.  Some
 * callers cannot hand the library scratch memory -- their device memory
 * belongs to another allocator (e.g. a serving process's pre-reserved pool)
 * or they may not allocate after start-up -- so this call runs
 * kla_chunk_fwd (same arguments and layouts, chunk = KLA_CHUNK, dtype
 * KLA_BF16 or KLA_FP32) with a fixed scratch array compiled into libkla.so
 * instead of a workspace.  It allocates nothing itself.
 *
 *   Limit (KLA_BF16 only; the KLA_FP32 path uses no scratch):
 *          B * H * ceil(T / KLA_CHUNK) <= KLA_NOALLOC_MAX_CHUNKS, else
 *          KLA_ERR_UNSUPPORTED (checked before any CUDA call, in 64-bit
 *          arithmetic).  The state chain is cut into segments only where
 *          their states also fit.
 *   Memory: every GPU that loads libkla.so holds KLA_NOALLOC_SCRATCH_BYTES
 *          for the life of the process.
 *   First call on a device looks up the array's device address
 *          (cudaGetSymbolAddress); make that first call before any stream
 *          capture.
 *   All calls share the one array, which keeps the previous call's contents
 *          (nothing in it needs to start at zero).  Calls whose work overlaps
 *          on the GPU (several streams or host threads at once) race on it:
 *          issue them one after another.
 */
#define KLA_NOALLOC_MAX_CHUNKS 1024
#define KLA_NOALLOC_SCRATCH_BYTES (KLA_NOALLOC_MAX_CHUNKS * 16384)
KLA_API kla_status kla_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                 const float *g, const float *eta, float eps,
                                 const float *h0, void *o, float *hT,
                                 int B, int T, int H, int dk, int dv, int dtype,
                                 void *stream);

/*
 * Reads and clears the library's device error word for the current device
 * after synchronising `stream`.  Kernels set it instead of hanging when a
 * bounded wait on an mbarrier runs out (KLA_ERR_TIMEOUT), and the debug
 * bound check sets it on a violation (KLA_ERR_BOUND; a timeout takes
 * precedence when both happened).  Returns KLA_OK when no kernel reported a
 * problem.
 */
KLA_API kla_status kla_check_device_error(void *stream);

/*
 * Self-test of that path, for failure-detection tests: launches one thread
 * that waits, with the same bounded mbarrier wait the tensor-core kernels
 * use, on a phase nothing ever completes, gives up after `limit_ms`
 * milliseconds (1 .. 10000, else KLA_ERR_INVALID_ARG), sets the device
 * error word and returns.  The next kla_check_device_error on that stream
 * reports KLA_ERR_TIMEOUT; the context stays usable.  No fault, trap or
 * hang is involved.
 */
KLA_API kla_status kla_selftest_wait_timeout(unsigned int limit_ms, void *stream);

/* Static description of a status code (never NULL). */
KLA_API const char *kla_status_string(int status);

/* ABI version: major * 10000 + minor * 100 + patch. */
KLA_API int kla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KLA_H_ */
