/*
 * prism.h - C ABI of the PRISM sequence-mixer scan for NVIDIA B200 (sm_100a).
 *
 * The operation (forward only), per batch row b and head h, with the state
 * S in R^{d_v x d_k} (S0, or zeros), m = L - 1 residual steps and a ShortConv of
 * width W:
 *
 *   a_t     = sum_{i<W} conv_w[h,:,i] * v_{t-i}      depthwise causal ShortConv anchor
 *   r_{t,0} = v_t - a_t                               anchor residual
 *   r_{t,l} = (1 - gain_{t,l}) * r_{t,l-1}            linearised residual chain, l = 1..m
 *   S_t     = gamma_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *             + sum_l alpha_{t,l} r_{t,l} u_{t,l}^T    gated-delta write + rank-m residual write
 *   o_t     = S_t q_t                                 post-update readout
 *
 * Sources (web pages on PRISM, Parallel Residual Iterative Sequence Model):
 *   - "ICML 2026 | 当线性注意力学会"写入前思考"：并行化的多步记忆写入" (Tencent Ads
 *     write-up): section 核心迭代形式 (the step-size x residual x direction write),
 *     消除 Token 间串行 (forget path kept as GDN, ShortConv anchor replaces the
 *     global state), 消除 Step 间串行 (closed-form element-wise residual chain),
 *     架构形式 (write = GDN write + low-rank residual; L = 1 is exactly GDN),
 *     混合架构是必然 (the anchor window covers the last 3-4 tokens).
 *   - "PRISM: Parallel Residual Iterative Sequence Model" technical summary,
 *     sections 2.1 (S_t = S_{t-1} A_t + B_t, A_t the rank-1 gated-delta
 *     transition) and 2.2 (two-stage proxy: anchor from a short convolution,
 *     then L parallel refinement steps with gain, residual and direction).
 *   - ICML 2026 poster abstract of the same paper (short-convolution anchor,
 *     rank-L accumulation).
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers (except in prism_scan_fwd_host),
 *     owned by the caller.  The library never allocates or frees device memory
 *     and never synchronises, except prism_stream_status.  Work is enqueued on
 *     `stream` (0 = legacy default stream).
 *   - Layouts are dense, row-major, token-major:
 *       q, k    [B, T, H, d_k]          dtype
 *       v       [B, T, H, d_v]          dtype
 *       gamma   [B, T, H]               fp32, decay gate in (0, 1]
 *       beta    [B, T, H]               fp32, delta-rule step size
 *       u       [B, T, H, L-1, d_k]     dtype, residual-write directions (NULL iff L == 1)
 *       alpha   [B, T, H, L-1]          fp32, residual step sizes        (NULL iff L == 1)
 *       gain    [B, T, H, L-1, d_v]     dtype, per-channel gains g       (NULL iff L == 1)
 *       conv_w  [H, d_v, W]             fp32, ShortConv taps, tap i multiplies v_{t-i}
 *       S0      [B, H, d_v, d_k]        fp32 or NULL (zeros)
 *       lengths [B]                     int32 or NULL (every row has T valid steps);
 *                                       right padding: steps t >= lengths[b] leave S
 *                                       unchanged and write o_t = 0
 *       o       [B, T, H, d_v]          dtype (output)
 *       S_final [B, H, d_v, d_k]        fp32 (output) or NULL: state after the last
 *                                       valid step of each row
 *     dtype is PRISM_BF16 (bfloat16) or PRISM_FP32.  Arithmetic is fp32 with an
 *     fp32 state; bf16 outputs are rounded to nearest even.
 *   - Every device pointer must be 16-byte aligned.
 *   - Return value: PRISM_OK or a PRISM_ERR_* code.  All argument checks run
 *     before anything is enqueued; on an error nothing is launched and the
 *     outputs are untouched.  Launch failures return PRISM_ERR_CUDA.  Device-side
 *     errors (a bounded wait that expired) are recorded in a per-device status
 *     word that prism_stream_status reports.
 */
#ifndef PRISM_H_
#define PRISM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* prism_stream_t; /* same type as cudaStream_t */

#define PRISM_VERSION_MAJOR 0
#define PRISM_VERSION_MINOR 1
#define PRISM_VERSION_PATCH 0

enum prism_dtype {
  PRISM_BF16 = 0,
  PRISM_FP32 = 1
};

/* Residual chain step.  Exact: gist.science PRISM explainer, 2.2 Input-Anchored Loop
 * Unrolling (Residual Update).  Linearised: ICML 2026 PRISM write-up, 消除 Step 间串行. */
enum prism_chain {
  PRISM_CHAIN_LINEAR = 0, /* r_l = (1 - g_l) * r_{l-1}: the linearised chain (default) */
  PRISM_CHAIN_GELU = 1    /* r_l = r_{l-1} - GELU(g_l * r_{l-1}), GELU(x) = x Phi(x) (erf form) */
};

enum prism_status {
  PRISM_OK = 0,
  PRISM_ERR_INVALID_ARG = 1, /* NULL where required, non-positive size, L < 1, W < 1, ... */
  PRISM_ERR_UNSUPPORTED = 2, /* valid but not implemented: head size, width, alignment, device */
  PRISM_ERR_WORKSPACE = 3,   /* workspace smaller than prism_scan_fwd_workspace_size() */
  PRISM_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  PRISM_ERR_TIMEOUT = 5,     /* a bounded device-side wait expired (from prism_stream_status) */
  PRISM_ERR_BOUNDS = 6       /* debug build only: a kernel computed an index outside its buffer
                                and skipped the access (from prism_stream_status) */
};

/* Limits of this build (checked; larger values return PRISM_ERR_UNSUPPORTED). */
#define PRISM_MAX_HEAD_DIM 128 /* d_k, d_v in {16, 32, 64, 128} */
#define PRISM_MAX_L 16         /* 1 <= L <= 16 */
#define PRISM_MAX_W 8          /* 1 <= W <= 8 */

/*
 * prism_scan_fwd - the whole mixer forward: ShortConv anchor, residual chain,
 * rank-(L-1) residual write and gated-delta write inside one scan, readout.
 * Defined by the sources above (write-up 核心迭代形式 / 架构形式, summary 2.1-2.2).
 *
 * chunk: chunk length of the chunkwise-parallel evaluation, a power of two in
 *   [16, 64].  The result does not depend on it beyond rounding.  The bf16
 *   tensor-core path runs chunk == 64 with d_k == d_v in {64, 128}.  fp32 with
 *   d_k == d_v in {16, 32, 64} runs the same chunk decomposition in fp32 FMAs on
 *   CUDA cores (one launch, chunk length `chunk`).  Every other supported shape runs
 *   the fp32 CUDA-core path that evaluates the recurrence token by token.
 * workspace / workspace_bytes: device scratch of at least
 *   prism_scan_fwd_workspace_size(...) bytes (may be NULL when that is 0), 16-byte
 *   aligned, owned by the caller, contents undefined on return.  The tensor-core
 *   path writes there, in one launch over all chunks before the scan, the residual
 *   write vectors alpha_{t,l} r_{t,l} of every token, scaled for the chunk form, as
 *   bf16 in the layout of gain (B * T * H * (L - 1) * d_v * 2 bytes, rounded up to
 *   256); a sequence cut into segments (long sequences over few (batch row, head)
 *   chains) adds three fp32 d_v x d_k states per segment, and a scan run in two halves
 *   (chains that leave SMs idle) adds two fp32 d_v x d_k states per chain.  The CUDA-core paths
 *   need none.  Too small or NULL: PRISM_ERR_WORKSPACE, before any launch.
 * Errors: PRISM_ERR_INVALID_ARG, PRISM_ERR_UNSUPPORTED, PRISM_ERR_WORKSPACE,
 *   PRISM_ERR_CUDA, as described above.
 */
int prism_scan_fwd(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const void* u, const float* alpha, const void* gain,
                   const float* conv_w, const float* S0, const int32_t* lengths,
                   int B, int T, int H, int d_k, int d_v, int L, int W, int chunk,
                   int dtype, void* o, float* S_final,
                   void* workspace, size_t workspace_bytes, prism_stream_t stream);

/*
 * prism_scan_fwd_ex - prism_scan_fwd with the residual chain selected by `chain`
 * (PRISM_CHAIN_LINEAR or PRISM_CHAIN_GELU; any other value is PRISM_ERR_INVALID_ARG),
 * and the ShortConv history of the sequences in `conv_state`.
 * For PRISM_CHAIN_GELU the `gain` tensor holds the predictor output p of the exact
 * refinement step r <- r - GELU(p * r) (gist.science PRISM explainer, 2.2), any real value.
 * conv_state [B,H,W-1,d_v] dtype (device, 16-byte aligned; NULL: zeros): v_{-W+1}, ...,
 *   v_{-1}, oldest first, the values of v before token 0 that the ShortConv anchors of
 *   the first W - 1 tokens read (ICML 2026 PRISM write-up, 消除 Token 间串行: the anchor
 *   reads the last few tokens).  A sequence scanned in two calls, the second with
 *   S0 = the first's S_final and conv_state = the first's last W - 1 rows of v, gives
 *   the result of one call over the whole sequence (the layout of prism_decode_step's
 *   conv_state).  Ignored when W == 1.
 * prism_scan_fwd is prism_scan_fwd_ex with PRISM_CHAIN_LINEAR and no history.
 */
int prism_scan_fwd_ex(const void* q, const void* k, const void* v,
                      const float* gamma, const float* beta,
                      const void* u, const float* alpha, const void* gain,
                      const float* conv_w, const float* S0, const int32_t* lengths,
                      int B, int T, int H, int d_k, int d_v, int L, int W, int chunk,
                      int dtype, void* o, float* S_final,
                      void* workspace, size_t workspace_bytes, prism_stream_t stream, int chain,
                      const void* conv_state);

/* Bytes of device workspace prism_scan_fwd needs for these sizes (0 if none).
 * Returns 0 for invalid sizes as well; prism_scan_fwd reports those. */
size_t prism_scan_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int L,
                                     int W, int chunk, int dtype);

/*
 * prism_scan_bwd - gradients of the scan (the training pass): for the cotangents dO of o
 * and (optionally) dS_final of S_final, the gradients of L = <o, dO> + <S_final, dS_final>
 * with respect to every input of prism_scan_fwd_ex with the same arguments.  Reverse-mode
 * differentiation of the recurrence defined above (ICML 2026 PRISM write-up, 核心迭代形式 /
 * 架构形式; PRISM explainer 2.1-2.2).
 *
 * Inputs: as prism_scan_fwd_ex (q, k, v, gamma, beta, u, alpha, gain, conv_w, S0, lengths,
 *   chain), plus dO [B,T,H,d_v] (dtype) and dS_final [B,H,d_v,d_k] fp32 or NULL (zero).
 * Outputs (fp32, device, caller-owned, same shapes as the inputs): dq, dk [B,T,H,d_k];
 *   dv [B,T,H,d_v]; dgamma, dbeta [B,T,H]; du [B,T,H,L-1,d_k], dalpha [B,T,H,L-1],
 *   dgain [B,T,H,L-1,d_v] (all three NULL iff L == 1); dconv_w [H,d_v,W]; dS0 [B,H,d_v,d_k]
 *   (the gradient with respect to the initial state, zeros or S0).  Padded steps get zero
 *   gradients.
 * Two algorithms, chosen by shape; both compute in fp32 and are deterministic:
 *   chunked (d_k = d_v in {64, 128}, L <= 4): a token-by-token forward records S at every
 *     64-token chunk boundary and v_t - gamma_t S_{t-1} k_t; a reverse token-by-token
 *     launch runs the adjoint recurrence G_t = dO_t q_t^T + gamma_{t+1} G_{t+1}
 *     (I - beta_{t+1} k_{t+1} k_{t+1}^T) and records G_t k_t, G_t u_{t,l}, the gradient
 *     entering every chunk end and its inner product with the state there; one launch
 *     per chunk then forms every gradient of the chunk's tokens from those records; a
 *     last launch adds the per-chunk dconv_w partials in a fixed order.  Workspace
 *     (fp32): B*H*(2*NC+1)*d*d for the boundary states and gradients (NC = ceil(T/64)),
 *     B*T*H*(L+1)*d for the per-token records, plus small per-chunk partials.
 *   token-by-token (every other shape): a forward records every state S_t
 *     (B*H*T*d_v*d_k fp32), a reverse launch walks the tokens, two launches reduce the
 *     per-row-block partial sums (of 32 rows; 64 for d_k = 16) of the gradients that
 *     are sums over rows (dq, dk, du, dgamma, dbeta, dalpha) and dconv_w.
 * workspace: prism_scan_bwd_workspace_size() bytes (the chunked form: 0.54 GB for the
 *   130M-LM layer, B=16 T=2048 H=6 d=128 L=4, against 12.9 GB token by token).
 * Sizes as prism_scan_fwd.  Four launches on `stream` after memsets of the outputs; no
 * synchronisation.
 */
size_t prism_scan_bwd_workspace_size(int B, int T, int H, int d_k, int d_v, int L, int W, int dtype);

int prism_scan_bwd(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const void* u, const float* alpha, const void* gain,
                   const float* conv_w, const float* S0, const int32_t* lengths,
                   const void* dO, const float* dS_final,
                   int B, int T, int H, int d_k, int d_v, int L, int W, int dtype, int chain,
                   float* dq, float* dk, float* dv, float* dgamma, float* dbeta,
                   float* du, float* dalpha, float* dgain, float* dconv_w, float* dS0,
                   void* workspace, size_t workspace_bytes, prism_stream_t stream);

/*
 * prism_state_affine - out = S M + N for every (batch, head): the composition step of
 * per-segment state maps.  The state update is affine in the state (see the recurrence
 * above), so a run over a segment of tokens maps a start state S to S M + N, with
 * M [d_k, d_k] the ordered product of the transitions gamma_t (I - beta_t k_t k_t^T) and
 * N [d_v, d_k] the segment's end state from a zero start.  Sequence sharding folds the
 * maps of earlier segments into a segment's start state with this call.
 *
 * S, N, out: [BH, d_v, d_k] fp32; M: [BH, d_k, d_k] fp32; device, caller-owned.  N may
 * be NULL (zero).  out may be exactly S or exactly N; any other overlap of out with S, M
 * or N returns PRISM_ERR_INVALID_ARG before any launch.  d_k, d_v in
 * {16, 32, 64, 128}; 1 <= BH <= 65535.  fp32, fixed summation order (deterministic).
 * One launch on `stream`, no synchronisation.
 */
int prism_state_affine(const float* S, const float* M, const float* N, float* out, int BH, int d_v, int d_k,
                       prism_stream_t stream);

/* Size of the device-global scratch behind prism_scan_fwd_static. */
#define PRISM_STATIC_WORKSPACE_BYTES (192u << 20)

/*
 * prism_scan_fwd_static - prism_scan_fwd_ex without a caller-supplied workspace and
 * without any allocation (an entry point of this library; the PRISM write-ups describe
 * no counterpart): the scratch is a file-scope device array of
 * PRISM_STATIC_WORKSPACE_BYTES (192 MiB, 256-byte aligned) inside the library, one per
 * device.  The first call on a device looks its address up with cudaGetSymbolAddress
 * (make that first call before any stream capture); later calls reuse it.  The array
 * sits in a module of its own: with lazy module loading (the default of CUDA 12, and
 * what PyTorch sets) it is held, until the process exits, on each device where this
 * entry point has run; with CUDA_MODULE_LOADING=EAGER, on every device where the
 * library is loaded.  Results are bit-for-bit those of prism_scan_fwd_ex with a
 * workspace.  Sizes whose
 * prism_scan_fwd_workspace_size() exceeds PRISM_STATIC_WORKSPACE_BYTES return
 * PRISM_ERR_WORKSPACE before any launch (the 130M-LM layer, B=16 T=2048 H=6 d=128
 * L=4, needs 144 MiB; a 65536-token sequence over 8 heads with L=8 needs more and is
 * refused).  Because the scratch is shared, calls on one device must not overlap
 * in time: issue them on one stream or order them; calls on one stream may follow each
 * other freely.  Other arguments, conventions and errors as for prism_scan_fwd_ex.
 */
int prism_scan_fwd_static(const void* q, const void* k, const void* v,
                          const float* gamma, const float* beta,
                          const void* u, const float* alpha, const void* gain,
                          const float* conv_w, const float* S0, const int32_t* lengths,
                          int B, int T, int H, int d_k, int d_v, int L, int W, int chunk,
                          int dtype, void* o, float* S_final, prism_stream_t stream, int chain,
                          const void* conv_state);

/*
 * prism_scan_fwd_host - the same operation on HOST buffers: copies every input
 * from host memory into the caller's device buffers, runs prism_scan_fwd on
 * them, and copies o (and S_final if both pointers are given) back to host
 * memory, all enqueued on `stream` with cudaMemcpyAsync (pinned host memory
 * makes the copies asynchronous).  host_* are host pointers with the layouts
 * above, dev_* the device buffers of the same sizes; dk, dv are d_k, d_v.  The
 * call returns once the work is enqueued; synchronise `stream` before reading
 * host_o / host_S_final.
 */
int prism_scan_fwd_host(const void* host_q, const void* host_k, const void* host_v,
                        const float* host_gamma, const float* host_beta,
                        const void* host_u, const float* host_alpha, const void* host_gain,
                        const float* host_conv_w, const float* host_S0, const int32_t* host_lengths,
                        void* dev_q, void* dev_k, void* dev_v, float* dev_gamma, float* dev_beta,
                        void* dev_u, float* dev_alpha, void* dev_gain, float* dev_conv_w,
                        float* dev_S0, int32_t* dev_lengths,
                        int B, int T, int H, int dk, int dv, int L, int W, int chunk,
                        int dtype, void* dev_o, float* dev_S_final, void* host_o, float* host_S_final,
                        void* workspace, size_t workspace_bytes, prism_stream_t stream);

/*
 * prism_prologue_fwd - steps before the scan, on their own: the ShortConv
 * anchor, the anchor residual and the closed-form residual chain, giving the
 * residual-write vectors rho_{t,l} = alpha_{t,l} r_{t,l} (write-up 消除 Step
 * 间串行: the chain is element-wise and linear, so it has a closed form).
 * Inputs as for prism_scan_fwd (L >= 2); lengths may be NULL.
 * rho_out: [B, T, H, L-1, d_v] fp32 device buffer; rows t >= lengths[b] are
 * written as 0.  Errors as for prism_scan_fwd.
 */
int prism_prologue_fwd(const void* v, const float* alpha, const void* gain,
                       const float* conv_w, const int32_t* lengths,
                       int B, int T, int H, int d_v, int L, int W, int dtype,
                       float* rho_out, prism_stream_t stream);

/* 1 if prism_scan_fwd runs these sizes on the tcgen05 tensor-core chunk
 * kernel, 0 if on a CUDA-core kernel (the fp32 chunk form or token by token;
 * sizes as for prism_scan_fwd; unsupported sizes also give 0). */
int prism_scan_fwd_uses_tensor_cores(int d_k, int d_v, int L, int W, int chunk, int dtype);

/* Number of kernel launches one prism_scan_fwd call with these sizes issues (0 for
 * invalid sizes).  Tensor-core path: the residual-write launch when L > 1, then one
 * scan launch, or four (three scans and a fold) when a long sequence over few
 * (batch row, head) chains is cut into segments; when the chains leave at least 24 of
 * a B200's SMs idle, L > 1 and the sequence has at least 8 chunks, four: the scan runs
 * in two halves, and the second half's residual write runs beside the first half's
 * scan (on an internal stream of the device, forked from and joined back into the
 * call's stream).  CUDA-core paths: 1. */
int prism_scan_fwd_launches(int B, int T, int H, int d_k, int d_v, int L, int W, int chunk, int dtype);

/* Chunks (of 64 tokens) in the first of the two scan launches when prism_scan_fwd runs
 * these sizes in two halves (see prism_scan_fwd_launches); 0 when it does not, or for
 * invalid sizes.  The cut is placed so that the second half's residual write, on the SMs
 * the chains leave idle, ends about when the first scan does: with x = 0.28 chains /
 * idle SMs, ceil(NC x / (1 + x)) chunks, clamped to [ceil(NC / 4), NC - 1] (11 of 32 for
 * the 130M-LM layer, B=16 T=2048 H=6).  A measurement aid; results do not depend on it
 * beyond rounding. */
int prism_scan_fwd_split_chunks(int B, int T, int H, int d_k, int d_v, int L, int W, int chunk, int dtype);

/* prism_prologue_fwd with the residual chain selected by `chain` (see prism_scan_fwd_ex). */
int prism_prologue_fwd_ex(const void* v, const float* alpha, const void* gain,
                          const float* conv_w, const int32_t* lengths,
                          int B, int T, int H, int d_v, int L, int W, int dtype,
                          float* rho_out, prism_stream_t stream, int chain);

/*
 * prism_decode_step - one recurrent step of the scan for every (b, h): the O(1)-state
 * inference form of the recurrence above (ICML 2026 PRISM write-up, 背景 and
 * Rank-1 写入瓶颈: a linear-attention layer keeps a fixed-size state and updates it
 * once per token).  For one token t and each (b, h):
 *   a = w[h,:,0] v_t + sum_{i=1}^{W-1} w[h,:,i] v_{t-i}   (v_{t-i} taken from conv_state)
 *   r_0 = v_t - a;  r_l = chain step of r_{l-1} with gain g_l (see prism_scan_fwd_ex)
 *   S <- gamma S (I - beta k k^T) + beta v_t k^T + sum_l alpha_l r_l u_l^T;   o = S q
 * Decoding tokens one at a time from S0 and a zero history gives what prism_scan_fwd
 * gives for the whole sequence; decoding after prism_scan_fwd continues that sequence
 * when S = its S_final and conv_state = its last W-1 values of v.
 *
 * Inputs (device pointers, contiguous, 16-byte aligned):
 *   q, k        [B,H,d_k]      dtype
 *   v           [B,H,d_v]      dtype
 *   gamma, beta [B,H]          fp32
 *   u           [B,H,L-1,d_k]  dtype   (NULL iff L == 1)
 *   alpha       [B,H,L-1]      fp32    (NULL iff L == 1)
 *   gain        [B,H,L-1,d_v]  dtype   (NULL iff L == 1)
 *   conv_w      [H,d_v,W]      fp32
 * In/out, updated in place:
 *   conv_state  [B,H,W-1,d_v]  dtype   v_{t-W+1}, ..., v_{t-1}, oldest first (zeros at the
 *                                      start of a sequence); becomes v_{t-W+2}, ..., v_t.
 *                                      NULL iff W == 1.
 *   S           [B,H,d_v,d_k]  fp32    the state before the token; becomes the state after it.
 * Output:
 *   o           [B,H,d_v]      dtype
 * d_k, d_v in {16, 32, 64, 128} (independently); 1 <= L <= PRISM_MAX_L; 1 <= W <= PRISM_MAX_W;
 * chain is PRISM_CHAIN_LINEAR or PRISM_CHAIN_GELU.  Enqueued on `stream`; allocates nothing;
 * no synchronisation.  Errors as for prism_scan_fwd, returned before any launch.
 */
int prism_decode_step(const void* q, const void* k, const void* v,
                      const float* gamma, const float* beta,
                      const void* u, const float* alpha, const void* gain,
                      const float* conv_w, void* conv_state, float* S,
                      int B, int H, int d_k, int d_v, int L, int W, int dtype, int chain,
                      void* o, prism_stream_t stream);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device: PRISM_OK, PRISM_ERR_TIMEOUT, PRISM_ERR_BOUNDS (debug build only), or
 * PRISM_ERR_CUDA if the synchronisation itself failed. */
int prism_stream_status(prism_stream_t stream);

/* Test hook: the spin limit of the device-side bounded waits (0 restores the
 * default).  A tiny limit makes those waits give up and record
 * PRISM_ERR_TIMEOUT instead of waiting, which tests the error path without
 * hanging a GPU.  Host-side setting; applies to launches made after the call. */
void prism_set_spin_limit(long long limit);

/* Measurement hook: `event` (a cudaEvent_t, or NULL to clear) is recorded on the
 * stream of the next prism_scan_fwd call that runs the tensor-core path with L > 1,
 * after its (first) residual-write launch, and is then forgotten.  Events recorded by
 * the caller before and after that call then time that launch and the rest apart.  Process-wide; set it from the thread that makes the call. */
void prism_set_split_event(void* event);

/* Static description of a status code; never NULL. */
const char* prism_status_string(int code);

/* (major << 16) | (minor << 8) | patch */
int prism_version(void);

/* 1 in the debug build of this library (libprism_debug.so, compiled with
 * PRISM_DEBUG_BOUNDS), 0 in the release build (libprism.so).  Both export the same
 * functions and compute the same results bit for bit.  In the debug build the kernels
 * check the global indices they compute against the extents of their buffers (and the
 * innermost coordinate of every TMA copy against the 16-byte rule); a failed check
 * records PRISM_ERR_BOUNDS in the device status word and skips the access. */
int prism_debug_bounds(void);

/* Test hook of the debug build: one launch on `stream` that runs the device-side check
 * of index i against extent n (no memory is accessed at that index), so that
 * prism_stream_status then reports PRISM_ERR_BOUNDS exactly when i is outside [0, n).
 * PRISM_ERR_UNSUPPORTED in the release build; PRISM_ERR_CUDA if the launch fails. */
int prism_debug_bounds_probe(long long i, long long n, prism_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PRISM_H_ */
