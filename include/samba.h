/*
 * samba.h -- C ABI of the B200 (sm_100a) kernels for Samba's two token mixers.
 *
 * Samba ("Samba: Simple Hybrid State Space Models for Efficient Unlimited
 * Context Language Modeling", Ren et al.) interleaves a Mamba layer (a
 * selective state-space scan) with a sliding-window attention (SWA) layer.
 * This library runs the prefill forward of both mixers and their single-token
 * decode steps:
 *
 *   - causal depthwise conv1d (width K, K = 4) in front of the scan;
 *   - selective scan h_t = exp(Δ_t A) h_{t-1} + Δ_t B_t u_t,
 *     y_t = (C_t . h_t + D u_t) * silu(z_t), with Δ_t = softplus(delta_t)
 *     (page "SAMBA混合注意力状态空间模型", section 数学框架 / Mamba层: the
 *     recurrence h_t = Ā_t h_{t-1} + B̄_t x_t, y_t = C_t h_t and its
 *     input-dependent B_t, C_t, Δ_t);
 *   - causal sliding-window attention with grouped KV heads, where query i
 *     sees key j exactly when 0 <= i - j < W (same page, section
 *     滑动窗口注意力; its mask is printed inverted, this is the causal band);
 *   - the decode steps mamba_step / swa_step of the page's section 推理效率.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer is a DEVICE pointer owned by the caller.  The library never
 *    allocates or frees device memory and never synchronises, except in
 *    samba_get_status().
 *  - Every call is asynchronous on the given stream (a cudaStream_t; NULL is
 *    the legacy default stream) and returns an int status.  Arguments are
 *    checked on the host before any launch; a rejected call launches nothing.
 *  - Tensors are dense and row-major in the layouts written beside each
 *    argument (channel-last activations).  Base pointers must be 16-byte
 *    aligned.
 *  - bf16 is IEEE bfloat16 (round-to-nearest-even on store).  All arithmetic
 *    of the scan is fp32; attention multiplies in bf16 on the tensor cores
 *    with fp32 accumulation and an fp32 softmax.
 *  - Errors: SAMBA_ERR_INVALID_ARG (null pointer where one is required, bad
 *    shape, misaligned pointer), SAMBA_ERR_UNSUPPORTED (dtype, state size,
 *    head_dim or head grouping outside what the kernels implement),
 *    SAMBA_ERR_WORKSPACE (workspace too small), SAMBA_ERR_CUDA (a CUDA call
 *    or launch failed).  samba_last_error() gives a one-line description of
 *    the last failure on the calling host thread.
 *  - Kernels never spin without a limit.  A device-side wait that runs out
 *    (which only a library bug can cause) stops the kernel cleanly and
 *    records SAMBA_ERR_TIMEOUT in a per-device status word that
 *    samba_get_status() returns.
 */
#ifndef SAMBA_H_
#define SAMBA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA. */
typedef struct CUstream_st* samba_stream_t;

/* element types */
enum { SAMBA_F32 = 0, SAMBA_BF16 = 1 };

/* status codes */
enum {
  SAMBA_OK = 0,
  SAMBA_ERR_INVALID_ARG = -1,
  SAMBA_ERR_UNSUPPORTED = -2,
  SAMBA_ERR_WORKSPACE = -3,
  SAMBA_ERR_CUDA = -4,
  SAMBA_ERR_TIMEOUT = -5,
  SAMBA_ERR_CHECK = -6          /* debug build only: a device-side index check failed */
};

/* flags of samba_scan_args.flags */
enum {
  SAMBA_SCAN_FUSE_CONV = 1,      /* x is the conv input; u = conv1d(x) (+ SiLU) */
  SAMBA_SCAN_DELTA_SOFTPLUS = 2, /* Δ = softplus(delta); otherwise Δ = delta    */
  SAMBA_SCAN_CONV_SILU = 4       /* apply SiLU to the conv output               */
};

/* Library version, major*10000 + minor*100 + patch. */
int samba_version(void);

/* One-line text of the last error reported on this host thread ("" if none). */
const char* samba_last_error(void);

/* Synchronises `stream`, then returns and clears this device's status word:
 * SAMBA_OK, or SAMBA_ERR_TIMEOUT if a kernel gave up a device-side wait since
 * the last call, or (debug build) SAMBA_ERR_CHECK if a device-side index
 * check failed.  Returns SAMBA_ERR_CUDA if the synchronisation itself fails.
 *
 * Debug build: libsamba_debug.so (hybrid_ssm_sliding_b200/build.py --debug)
 * is the same library compiled with SAMBA_DEBUG.  Its kernels check the
 * index of every global output store against the extent of the tensor it
 * writes (computed from the call's sizes); a failed check skips the store and
 * records SAMBA_ERR_CHECK instead of trapping, so the context stays usable.
 * The release build compiles the checks away. */
int samba_get_status(samba_stream_t stream);

/* Self-test of the failure path: launches one small kernel that waits on an
 * mbarrier nothing ever completes.  The bounded wait gives up after its limit
 * (200 ms), the kernel records SAMBA_ERR_TIMEOUT in the status word and
 * returns, and the CUDA context stays usable; samba_get_status(stream) then
 * returns SAMBA_ERR_TIMEOUT (and clears it).  Returns SAMBA_OK if the launch
 * was issued.  Not part of the mixers; it exists so the timeout handling can
 * be tested on a GPU without faulting or hanging it. */
int samba_selftest_wait_timeout(samba_stream_t stream);

/* Self-test of the debug build's checks: launches one small kernel whose
 * guarded store has an index past its (16-element, library-owned) buffer;
 * the check skips the store and records SAMBA_ERR_CHECK, which
 * samba_get_status(stream) then returns.  Returns SAMBA_OK if the launch was
 * issued, SAMBA_ERR_UNSUPPORTED in the release build (no checks there). */
int samba_selftest_check(samba_stream_t stream);

/* ------------------------------------------------------------------ conv1d
 * Causal depthwise conv1d over time, the conv that a Mamba layer puts in front
 * of its selective scan.  The pages do not print this step: their Mamba
 * equations start from the scan input x_t.  It is part of the Mamba layer
 * that Samba builds on, and this library runs it fused inside
 * samba_selective_scan_fwd (SAMBA_SCAN_FUSE_CONV); this standalone form
 * exists for callers that want u itself.
 *   u[b,t,c] = bias[c] + sum_{k<K} w[c,k] * xpad[b,t+k,c],  then SiLU if silu,
 * where xpad is x preceded by the K-1 inputs of conv_state_in (oldest first;
 * zeros when conv_state_in is NULL), so w[c,K-1] multiplies x_t.
 *
 *   x              [B, L, D]   x_dtype (SAMBA_F32 or SAMBA_BF16)
 *   w              [D, K]      fp32
 *   bias           [D]         fp32, or NULL (no bias)
 *   conv_state_in  [B, D, K-1] fp32, or NULL (zeros)
 *   u              [B, L, D]   u_dtype
 *   conv_state_out [B, D, K-1] fp32, or NULL: the last K-1 entries of xpad.
 *                  May be conv_state_in itself only when L = 1 (a decode
 *                  step: one launch then updates the state in place);
 *                  otherwise it may not alias conv_state_in.
 * K must be 2..4; B, L >= 1; D >= 1.  L may be smaller than K-1.
 * Errors: SAMBA_ERR_INVALID_ARG for a missing x, w or u, a bad shape, a
 * misaligned x or u, or conv_state_out == conv_state_in with L > 1;
 * SAMBA_ERR_UNSUPPORTED for K outside 2..4 or another dtype.
 */
int samba_conv1d_fwd(const void* x, int x_dtype, const float* w, const float* bias,
                     const float* conv_state_in, void* u, int u_dtype, float* conv_state_out,
                     int64_t batch, int64_t seqlen, int64_t dim, int dconv, int silu,
                     samba_stream_t stream);

/* ------------------------------------------------------------------- scan
 * Selective-scan prefill, fused with the conv, softplus, D skip and gate:
 *   u      = SiLU(conv1d(x))  with SAMBA_SCAN_FUSE_CONV (|CONV_SILU), else x
 *   Δ      = softplus(delta)  with SAMBA_SCAN_DELTA_SOFTPLUS, else delta
 *   h_t[n] = exp(Δ_t A[c,n]) h_{t-1}[n] + Δ_t B_t[n] u_t        (fp32 state)
 *   y_t    = (sum_n C_t[n] h_t[n] + Dskip[c] u_t) * silu(z_t)
 * for every batch b and channel c, t = 0..L-1, starting from h0 (zeros if
 * NULL).  B and C are shared by all channels (one group).
 * With delta_sum, the call also writes sum_t Δ_t per (b, c): the decay of
 * state n over the whole call is exp(A[c,n] * delta_sum[b,c]), which is what
 * samba_scan_carry needs to join this segment of a longer sequence to the
 * segment before it (see there).
 * Errors: SAMBA_ERR_INVALID_ARG for a missing x, delta, A, Bm, Cm, y (or
 * conv_w with FUSE_CONV), D not a multiple of 8, unknown flag bits or a
 * pointer not 16-byte aligned; SAMBA_ERR_UNSUPPORTED for B > 65535,
 * L >= 2^31 - 1024, N or K outside the sets below, or z_dtype != x_dtype.
 */
typedef struct samba_scan_args {
  const void* x;               /* [B, L, D]   x_dtype                         */
  const void* z;               /* [B, L, D]   z_dtype, or NULL (no gate)      */
  const float* delta;          /* [B, L, D]   fp32                            */
  const float* A;              /* [D, N]      fp32                            */
  const float* Bm;             /* [B, L, N]   fp32                            */
  const float* Cm;             /* [B, L, N]   fp32                            */
  const float* Dskip;          /* [D]         fp32, or NULL (no skip)         */
  const float* conv_w;         /* [D, K]      fp32 (needed with FUSE_CONV)    */
  const float* conv_b;         /* [D]         fp32, or NULL                   */
  const float* conv_state_in;  /* [B, D, K-1] fp32, or NULL (zeros)           */
  float* conv_state_out;       /* [B, D, K-1] fp32, or NULL                   */
  const float* h0;             /* [B, D, N]   fp32, or NULL (zeros)           */
  float* h_final;              /* [B, D, N]   fp32, or NULL; may alias h0     */
  void* y;                     /* [B, L, D]   y_dtype                         */
  int64_t batch, seqlen, dim;  /* B >= 1, L >= 1, D >= 1 with D % 8 == 0      */
  int32_t dstate, dconv;       /* N in {4, 8, 16}; K in 2..4                  */
  int32_t x_dtype, z_dtype, y_dtype;
  uint32_t flags;
  float* delta_sum;            /* [B, D] fp32, or NULL: sum over t of Δ_t     */
  float* h_ckpt;               /* [B, ceil(L/16), N, D] fp32, or NULL: the
                                  state at the start of every 16-token chunk
                                  (h0 for the first), the checkpoints
                                  samba_selective_scan_bwd can start from     */
} samba_scan_args;

int samba_selective_scan_fwd(const samba_scan_args* args, samba_stream_t stream);

/* --------------------------------------------------------- scan backward
 * Reverse-mode gradients of samba_selective_scan_fwd's output y (the
 * recurrence of page "SAMBA混合注意力状态空间模型", section 数学框架 /
 * Mamba层, with the forward's readings): given dy = ∂L/∂y, the call writes
 * ∂L/∂ of every input.  With G_t = ∂L/∂h_t = C_t g_t + exp(Δ_{t+1} A) G_{t+1}
 * and g_t = dy_t silu(z_t):
 *   dC_t = Σ_c g_t h_t      dB_t = Σ_c G_t Δ_t u_t     dA = Σ_{b,t} G_t Δ_t Ā_t h_{t-1}
 *   dΔ_t = Σ_n G_t (A Ā_t h_{t-1} + B_t u_t)          du_t = D g_t + Δ_t Σ_n G_t B_t
 *   dD = Σ_{b,t} g_t u_t    dz_t = dy_t (C_t·h_t + D u_t) silu'(z_t)   dh0 = Ā_0 G_0
 * then ddelta = dΔ σ(delta) (with DELTA_SOFTPLUS) and, with FUSE_CONV, the
 * gradients through the conv's SiLU and the depthwise conv (dx, dconv_w,
 * dconv_b, dconv_state).  The forward states are recomputed: a first pass
 * stores the state at the start of every 16-token chunk in the workspace,
 * then every chunk is recomputed and walked from its last token to its first.
 * When `ckpt` holds the checkpoints the forward wrote (samba_scan_args.h_ckpt,
 * same inputs), the first pass is skipped and the chunks start from them.
 *
 * Inputs are those of the forward (same shapes, dtypes and flags; y_dtype is
 * the dtype of dy).  Outputs:
 *   dx      [B, L, D]  x_dtype          ddelta [B, L, D] fp32
 *   dz      [B, L, D]  x_dtype, required iff z is given
 *   dA      [D, N]     fp32 (summed over the batch)
 *   dB, dC  [B, L, N]  fp32 (summed over the channels)
 *   dD      [D]        fp32, required iff Dskip is given
 *   dconv_w [D, K], dconv_b [D] fp32, required with FUSE_CONV (dconv_b iff conv_b)
 *   dh0     [B, D, N]  fp32, or NULL
 *   dconv_state [B, D, K-1] fp32, or NULL (meaningful with FUSE_CONV)
 * dA, dB, dC, dD, dconv_w and dconv_b are sums of contributions added with
 * atomics: the call clears them on the stream first, and their summation
 * order (hence the last bits) varies between runs.  The workspace is
 * caller-owned device memory of samba_scan_bwd_workspace_size() bytes,
 * 16-byte aligned; nothing else is allocated.
 * Errors: as samba_selective_scan_fwd for the inputs, plus
 * SAMBA_ERR_INVALID_ARG for a missing dy, dx, ddelta, dA, dB or dC, a missing
 * dz / dD / dconv_w / dconv_b where the forward input exists, or a misaligned
 * pointer; SAMBA_ERR_WORKSPACE for a missing or short workspace.
 */
typedef struct samba_scan_bwd_args {
  const void* x;               /* forward inputs, as samba_scan_args           */
  const void* z;
  const float* delta;
  const float* A;
  const float* Bm;
  const float* Cm;
  const float* Dskip;
  const float* conv_w;
  const float* conv_b;
  const float* conv_state_in;
  const float* h0;
  const void* dy;              /* [B, L, D]   y_dtype                          */
  void* dx;                    /* [B, L, D]   x_dtype                          */
  float* ddelta;               /* [B, L, D]                                    */
  void* dz;                    /* [B, L, D]   x_dtype, iff z                   */
  float* dA;                   /* [D, N]                                       */
  float* dB;                   /* [B, L, N]                                    */
  float* dC;                   /* [B, L, N]                                    */
  float* dD;                   /* [D], iff Dskip                               */
  float* dconv_w;              /* [D, K], with FUSE_CONV                       */
  float* dconv_b;              /* [D], with FUSE_CONV and conv_b               */
  float* dh0;                  /* [B, D, N] or NULL                            */
  float* dconv_state;          /* [B, D, K-1] or NULL                          */
  void* workspace;             /* samba_scan_bwd_workspace_size() bytes        */
  size_t workspace_bytes;
  int64_t batch, seqlen, dim;  /* as the forward                               */
  int32_t dstate, dconv;
  int32_t x_dtype, z_dtype, y_dtype;
  uint32_t flags;
  const float* ckpt;           /* NULL, or the forward's h_ckpt for these inputs:
                                  the first pass is then skipped              */
} samba_scan_bwd_args;

/* Bytes of workspace samba_selective_scan_bwd needs (the chunk checkpoints,
 * B * ceil(L/16) * N * D fp32); SIZE_MAX if that overflows. */
size_t samba_scan_bwd_workspace_size(int64_t batch, int64_t seqlen, int64_t dim, int32_t dstate);

int samba_selective_scan_bwd(const samba_scan_bwd_args* args, samba_stream_t stream);

/* ---------------------------------------------------------- SWA backward
 * Reverse-mode gradients of samba_swa_fwd (the banded attention of page
 * "SAMBA混合注意力状态空间模型", section 滑动窗口注意力, causal band
 * 0 <= i - j < W, grouped kv heads).  With P the softmax, dO = ∂L/∂o and
 * D_i = dO_i · o_i:  dv_j = Σ_i P_ij dO_i,  dS_ij = P_ij (dO_i · v_j - D_i),
 * dq_i = scale Σ_j dS_ij k_j,  dk_j = scale Σ_i dS_ij q_i, the kv gradients
 * summed over the query heads that read the kv head.  P is recomputed from
 * q, k and the forward's log-sum-exp (samba_swa_args.lse).
 *
 *   q, dO, o   [B, L, Hq, d]   bf16  (o and lse: the forward's outputs)
 *   k, v       [B, L, Hkv, d]  bf16
 *   lse        [B, Hq, L]      fp32, natural log
 *   dq         [B, L, Hq, d]   bf16, written
 *   dk, dv     [B, L, Hkv, d]  bf16, written
 * Shapes, scale and limits as samba_swa_fwd.  The workspace is caller-owned
 * device memory of samba_swa_bwd_workspace_size() bytes, 16-byte aligned
 * (per row: the base-2 log-sum-exp and D).  Three kernels run on the stream:
 * the per-row terms, then dk/dv (one CTA per 128-key tile), then dq.
 * Errors: as samba_swa_fwd, plus SAMBA_ERR_INVALID_ARG for a missing o,
 * lse, dO, dq, dk or dv or a misaligned pointer, SAMBA_ERR_WORKSPACE for a
 * missing or short workspace.
 */
typedef struct samba_swa_bwd_args {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const float* lse;
  const void* dO;
  void* dq;
  void* dk;
  void* dv;
  void* workspace;
  size_t workspace_bytes;
  int64_t batch, seqlen, window;
  int32_t heads_q, heads_kv, head_dim;
  float scale;                 /* 0: 1/sqrt(d)                                 */
} samba_swa_bwd_args;

size_t samba_swa_bwd_workspace_size(int64_t batch, int64_t seqlen, int32_t heads_q);

int samba_swa_bwd(const samba_swa_bwd_args* args, samba_stream_t stream);

/* The backward of both mixers (a training step's gradients of the two token
 * mixers; their backward passes are independent): samba_selective_scan_bwd
 * and samba_swa_bwd on their own arguments, with the same checks and errors.
 * With aux == NULL both run in order on `stream`; otherwise the scan's
 * backward runs on `stream` and the attention's on `aux`, forked from and
 * joined back into `stream` with events, so that the attention's kernels can
 * take the SMs the scan's last wave leaves free and the call as a whole stays
 * ordered on `stream`. */
int samba_mixer_bwd(const samba_scan_bwd_args* scan, const samba_swa_bwd_args* swa, samba_stream_t stream,
                    samba_stream_t aux);

/* ------------------------------------------------------ sequence segments
 * A sequence split into consecutive segments (for example one per GPU) can be
 * scanned segment by segment with exactly the result of one pass, because the
 * recurrence is linear in its state: over a segment s, the final state is
 *   h_end(s) = exp(A * dsum(s)) ⊙ h_start(s) + h_local(s),
 * where h_local(s) is the final state of the segment scanned from zero and
 * dsum(s) = sum_t Δ_t over the segment (samba_scan_args.delta_sum).  So every
 * segment can first be scanned from zero (giving h_local and dsum), the
 * segments' start states follow by folding this carry from the first segment
 * on, and a second pass from the right start state gives the outputs.  The
 * page's recurrence (section 数学框架 / Mamba层) is the same in every segment;
 * the split is only an order of evaluation.
 *
 * samba_scan_carry: h_out = exp(A ⊙ dsum) ⊙ h_in + h_local, elementwise over
 * [B, D, N] (A [D, N] fp32, dsum [B, D] fp32, h_in, h_local, h_out
 * [B, D, N] fp32; h_in may be NULL for a zero start state; h_out may alias
 * h_in or h_local).  exp is evaluated as the scan evaluates its decays.
 * Errors: SAMBA_ERR_INVALID_ARG for a missing A, dsum, h_local or h_out or a
 * non-positive size; SAMBA_ERR_UNSUPPORTED for N outside {4, 8, 16}.
 */
int samba_scan_carry(const float* h_in, const float* dsum, const float* A, const float* h_local, float* h_out,
                     int64_t batch, int64_t dim, int dstate, samba_stream_t stream);

/* samba_conv_state: the conv state a segment hands to the next one, the last
 * K-1 inputs of (conv_state_in, x) ([B, D, K-1] fp32, oldest first), without
 * computing the conv.  x is [B, L, D] x_dtype (L >= 0); conv_state_in is
 * [B, D, K-1] fp32 or NULL (zeros); conv_state_out may not alias it.  Equals
 * the conv_state_out of samba_selective_scan_fwd and samba_conv1d_fwd.
 * Errors: SAMBA_ERR_INVALID_ARG for a missing x or conv_state_out, aliasing,
 * or a bad shape; SAMBA_ERR_UNSUPPORTED for K outside 2..4 or a dtype. */
int samba_conv_state(const void* x, int x_dtype, const float* conv_state_in, float* conv_state_out,
                     int64_t batch, int64_t seqlen, int64_t dim, int dconv, samba_stream_t stream);

/* -------------------------------------------------------------------- SWA
 * Causal sliding-window attention prefill with grouped KV heads:
 *   o[b,i,h] = sum_{j : 0 <= i-j < W} softmax_j(scale * q[b,i,h] . k[b,j,g])
 *              * v[b,j,g],   g = h / (Hq / Hkv)
 * computed with tcgen05 bf16 MMAs (fp32 accumulate in tensor memory) and an
 * fp32 online softmax; o is rounded to bf16 once.  lse (optional) receives the
 * natural-log logsumexp of the scaled scores of every row.
 * W >= L gives plain causal attention.
 * Errors: SAMBA_ERR_INVALID_ARG for a missing q, k, v or o, a non-positive
 * size, Hq not a multiple of Hkv or a pointer not 16-byte aligned;
 * SAMBA_ERR_UNSUPPORTED for Hq/Hkv outside {1, 2, 4, 8, 16}, d outside
 * {16, 32, 64}, B > 65535 or L > 2^30.
 */
typedef struct samba_swa_args {
  const void* q;      /* [B, L, Hq, d]   bf16 */
  const void* k;      /* [B, L, Hkv, d]  bf16 */
  const void* v;      /* [B, L, Hkv, d]  bf16 */
  void* o;            /* [B, L, Hq, d]   bf16 */
  float* lse;         /* [B, Hq, L]      fp32, or NULL */
  int64_t batch, seqlen, window;   /* B >= 1, L >= 1, W >= 1 */
  int32_t heads_q, heads_kv, head_dim;  /* Hq % Hkv == 0, Hq/Hkv in {1,2,4,8,16}; d in {16,32,64} */
  float scale;        /* softmax scale; <= 0 selects 1/sqrt(d) */
} samba_swa_args;

int samba_swa_fwd(const samba_swa_args* args, samba_stream_t stream);

/* ------------------------------------------------------------- projections
 * The linear maps around the two mixers (a Mamba layer's input projection to
 * x and z, its selective-parameter projection to the low-rank Δ, B and C, the
 * Δ up-projection, its output projection; the attention's Q/K/V and output
 * projections: page "SAMBA混合注意力状态空间模型", section 数学框架 /
 * Mamba层, B_t = Linear_B(x_t), C_t = Linear_C(x_t), Δ_t = τ_Δ(Linear_Δ(x_t)))
 * as one GEMM on the tensor cores:
 *   C[m, n] = sum_k A[m, k] * B[n, k]     (bf16 inputs, fp32 accumulation)
 * A is [M, K] with row stride lda, B is [N, K] with row stride ldb (a
 * weight in the usual [out_features, in_features] layout), both bf16,
 * 16-byte aligned, lda and ldb multiples of 8.  The columns of C go to up to
 * three outputs: out[i] receives columns [col0, col1) as a row-major
 * [M, col1 - col0] matrix with row stride ld (elements), in bf16 or fp32,
 * plus bias[col - col0] when bias is not NULL.  Columns outside every range
 * are dropped.
 *
 * Workspace (optional; only for M <= 32, a decode step's rows): with a
 * workspace of at least samba_gemm_workspace_size(M, N) bytes the call
 * splits K over all SMs, so that the whole weight is streamed at once even
 * though C has few tiles; partial sums meet in the workspace in fp32 (their
 * order of addition, hence the last bits of C, may vary from run to run).
 * The workspace is caller-owned device memory, 16-byte aligned, and must be
 * zero-filled before its first use; every call that returns SAMBA_OK and
 * completes without a device error leaves it zero-filled again, so one
 * workspace serves any number of calls made one after another (on one
 * stream, or otherwise ordered).  Calls that may run at the same time need
 * workspaces of their own.  After a call whose status word reports an error
 * its content is undefined: fill it with zeros again.  Without a workspace
 * (NULL, or fewer bytes) the call tiles C as usual.
 * Errors: SAMBA_ERR_INVALID_ARG for a missing operand or output, a
 * non-positive size, a stride below its row length or not a multiple of 8, an
 * empty or out-of-range column range or a misaligned pointer (workspace
 * included);
 * SAMBA_ERR_UNSUPPORTED for M above 65535 * 128, N or K above 2^31 - 1, an
 * output dtype other than SAMBA_F32 / SAMBA_BF16, or nout outside 1..3.
 */
typedef struct samba_gemm_out {
  void* ptr;          /* [M, col1 - col0] row-major, row stride ld        */
  const float* bias;  /* [col1 - col0] fp32, or NULL                      */
  int64_t ld;
  int64_t col0, col1;
  int32_t dtype;      /* SAMBA_F32 or SAMBA_BF16                          */
} samba_gemm_out;

typedef struct samba_gemm_args {
  const void* A;      /* [M, K] bf16, row stride lda                      */
  const void* B;      /* [N, K] bf16, row stride ldb                      */
  int64_t lda, ldb;
  int64_t M, N, K;
  samba_gemm_out out[3];
  int32_t nout;
  void* workspace;         /* NULL, or samba_gemm_workspace_size() bytes (see above) */
  size_t workspace_bytes;
} samba_gemm_args;

int samba_gemm(const samba_gemm_args* args, samba_stream_t stream);

/* Bytes of workspace the split-K form of samba_gemm needs for M rows and N
 * columns (for M <= 32; 0 otherwise, when no workspace is used). */
size_t samba_gemm_workspace_size(int64_t M, int64_t N);

/* ------------------------------------------------------------ mixer prefill
 * One Mamba mixer (scan) and one SWA mixer on their own inputs (the two token
 * mixers of a Samba block: the forward pseudo-code of the page's section
 * 推理效率 runs mamba(x), then swa(x) after the MLP).  The two are independent: with aux == NULL both run
 * in order on `stream`; otherwise the attention runs on `aux`, forked from
 * and joined back into `stream` with events, so that the call as a whole is
 * still ordered on `stream`.
 */
int samba_mixer_prefill(const samba_scan_args* scan, const samba_swa_args* swa,
                        samba_stream_t stream, samba_stream_t aux);

/* ------------------------------------------------------------- decode: scan
 * One token of the selective scan (mamba_step): updates h and the conv state
 * in place and writes y_t.  Same arithmetic as the prefill with L = 1.
 *   h          [B, D, N]   fp32, read and written
 *   conv_state [B, D, K-1] fp32, read and written (oldest first)
 *   x_t, z_t   [B, D]      x_dtype / z_dtype (z_t may be NULL)
 *   delta_t    [B, D]      fp32 (softplus applied with DELTA_SOFTPLUS)
 *   B_t, C_t   [B, N]      fp32;  A [D, N], Dskip [D] (or NULL), conv_w
 *                          [D, K], conv_b [D] (or NULL) as in the prefill
 *   y_t        [B, D]      y_dtype
 * flags: as samba_scan_args.flags (FUSE_CONV requires conv_state and conv_w).
 * B <= 65535 (SAMBA_ERR_UNSUPPORTED beyond); N in {4, 8, 16}; K in 2..4;
 * z_dtype == x_dtype.  h, A, B_t and C_t must be 16-byte aligned
 * (SAMBA_ERR_INVALID_ARG otherwise): the states are read as vectors.
 */
int samba_scan_step(float* h, float* conv_state, const void* x_t, int x_dtype, const void* z_t,
                    int z_dtype, const float* delta_t, const float* B_t, const float* C_t,
                    const float* A, const float* Dskip, const float* conv_w, const float* conv_b,
                    void* y_t, int y_dtype, int64_t batch, int64_t dim, int dstate, int dconv,
                    uint32_t flags, samba_stream_t stream);

/* -------------------------------------------------------------- decode: SWA
 * Ring-buffer KV window.  Slot p mod W of k_ring/v_ring holds the key/value
 * of absolute position p; pos[b] is the next position of sequence b.
 *
 * k_ring, v_ring are [B, W, Hkv, d] bf16; head_dim d is 16, 32, 64 or 128
 * (SAMBA_ERR_UNSUPPORTED otherwise).
 *
 * samba_swa_ring_fill: after a prefill of L tokens (L >= 0), copy the last
 * min(L, W) keys/values of k, v ([B, L, Hkv, d] bf16) into their slots and
 * set pos[b] = L.  Slots of positions < L - W are left untouched.  This is the
 * hand-off of the page's inference pseudo-code (section 推理效率): its
 * forward(prompt) leaves the window's keys and values in the cache that the
 * following swa_step calls read.
 * Limits of the ring (every decode SWA entry point): W <= 2^30 and
 * Hkv <= 65535 (SAMBA_ERR_UNSUPPORTED beyond).
 */
int samba_swa_ring_fill(const void* k, const void* v, int64_t seqlen, void* k_ring, void* v_ring,
                        int64_t* pos, int64_t batch, int heads_kv, int head_dim, int64_t window,
                        samba_stream_t stream);

/* Bytes of device workspace samba_swa_step needs for these sizes; 0 for a
 * non-positive size, SIZE_MAX when the byte count does not fit in size_t. */
size_t samba_swa_step_workspace_size(int64_t batch, int heads_q, int head_dim, int64_t window);

/* samba_swa_step (swa_step): writes k_t, v_t ([B, Hkv, d]) into slot
 * pos[b] mod W, then each query q_t ([B, Hq, d]) attends the keys of
 * positions max(0, pos-W+1) .. pos and writes o_t ([B, Hq, d] bf16); finally
 * pos[b] += 1.  All of it happens on the device (pos is a device int64 [B]),
 * so consecutive steps can be captured in one CUDA graph.  `workspace` is
 * caller-owned device memory of at least samba_swa_step_workspace_size()
 * bytes (split partial results); it needs no initialisation.  scale <= 0
 * selects 1/sqrt(d).
 * Errors: SAMBA_ERR_INVALID_ARG for a null pointer, a non-positive size, Hq
 * not a multiple of Hkv or a pointer (workspace included) not 16-byte
 * aligned; SAMBA_ERR_UNSUPPORTED for Hq/Hkv > 16, d outside the set above
 * or B > 65535; SAMBA_ERR_WORKSPACE for a missing or smaller workspace.
 */
int samba_swa_step(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring,
                   int64_t* pos, void* o_t, int64_t batch, int heads_q, int heads_kv, int head_dim,
                   int64_t window, float scale, void* workspace, size_t workspace_bytes,
                   samba_stream_t stream);

/* samba_swa_step_noalloc: the same decode step as samba_swa_step, for
 * callers that cannot allocate device memory.  Examples are a host framework
 * that owns every device allocation and hands plug-ins only tensors, or code
 * running where a cudaMalloc would be refused or would synchronise the device.
 * Such a caller has no way to pass samba_swa_step a workspace.
 *
 * The split partials live in a 4 MiB array inside the library (a file-scope
 * __device__ array), which every GPU that loads the library holds until the
 * process exits.  Calls whose partials do not fit, that is
 * samba_swa_step_workspace_size(batch, heads_q, head_dim, window) > 4 MiB,
 * are rejected with SAMBA_ERR_WORKSPACE before anything is launched; the
 * 16 x 32-head, d = 64, W = 2048 decode needs 2.16 MB.
 *
 * Every call looks up the array's device address (cudaGetSymbolAddress) on
 * the current device; this is a table lookup once the library's device code
 * is loaded there, and it keeps the address right after cudaDeviceReset.
 * The first call on a device may load that code, so make it before any
 * stream capture.  The function calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 * Every call shares the one array and finds the previous call's partials in
 * it.  That is harmless, because each step writes every partial it reads and
 * nothing has to start at zero.  But two calls that may run at the same time
 * on the GPU (different streams, or different threads without ordering)
 * race on the array and give wrong results; order them, or use
 * samba_swa_step with separate workspaces.
 *
 * Arguments, layouts and errors are those of samba_swa_step without the
 * workspace; the argument checks (SAMBA_ERR_UNSUPPORTED for B > 65535
 * included) come before the size check.  The paper has no counterpart to this entry point; it exists
 * only for callers that cannot allocate.
 */
int samba_swa_step_noalloc(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring,
                           int64_t* pos, void* o_t, int64_t batch, int heads_q, int heads_kv, int head_dim,
                           int64_t window, float scale, samba_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SAMBA_H_ */
