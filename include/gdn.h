/*
 * gdn.h — C ABI of libgdn.so: chunkwise causal linear attention (plain, gated),
 * DeltaNet and Gated DeltaNet prefill, plus the one-token recurrent decode step,
 * as hand-written CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * The operator (per head; dk x dv state S stored key-rows by value-columns):
 *     alpha_t = exp(g_t)                    (alpha_t = 1 when g is NULL)
 *     u_t     = beta_t (v_t - alpha_t S^T k_t)   (u_t = v_t when beta is NULL)
 *     S_t     = alpha_t S_{t-1} + k_t u_t^T
 *     o_t     = S_t^T (scale * q_t)
 * This is the Gated DeltaNet recurrence S_t = alpha_t S_{t-1}(I - beta_t k k^T)
 * + beta_t v k^T written in the transposed (dk, dv) storage layout.
 * Sources: "混合注意力学习(1): 线性注意力" (sections "Fast Weight Programmers与DeltaNet",
 * "Gated DeltaNet", "FWP分块并行机制", "DeltaNet 分块并行机制", "HouseHolder变换和WY表示");
 * "LinearAttention 概述" (sections "FLASH", "Lightning Attention": the chunkwise
 * form is exact and position t sees 1..t inclusive); "【CS336】lecture4 线性注意力|
 * Mamba|GDN|DSA" (sections "朴素线性注意力", "继续改进：Mamba", "继续改进：GDN").
 *
 * Conventions for every entry point
 *  - Ownership: the caller allocates and owns every buffer (device memory unless
 *    stated). Three prefill forms take a stream-ordered workspace from a memory pool the
 *    library creates per device, and release it on the stream once their kernels have
 *    run (the pool keeps what it reserved for later calls): vector-valued gates on the
 *    tensor cores, Gated DeltaNet over few heads with long sequences (dense bf16 calls at
 *    dk = dv = 128, chunk 64, with at most a third of the SM count of (sequence, head)
 *    pairs and at least 128 chunks), and bf16 calls with dk or dv = 64 that take
 *    zero-padded copies (below); if that memory cannot be had they run on kernels that need none. Otherwise the library allocates no memory and keeps no
 *    per-call state; its only state is per device: the condition word that
 *    gdn_sync_status reads, cached kernel attributes, the wait limit of
 *    gdn_set_wait_limit_for_testing, the workspace pool and the two streams below.
 *  - Layout: dense, contiguous, row-major, as annotated. Device pointers must be
 *    16-byte aligned, except beta and g, which need 4-byte alignment.
 *  - Asynchrony: work is enqueued on `cuda_stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and the call returns without synchronising. The
 *    return value reports argument validation and launch errors only; a kernel
 *    that gave up on a bounded wait records it in a device-side word that
 *    gdn_sync_status() reads. The long-sequence form runs its kernels on two streams
 *    of the library's (after the work already on `cuda_stream`) and makes `cuda_stream`
 *    wait for the last of them, so later work on `cuda_stream` sees the results.
 *  - Errors: on any non-OK return nothing was enqueued (validation) or the
 *    launch failed (GDN_ERR_CUDA). No exceptions cross this boundary.
 *  - Aliasing: s_final may alias s0. q, k, v, beta, g must not alias o.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* NULL required pointer, bad size, misaligned pointer */
    GDN_ERR_UNSUPPORTED = 2,   /* valid but not implemented (head dim, chunk, dtype)  */
    GDN_ERR_CUDA = 3,          /* a CUDA runtime/driver call or launch failed          */
    GDN_ERR_TIMEOUT = 4,       /* a kernel gave up on a bounded wait (see sync_status) */
    GDN_ERR_NONFINITE = 5,     /* a tensor-core prefill stored inf / NaN in o or S_final
                                  (checked on a sample, see sync_status)               */
    GDN_ERR_BOUNDS = 6         /* bounds-checked debug build only: a kernel index fell
                                  outside its extent; the access was skipped            */
} gdn_status_t;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype_t;

/*
 * lin_attn_chunk_fwd — causal linear attention without normaliser, plain
 * (g == NULL: alpha = 1) or with a scalar per-token decay (g != NULL).
 * Page "混合注意力学习(1)" section "FWP分块并行机制" (chunk-mixed intra/inter form);
 * page "LinearAttention 概述" sections "快速预览" (O = (QK^T o M)V) and "Lightning
 * Attention" (positions 1..t inclusive); page "【CS336】lecture4" section
 * "继续改进：Mamba" (gated state decay).
 *
 *  q, k     (B, H, L, dk) in_dtype            device, read
 *  v        (B, H, L, dv) in_dtype            device, read
 *  g        (B, H, L) fp32 log-alpha (<= 0 expected), nullable
 *  o        (B, H, L, dv) fp32                device, written
 *  s0       (B, H, dk, dv) fp32 initial state, nullable (zero state)
 *  s_final  (B, H, dk, dv) fp32 final state,   nullable (not written)
 *  B, H >= 1; L >= 0 (L == 0: only s_final is written, = s0 or 0)
 *  dk, dv in {64, 128}; chunk: 1..64. bf16 inputs with chunk 64 run on the tensor-core
 *  kernels: at dk = dv = 128 directly, with dk or dv = 64 through copies of the operands
 *  zero-padded to 128 (the padded results, cropped, are the call's: zero key coordinates
 *  and value columns leave the other entries unchanged; a stream-ordered workspace from the
 *  library's pool, see Ownership; not with the output normalisation). Calls with the plain
 *  fp32 output and a scalar gate (or none) read the 64-wide operands directly instead (the
 *  same bits, no copies and no workspace): linear attention always, Gated DeltaNet on
 *  batches of enough (sequence, head) pairs for its one-CTA kernel (more than a third of the
 *  SM count). Every other
 *  combination runs on the fp32 chunk kernel (the same result within its tolerance, at
 *  CUDA-core speed).
 *  scale multiplies q.  in_dtype: GDN_BF16 or GDN_F32 (q, k, v share it).
 */
gdn_status_t lin_attn_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                                float *o, const float *s0, float *s_final,
                                int B, int H, int L, int dk, int dv, int chunk, float scale,
                                gdn_dtype_t in_dtype, void *cuda_stream);

/*
 * gdn_chunk_fwd — DeltaNet (g == NULL) or Gated DeltaNet (g != NULL), chunkwise:
 * per chunk the UT transform T = (I + tril(diag(beta) K K^T o Gamma, -1))^-1 by
 * forward substitution, W = T diag(beta gamma) K, U = T diag(beta) V, the
 * state-dependent pseudo-values U - W S_c, the output diag(gamma) Q S_c +
 * tril(Q K^T o Gamma)(U - W S_c) and the state scan
 * S_{c+1} = gamma_C S_c + K~^T (U - W S_c).
 * Page "混合注意力学习(1)" sections "DeltaNet 分块并行机制", "重新定义降低内存占用",
 * "HouseHolder变换和WY表示"; page "LinearAttention 概述" section "FLASH".
 *
 *  beta     (B, H, L) fp32, required (the delta term's learning rate)
 *  other arguments as for lin_attn_chunk_fwd. Few (sequence, head) pairs with long
 *  sequences (see Ownership above) run as a per-chunk prep kernel on every SM and a
 *  per-head chain kernel, in segments of 64 chunks whose prep overlaps the chain of the
 *  segment before; the same result within the tolerance of the tensor-core kernels.
 */
gdn_status_t gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *beta,
                           const float *g, float *o, const float *s0, float *s_final,
                           int B, int H, int L, int dk, int dv, int chunk, float scale,
                           gdn_dtype_t in_dtype, void *cuda_stream);

/*
 * Packed variable-length batches. N sequences of different lengths share one
 * head-major token grid: sequence n of head h is rows cu_seqlens[n] ..
 * cu_seqlens[n+1]-1 of row h of (H, T, d) tensors. Each (sequence, head) is an
 * independent recurrence with its own initial and final state. The pages serve
 * prefill and decode batches ("【CS336】lecture4", section "朴素线性注意力": the
 * prefill/decode split); packing sequences of different lengths is this library's
 * layout for such a prefill batch, with exactly the per-sequence result of the
 * dense entry points.
 *
 *  q, k        (H, T, dk) in_dtype; v (H, T, dv) in_dtype     device, read
 *  beta, g     (H, T) fp32 (g nullable)                        device, read
 *  o           (H, T, dv) fp32                                 device, written at the
 *              rows of the N sequences (rows outside every sequence are not written)
 *  s0, s_final (N, H, dk, dv) fp32, nullable as in the dense calls
 *  cu_seqlens  (N + 1) int32, device, 4-byte aligned: 0 <= cu[0] <= cu[1] <= ... <=
 *              cu[N] <= T. Sequences may be empty (then s_final = s0 or 0). The
 *              offsets are read on the device; a list that breaks this rule makes
 *              the affected (sequence, head) empty and is reported by the next
 *              gdn_sync_status() as GDN_ERR_INVALID_ARG.
 *  N, H >= 1; T >= 0; other arguments as for the dense calls.
 */
gdn_status_t lin_attn_chunk_fwd_varlen(const void *q, const void *k, const void *v, const float *g,
                                       float *o, const float *s0, float *s_final,
                                       const int *cu_seqlens, int N, int H, int T, int dk, int dv,
                                       int chunk, float scale, gdn_dtype_t in_dtype,
                                       void *cuda_stream);
gdn_status_t gdn_chunk_fwd_varlen(const void *q, const void *k, const void *v, const float *beta,
                                  const float *g, float *o, const float *s0, float *s_final,
                                  const int *cu_seqlens, int N, int H, int T, int dk, int dv,
                                  int chunk, float scale, gdn_dtype_t in_dtype, void *cuda_stream);

/*
 * Options of the *_ex prefill calls (zero-initialise, then set what is used; a NULL
 * options pointer means the defaults).
 *  out_dtype  dtype of o: GDN_F32 (default) or GDN_BF16 (each fp32 result rounded to
 *             the nearest bf16, ties to even; an option of this library that halves the
 *             output bytes).
 *  d_skip     (H, dv) fp32 device pointer, 4-byte aligned, nullable. When set, the
 *             output gains the skip term of Mamba: o_t += d_skip[h] (elementwise) v_t,
 *             v_t being the input value row (page "【CS336】lecture4", section
 *             "继续改进：Mamba": a term in v added at the output, like a residual
 *             connection, so the input reaches the output without the state).
 *  g_per_key  0 (default): g holds one log-decay per token, (B, H, L) or (H, T).
 *             1: vector-valued gate, g holds one log-decay per token and key
 *             coordinate, (B, H, L, dk) or (H, T, dk) fp32, and row j of the state
 *             decays by exp(g_t[j]):  S_t = (I - beta_t k_t k_t^T) diag(exp(g_t)) S_{t-1}
 *             + beta_t k_t v_t^T (without beta: S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T),
 *             the per-coordinate form of the scalar gate (GLA-style gates, next to the
 *             scalar gate of page "混合注意力学习(1)", section "Gated DeltaNet"). Dense
 *             bf16 calls with dk = dv = 128 and chunk 64 run on the tensor cores as two
 *             kernels (a per-chunk prep kernel, then a per-head chain kernel) and take a
 *             stream-ordered workspace of 74 240 bytes per chunk of 64 tokens from a memory
 *             pool the library owns (reserved memory stays in the pool for later calls); if
 *             that workspace cannot be had, and for every other dtype, size or layout, the
 *             call runs on the fp32 chunk kernel. Any other value: GDN_ERR_INVALID_ARG.
 *  xnorm      output normalisation (page "LinearAttention 概述", section "The Devil in Linear
 *             Transformer": the normaliser's denominator is dropped and the output is
 *             normalised instead, O = XNorm(Q (K^T V))). GDN_XNORM_NONE (0, default),
 *             GDN_XNORM_RMS: o_t <- w_h (elementwise) o_t / sqrt(mean(o_t^2) + eps), or
 *             GDN_XNORM_LAYER: o_t <- w_h (elementwise) (o_t - mean(o_t)) / sqrt(var(o_t)
 *             + eps), over the dv values of each output row of each head (var: mean square
 *             of the centred row), after the skip term and before the output rounding.
 *  xnorm_weight  (H, dv) fp32 device pointer, 4-byte aligned, nullable (w = 1).
 *  xnorm_eps  > 0 and finite when xnorm is set (e.g. 1e-6).
 *  An unknown xnorm value, or a non-positive eps with xnorm set, returns GDN_ERR_INVALID_ARG.
 */
typedef enum { GDN_XNORM_NONE = 0, GDN_XNORM_RMS = 1, GDN_XNORM_LAYER = 2 } gdn_xnorm_t;

typedef struct gdn_fwd_opts {
    gdn_dtype_t out_dtype;
    const float *d_skip;
    int g_per_key;
    int xnorm;                  /* gdn_xnorm_t */
    const float *xnorm_weight;
    float xnorm_eps;
} gdn_fwd_opts_t;

/*
 * lin_attn_chunk_fwd_ex / gdn_chunk_fwd_ex — the prefill calls with output options and
 * an optional packed layout:
 *  cu_seqlens == NULL: dense batch, arguments exactly as lin_attn_chunk_fwd /
 *                      gdn_chunk_fwd (B sequences, L tokens each, (B, H, L, d) tensors).
 *  cu_seqlens != NULL: packed batch, arguments as the *_varlen calls with B = N (the
 *                      number of sequences) and L = T (the packed length of each head).
 *  o          written in opts->out_dtype (fp32 when opts is NULL), same shape as before.
 *  opts       nullable, see gdn_fwd_opts_t; an unknown out_dtype or a misaligned d_skip
 *             returns GDN_ERR_INVALID_ARG.
 * Every other rule (sizes, alignment, aliasing, errors) is that of the dense / packed call.
 */
gdn_status_t lin_attn_chunk_fwd_ex(const void *q, const void *k, const void *v, const float *g, void *o,
                                   const float *s0, float *s_final, const int *cu_seqlens, int B, int H, int L,
                                   int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                                   const gdn_fwd_opts_t *opts, void *cuda_stream);
gdn_status_t gdn_chunk_fwd_ex(const void *q, const void *k, const void *v, const float *beta, const float *g,
                              void *o, const float *s0, float *s_final, const int *cu_seqlens, int B, int H, int L,
                              int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                              const gdn_fwd_opts_t *opts, void *cuda_stream);

/*
 * gdn_decode_step — one token for N independent sequences, state updated in place:
 *   u = beta (v - alpha S^T k);  o = alpha S^T q' + (q'.k) u;  S <- alpha S + k u^T
 * with q' = scale q (o equals S_new^T q'). The state is read once and written
 * once. Page "【CS336】lecture4" sections "朴素线性注意力" (O(d^2) per decoded token)
 * and "继续改进：GDN" (k^T S first keeps the erase term O(d^2)).
 *
 *  q, k   (N, H, dk) in_dtype; v (N, H, dv) in_dtype
 *  beta   (N, H) fp32, nullable (NULL: no delta term, u = v)
 *  g      (N, H) fp32 log-alpha, nullable (alpha = 1)
 *  state  (N, H, dk, dv) fp32, read and written in place
 *  o      (N, H, dv) fp32, written
 *  N, H >= 1; dk, dv in {64, 128}.
 */
gdn_status_t gdn_decode_step(const void *q, const void *k, const void *v, const float *beta,
                             const float *g, float *state, float *o, int N, int H, int dk,
                             int dv, float scale, gdn_dtype_t in_dtype, void *cuda_stream);

/*
 * gdn_decode_step_ex — gdn_decode_step with the options of gdn_fwd_opts_t (opts NULL: the
 * plain call). g_per_key = 1: g is (N, H, dk), row j of each state decays by
 * exp(g[n, h, j]) (o = (diag(alpha) S)^T q' + (q'.k) u, S <- diag(alpha) S + k u^T);
 * out_dtype GDN_BF16: o is bf16 (N, H, dv); d_skip (H, dv): o += d_skip[h] * v; xnorm:
 * the output normalisation of each o row, as in the prefill calls.
 * Validation as for gdn_decode_step, plus the options' own rules.
 */
gdn_status_t gdn_decode_step_ex(const void *q, const void *k, const void *v, const float *beta,
                                const float *g, float *state, void *o, int N, int H, int dk, int dv,
                                float scale, gdn_dtype_t in_dtype, const gdn_fwd_opts_t *opts,
                                void *cuda_stream);

/*
 * gdn_chunk_bwd — gradients of the prefill for training on full sequences (page
 * "混合注意力学习(1)", section "Transformers 就是 RNNs": on the full sequence every gradient
 * follows from the chain rule through the recurrence). For the loss
 * sum(o * d_o) + sum(S_final * ds_final) of the operator of lin_attn_chunk_fwd (beta ==
 * NULL) or gdn_chunk_fwd (beta != NULL), with the same q, k, v, beta, g, s0 and scale:
 *
 *  d_o       (B, H, L, dv) fp32, the gradient of o                    device, read
 *  ds_final  (B, H, dk, dv) fp32, nullable (zero)                     device, read
 *  dq, dk    (B, H, L, dk) fp32; dv (B, H, L, dv) fp32                device, written
 *  dbeta     (B, H, L) fp32, required when beta != NULL               device, written
 *  dg        (B, H, L) fp32 (gradient of the log-decay g), required when g != NULL
 *  ds0       (B, H, dk, dv) fp32, nullable (not written)              device, written
 *  workspace device memory of at least gdn_chunk_bwd_workspace_bytes(B, H, L, dk, dv, chunk)
 *            bytes, 16-byte aligned, owned by the caller; its contents on entry do not
 *            matter and on return are unspecified. It holds the state at the start of every
 *            chunk of `chunk` tokens and the recomputed states inside one chunk, per head.
 *  chunk     1..128: tokens between stored states (a memory / recompute trade-off; the
 *            result does not depend on it beyond rounding).
 *  The kernel runs on CUDA cores in fp32 (a reverse-mode pass over the token recurrence).
 *  Sizes, dtypes and alignment as for the prefill calls; L >= 0 (L == 0: ds0 = ds_final).
 */
size_t gdn_chunk_bwd_workspace_bytes(int B, int H, int L, int dk, int dv, int chunk);
gdn_status_t gdn_chunk_bwd(const void *q, const void *k, const void *v, const float *beta, const float *g,
                           const float *s0, const float *d_o, const float *ds_final, float *dq, float *dk,
                           float *dv, float *dbeta, float *dg, float *ds0, void *workspace,
                           size_t workspace_bytes, int B, int H, int L, int dk_size, int dv_size, int chunk,
                           float scale, gdn_dtype_t in_dtype, void *cuda_stream);

/*
 * gdn_chunk_bwd_noalloc — gdn_chunk_bwd for callers that cannot allocate device memory:
 * same arguments and results, without the workspace. (This entry point has no counterpart
 * in the pages; it is a deployment convenience of this library.) Some callers have no
 * allocator to hand when they run the backward — a plugin interface that passes only
 * input and output buffers, or a runtime whose allocator has reserved all device memory
 * up front so that a cudaMalloc would fail or fragment it — and cannot size and pass the
 * workspace that gdn_chunk_bwd needs.
 *
 *  Workspace: a fixed 16 MiB array in the library's static device memory (every device
 *  that loads the library holds it until the process exits). A call whose
 *  gdn_chunk_bwd_workspace_bytes(B, H, L, dk, dv, chunk) exceeds 16 MiB returns
 *  GDN_ERR_UNSUPPORTED and enqueues nothing (e.g. 2 heads of 4096 tokens at d = 128,
 *  chunk 64, need 16 MiB; use gdn_chunk_bwd for larger calls).
 *  The entry point calls no cudaMalloc, cudaFree or other allocating routine. Its first
 *  call on a device looks up the array's device address (cudaGetSymbolAddress, with that
 *  device current); make that first call before any stream capture.
 *  Every call on a device shares the array and leaves its last contents there (the backward
 *  writes every word it reads, so nothing needs clearing). Calls that overlap on the GPU
 *  race on the array: serialise them (one stream, or events between streams).
 */
gdn_status_t gdn_chunk_bwd_noalloc(const void *q, const void *k, const void *v, const float *beta,
                                   const float *g, const float *s0, const float *d_o, const float *ds_final,
                                   float *dq, float *dk, float *dv, float *dbeta, float *dg, float *ds0,
                                   int B, int H, int L, int dk_size, int dv_size, int chunk, float scale,
                                   gdn_dtype_t in_dtype, void *cuda_stream);

/*
 * Sequence-split (context-parallel) prefill: the segments of a long sequence run at once
 * (on several devices, or as the sequences of one packed launch). Over a segment the
 * token recurrence is affine in the state that enters it (page "混合注意力学习(1)",
 * section "Gated DeltaNet": each token maps the key-row state by
 * S -> alpha (I - beta k k^T) S + beta k v^T; plain and gated linear attention drop the
 * erase term): S_out = M S_in + N, with M the ordered product of the segment's token maps
 * and N the segment's end state from a zero start. With dk = dv = d, a prefill of the
 * segment from s0 = lambda I ends in lambda M + N and one from s0 = 0 ends in N; composing
 * these pairs in segment order gives the state entering each segment, from which a last
 * prefill of the segment gives its outputs. A large lambda (a power of two, e.g. 256) keeps
 * the rounding of N, which the composition subtracts, small next to M; it must keep
 * lambda M + N inside the prefill's fp16 operand range (|entries| well below 65504).
 *
 * gdn_state_compose — s_out = ((lambda M + N) - N) / lambda s_in + N for `count` states, fp32:
 *  mn        (count, d, d) fp32, the end states from s0 = lambda I      device, read
 *  n         (count, d, d) fp32, the end states from s0 = 0 (N)         device, read
 *  s_in      (count, d, d) fp32, nullable (zero: s_out = N)             device, read
 *  s_out     (count, d, d) fp32, must not overlap mn, n or s_in         device, written
 *  lambda    the diagonal of the s0 of the mn runs; finite, nonzero, 1/lambda finite
 *  d in {64, 128}; count >= 0 (0: nothing is enqueued); pointers 16-byte aligned.
 *  Returns GDN_ERR_INVALID_ARG for a NULL/misaligned pointer, an overlap or a bad lambda,
 *  GDN_ERR_UNSUPPORTED for another d.
 *
 * gdn_state_identity — writes value * I into `count` d x d fp32 states at `s` (the initial
 *  states of the s0 = lambda I runs); value finite; d in {64, 128}; s 16-byte aligned.
 */
gdn_status_t gdn_state_compose(const float *mn, const float *n, const float *s_in, float *s_out, float lambda,
                               int count, int d, void *cuda_stream);
gdn_status_t gdn_state_identity(float *s, float value, int count, int d, void *cuda_stream);

/*
 * gdn_chunk_fwd_host — gdn_chunk_fwd from pinned host buffers, the copies overlapped with the
 * computation (a serving step whose inputs are in host memory). The batch crosses PCIe in
 * groups of `group` sequences: while group i is computed, group i + 1 is uploaded and group
 * i - 1 downloaded, on three streams of the library's own (created and released by the call)
 * with two staging slots in `staging`; every tensor of a group is one cudaMemcpyAsync. Each
 * group is one dense prefill, and the (sequence, head) recurrences are independent, so the
 * result equals one gdn_chunk_fwd on the whole batch, bit for bit.
 *
 *  q, k, v, beta, g, s0    as gdn_chunk_fwd, in page-locked (pinned) host memory
 *  o, s_final              as gdn_chunk_fwd, in pinned host memory (s_final nullable)
 *  staging                 device memory of at least gdn_chunk_fwd_host_staging_bytes(...)
 *                          bytes, 256-byte aligned, owned by the caller (contents on entry
 *                          irrelevant, unspecified on return)
 *  group                   sequences per transfer (>= 1)
 *  cuda_stream             the caller's stream: the call's work starts after the work already
 *                          enqueued on it, and work enqueued on it afterwards starts after the
 *                          call's last download. The call returns without waiting.
 *  Returns GDN_ERR_INVALID_ARG for a pageable or NULL required host pointer, a staging buffer
 *  too small or misaligned, or a bad size (L >= 1); other rules as gdn_chunk_fwd.
 */
size_t gdn_chunk_fwd_host_staging_bytes(int B, int H, int L, int dk, int dv, int group, gdn_dtype_t in_dtype,
                                        int has_g, int has_s0, int has_s_final);
gdn_status_t gdn_chunk_fwd_host(const void *q, const void *k, const void *v, const float *beta, const float *g,
                                float *o, const float *s0, float *s_final, void *staging, size_t staging_bytes,
                                int B, int H, int L, int dk, int dv, int chunk, float scale, gdn_dtype_t in_dtype,
                                int group, void *cuda_stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char *gdn_status_str(gdn_status_t status);

/*
 * gdn_sync_status — synchronise `cuda_stream`, then report and clear one device-side
 * condition met by a kernel of this library on the current device since it was last
 * reported, in this order: GDN_ERR_INVALID_ARG for a malformed cu_seqlens list,
 * GDN_ERR_TIMEOUT for a bounded wait that gave up, GDN_ERR_BOUNDS (only in the library built
 * with -DGDN_DEBUG_BOUNDS, libgdn_debug.so) when a kernel's global access index fell outside
 * the extent its launch implies, GDN_ERR_NONFINITE when a tensor-core
 * prefill kernel found inf or NaN among the results it stored (non-finite inputs, or an
 * intermediate beyond the fp16 operand range, |x| > 65504, of those kernels). The kernels
 * check the last 64-token output tile of each sequence and its final state: a non-finite
 * value in the state reaches both, while one confined to rows of an earlier tile (inputs
 * whose q or q.k exceed the fp16 range) can go unreported;
 * GDN_OK when none is pending, GDN_ERR_CUDA if the stream or the read failed. When several
 * conditions are pending the next calls report the others. The conditions live in one word per device, shared by
 * every caller and stream of this process: a condition raised by another caller's kernel
 * is reported to whichever caller asks first. The word is taken with a one-thread kernel
 * on `cuda_stream` (atomic, so a condition raised meanwhile on another stream is kept).
 */
gdn_status_t gdn_sync_status(void *cuda_stream);

/*
 * gdn_set_wait_limit_for_testing — for tests of the failure path only: the number of
 * clock cycles each bounded wait of the tensor-core prefill kernels may take before it
 * gives up (default about 2 s; cycles <= 0 restores the default). It applies to kernels
 * launched after the call, from any thread. With a limit of a few hundred cycles the waits
 * give up while the work they wait for is still legitimately in flight: the kernel then
 * stops issuing, waits for the copies and tensor-core products it has already issued
 * (always with the default limit), frees its tensor memory and returns, and the next
 * gdn_sync_status reports GDN_ERR_TIMEOUT; the outputs of that launch are undefined.
 */
void gdn_set_wait_limit_for_testing(long long cycles);

/* Library version as major*10000 + minor*100 + patch. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GDN_H_ */
