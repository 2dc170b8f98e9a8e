/*
 * kda.h -- C ABI of libkda, the B200 (sm_100a) implementation of Kimi Delta
 * Attention (KDA): chunked prefill and single-token recurrent decode.
 *
 * The operator. Per (batch b, head h) a d_k x d_v fp32 state S evolves token by
 * token as
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t,        alpha_t = exp(log_alpha_t) in (0,1]^{d_k}.
 * Kimi Linear summary (es.news.hada.io/topic?id=31936): section "De la atencion
 * lineal a Gated DeltaNet" gives the delta rule as a rank-1 generalised
 * Householder update and GDN's forget gate; section "Control fino de memoria en
 * Kimi Delta Attention" makes the gate diagonal and per channel, a
 * Diagonal-Plus-Low-Rank transition tied to the key; section "Algoritmo
 * paralelo por chunks" gives the chunked form that kda_chunk_fwd evaluates.
 * There is no scale factor on q and no grouped heads: q, k, v all have H heads.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *    16-byte aligned. The library never allocates, frees or keeps a pointer
 *    after the call returns.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*, NULL = the
 *    legacy default stream) and the call returns without synchronising.
 *  - Errors are returned as kda_status codes (never thrown, never trapped).
 *    Argument errors are detected on the host before anything is enqueued;
 *    kda_last_error_detail() names the offending argument.
 *  - Preconditions that are documented but not checked (checking would cost a
 *    pass over the data): log_alpha <= 0, beta in [0,1], finite inputs. Any
 *    decay is supported: no gate factor of the chunked form leaves the
 *    floating-point range, whatever log_alpha is (16-token sub-chunks, see
 *    kda_chunk_fwd). L2 normalisation of q and k is the caller's job.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = -1,    /* NULL where a pointer is required, negative size, bad enum */
    KDA_ERR_UNSUPPORTED = -2,    /* shape, chunk or dtype outside what the kernels implement */
    KDA_ERR_ALIGNMENT = -3,      /* a tensor pointer is not 16-byte aligned */
    KDA_ERR_WORKSPACE = -4,      /* workspace NULL or smaller than kda_workspace_bytes() */
    KDA_ERR_CUDA = -5,           /* a CUDA runtime call or kernel launch failed */
    KDA_ERR_DEVICE_TIMEOUT = -6  /* a bounded device-side wait gave up (kda_device_status) */
} kda_status;

/* Element type of q, k, v and out. Gates, beta and states are always fp32. */
typedef enum { KDA_BF16 = 0, KDA_F32 = 1 } kda_dtype;

/* Which prefill engine kda_chunk_fwd_engine runs (the value 2 is not used). */
typedef enum {
    KDA_ENGINE_AUTO = 0,     /* cluster tensor-core engine where supported, else the generic one */
    KDA_ENGINE_GENERIC = 1,  /* fp32 CUDA-core chunked engine: any d_k, d_v <= 128, chunk 16/32/64 */
    KDA_ENGINE_TC_CLUSTER = 3 /* tcgen05/TMEM engine, one 4-CTA cluster per (b, h): three
                                CTAs build chunk operands, one runs the state chain;
                                bf16, d_k = d_v = 128, chunk = 64 */
} kda_engine;

/*
 * Bytes of device workspace kda_chunk_fwd needs for this problem (0 when the
 * chosen engine needs none). Returns 0 for unsupported shapes as well; the
 * forward call reports those. The tensor-core engine's workspace is a pool of
 * operand rings behind a 256-byte in-use bitmap, min(B*H, 40) rings of
 * 746,496 bytes (at most 29.9 MiB whatever the batch): each cluster claims a
 * ring when it starts and returns it when it ends, and 40 is more than the
 * clusters a B200 holds at once. The call clears the bitmap itself, so the
 * workspace needs no initialisation.
 */
size_t kda_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int dtype);

/*
 * Chunked prefill over T tokens (Kimi Linear summary, section "Algoritmo
 * paralelo por chunks": fixed-length chunks, each starting from the previous
 * chunk's last state; WY/UT form of the rank-1 updates; lower-triangular
 * inverse by forward substitution; state update in matrix form; output that
 * combines the inter-chunk recurrent part with the intra-chunk parallel part).
 *
 *   q, k       [B,T,H,dk]  dtype        queries and keys
 *   v          [B,T,H,dv]  dtype        values
 *   log_alpha  [B,T,H,dk]  fp32         log of the per-channel forget gate
 *   beta       [B,T,H]     fp32         delta-rule write/erase strength
 *   S0         [B,H,dk,dv] fp32         initial state; NULL means zeros
 *   out        [B,T,H,dv]  dtype        o_t (written)
 *   S_T        [B,H,dk,dv] fp32         final state (written); NULL skips it
 *   chunk      16, 32 or 64             chunk length C; a ragged last chunk is
 *                                       padded with identity steps (exact)
 *   dtype      KDA_BF16 or KDA_F32
 *   workspace, workspace_bytes          device scratch of at least
 *                                       kda_workspace_bytes(...) bytes; may be
 *                                       NULL/0 when that is 0
 *   stream     cudaStream_t as void*
 * S0 and S_T may alias (in-place state update). out must not alias inputs.
 * T = 0 copies S0 (or zeros) to S_T. B = 0 or H = 0 is a no-op.
 * Supported: dk, dv in [1,128] with dv % 4 == 0 (generic engine); the
 * tensor-core engine additionally needs bf16, dk = dv = 128, chunk = 64.
 * Gate range: any log_alpha <= 0. The intra-chunk products carry the decay
 * e^{g_i - g_j} between tokens of a chunk (section "Menor cantidad de
 * operaciones que DPLR general" names the precision problem of fine-grained
 * decay there). The generic engine evaluates every such factor directly. The
 * tensor-core engine splits the chunk into 16-token sub-chunks: blocks between
 * two sub-chunks use factors anchored at the sub-chunk boundary (both <= 1);
 * a diagonal block anchors at its 8th token, and a channel that decays by more
 * than e^-87 inside one sub-chunk takes its diagonal-block factors from
 * log_alpha clamped at -10 per token there (every factor this changes is below
 * e^-10 either way: a change smaller than the tf32 rounding of the factor).
 * Limits: B*T <= 2^31 - 1 tokens and B*H <= 2^29 - 1 heads; larger problems
 * return KDA_ERR_UNSUPPORTED (split the batch).
 */
int kda_chunk_fwd(const void *q, const void *k, const void *v,
                  const float *log_alpha, const float *beta, const float *S0,
                  void *out, float *S_T,
                  int B, int T, int H, int dk, int dv, int chunk, int dtype,
                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * Chunked prefill with the layer's prologue fused into it (Kimi Linear summary,
 * section "Configuracion del modelo Kimi Linear": q and k are L2-normalised,
 * and the per-channel decay comes from a data-dependent gate like GDN's and
 * Mamba's). Computes exactly what kda_chunk_fwd computes on
 *     q / ||q||, k / ||k|| (over the head dimension, per token; a zero row
 *     stays zero) and log_alpha = -softplus(gate) = -log(1 + e^gate),
 * without those tensors ever being written: the prefill reads raw q, k and
 * the gate's pre-activation (bf16, 2 bytes per channel instead of 4 for
 * log_alpha).
 *   q, k       [B,T,H,dk]  bf16         un-normalised queries and keys
 *   v          [B,T,H,dv]  bf16
 *   gate       [B,T,H,dk]  bf16         the gate's pre-activation x
 *   beta, S0, out, S_T, workspace, stream: as kda_chunk_fwd
 * Supported: dtype KDA_BF16, dk = dv = 128, chunk = 64 (the tensor-core
 * engine); anything else returns KDA_ERR_UNSUPPORTED. Limits and T = 0 as
 * kda_chunk_fwd. The workspace is kda_workspace_bytes(...) bytes.
 */
int kda_chunk_fwd_fused(const void *q, const void *k, const void *v, const void *gate,
                        const float *beta, const float *S0, void *out, float *S_T,
                        int B, int T, int H, int dk, int dv, int chunk, int dtype,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * 1 if `engine` (kda_engine) can run a prefill of this shape and dtype, else 0.
 * KDA_ENGINE_AUTO always can when the generic engine can.
 */
int kda_engine_supported(int engine, int dk, int dv, int chunk, int dtype);

/* kda_chunk_fwd with an explicit engine (kda_engine). Same arguments otherwise. */
int kda_chunk_fwd_engine(int engine, const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta, const float *S0,
                         void *out, float *S_T,
                         int B, int T, int H, int dk, int dv, int chunk, int dtype,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * One decode step for N sequences against a state cache, in place (the
 * recurrent form of the same operator; the state is the constant-size cache
 * that replaces a KV cache, Kimi Linear summary, sections "Hibrido 3:1 de KDA
 * y MLA" and "Uso de NoPE y resultados de evaluacion").
 *
 *   q, k       [N,H,dk]    dtype
 *   v          [N,H,dv]    dtype
 *   log_alpha  [N,H,dk]    fp32
 *   beta       [N,H]       fp32
 *   state      [slots,H,dk,dv] fp32     read and updated in place
 *   slot       [N] int32               state row of sequence n; NULL means n.
 *                                       Entries must be distinct and in
 *                                       [0, slots) (not checked: device data)
 *   out        [N,H,dv]    dtype        o = S_new^T q (written)
 * Supported: dk, dv in [1,128], dv % 4 == 0; N*H <= 2^30 - 1 (larger batches
 * return KDA_ERR_UNSUPPORTED).
 */
int kda_recurrent_step(const void *q, const void *k, const void *v,
                       const float *log_alpha, const float *beta,
                       float *state, const int32_t *slot, void *out,
                       int N, int H, int dk, int dv, int dtype, void *stream);

/*
 * Chunked prefill of a packed batch of N sequences of different lengths.
 * Sequence n is tokens cu_seqlens[n] .. cu_seqlens[n+1]-1 of the packed
 * tensors and starts from its own initial state (or zeros); no state crosses a
 * sequence boundary. With a slot map the states live in a state cache of the
 * decode step's layout: a prefill reads and writes row slot[n], and
 * kda_recurrent_step continues from the same rows (the serving path: packed
 * prompts prefill the decode step's cache "without modifying the cache or
 * scheduling interfaces", Kimi Linear summary, section "Uso de NoPE y
 * resultados de evaluacion"). This entry runs the 16-token engine: fp32 state,
 * dense products as warp-level tensor-core tiles in the 3xTF32 form (about fp32
 * accuracy); kda_chunk_fwd_varlen_engine below also runs the tcgen05 engine.
 *
 *   q, k       [total_T,H,dk]  dtype     (packed over sequences)
 *   v          [total_T,H,dv]  dtype
 *   log_alpha  [total_T,H,dk]  fp32
 *   beta       [total_T,H]     fp32
 *   cu_seqlens [N+1]       int32 (device) nondecreasing token offsets, usually
 *                                       cu_seqlens[0] = 0 and cu_seqlens[N] =
 *                                       total_T. Offsets are device data and
 *                                       are not checked; the kernel clamps them
 *                                       to [0, total_T], so no access leaves the
 *                                       tensors. Tokens outside every sequence
 *                                       keep their previous out values.
 *   slot       [N] int32 (device)       state row of sequence n; NULL means n.
 *                                       Entries must be distinct and in
 *                                       [0, slots) (not checked: device data)
 *   S0         [rows,H,dk,dv] fp32      initial states (rows = slots, or N
 *                                       without a slot map); NULL means zeros
 *   out        [total_T,H,dv] dtype     written for every token of a sequence
 *   S_T        [rows,H,dk,dv] fp32      final states; NULL skips them. S_T may
 *                                       be S0 (the state cache, in place)
 * N = 0 or H = 0 is a no-op. Supported: dtype KDA_BF16 or KDA_F32, dk and dv
 * in [1,128], N*H <= 2^29 - 1.
 */
int kda_chunk_fwd_varlen(const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta,
                         const int32_t *cu_seqlens, const int32_t *slot,
                         const float *S0, void *out, float *S_T,
                         int N, int total_T, int H, int dk, int dv, int dtype,
                         void *stream);

/*
 * Device scratch of kda_chunk_fwd_varlen_engine's tensor-core engine for N
 * packed sequences of H heads: the pool of operand rings of kda_workspace_bytes
 * for N*H clusters (one per sequence and head), at most 29.9 MiB, independent of
 * the lengths. 0 when the engine does not support (dk, dv, dtype).
 */
size_t kda_varlen_workspace_bytes(int N, int H, int dk, int dv, int dtype);

/*
 * kda_chunk_fwd_varlen with a choice of engine. Arguments, layouts, results
 * and limits as kda_chunk_fwd_varlen, plus:
 *   engine     KDA_ENGINE_GENERIC: the 16-token engine of kda_chunk_fwd_varlen;
 *              KDA_ENGINE_TC_CLUSTER: the tensor-core engine of kda_chunk_fwd
 *              (bf16, dk = dv = 128, chunk 64), one 4-CTA cluster per
 *              (sequence, head) over the same packed tensors; anything else
 *              returns KDA_ERR_UNSUPPORTED, a missing or small workspace
 *              KDA_ERR_WORKSPACE;
 *              KDA_ENGINE_AUTO: the tensor-core engine when it supports the
 *              shape and the workspace is large enough, else the 16-token one.
 *   workspace  device scratch, 16-byte aligned, kda_varlen_workspace_bytes(...)
 *              bytes (the caller owns it; not kept after the call; one call at
 *              a time per workspace). May be NULL for KDA_ENGINE_GENERIC.
 * Calls with total_T = 0 only move the states and run the 16-token kernel.
 * A bounded device wait that gives up on the tensor-core engine is reported by
 * kda_device_status as KDA_ERR_DEVICE_TIMEOUT, as for kda_chunk_fwd.
 */
int kda_chunk_fwd_varlen_engine(int engine, const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta,
                                const int32_t *cu_seqlens, const int32_t *slot,
                                const float *S0, void *out, float *S_T,
                                int N, int total_T, int H, int dk, int dv, int dtype,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * The KDA layer between its projections, on the tensor-core engine: the fused
 * prologue of kda_chunk_fwd_fused, the recurrence, and the layer's epilogue on
 * every output row (Kimi Linear summary, section "Configuracion del modelo
 * Kimi Linear": per-head RMSNorm and a data-dependent output gate before the
 * output projection; the page gives no formulas). With o the output that
 * kda_chunk_fwd_fused would write, this entry writes instead
 *     out[t][h][c] = o[t][h][c] / sqrt(mean_c'(o[t][h][c']^2) + eps)
 *                    * norm_weight[c] * sigmoid(out_gate[t][h][c]),
 * the mean over the head's dv channels; o itself is never written.
 *   out_gate     [B,T,H,dv] bf16  the output gate's pre-activation
 *   norm_weight  [dv]       fp32  the RMSNorm weight (shared by the heads)
 *   eps          finite, >= 0 (1e-6 is usual)
 *   everything else as kda_chunk_fwd_fused (same support, limits, workspace);
 *   out_gate and norm_weight may be NULL only when T = 0.
 */
int kda_layer_fwd(const void *q, const void *k, const void *v, const void *gate,
                  const float *beta, const void *out_gate, const float *norm_weight, float eps,
                  const float *S0, void *out, float *S_T, int B, int T, int H, int dk, int dv,
                  int chunk, int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * The comparator of KDA's operator efficiency: the chunked forward of the general
 * diagonal-plus-low-rank delta recurrence (Kimi Linear summary, section "Menor
 * cantidad de operaciones que DPLR general": KDA ties both low-rank vectors of the
 * DPLR transition to the key, halving the secondary-chunk products and removing
 * three matrix products, for about twice the operator efficiency; the page gives
 * the claim, not the formula). Per head, with a d_k x d_v fp32 state,
 *     S_t = (Diag(e^{log_alpha_t}) + a_t b_t^T) S_{t-1} + k_t v_t^T,  o_t = S_t^T q_t;
 * KDA is a_t = -beta_t k_t, b_t = e^{log_alpha_t} * k_t with write vector
 * beta_t k_t. Computes in fp32 on CUDA cores with the structure of the fp32 KDA
 * engine (KDA_ENGINE_GENERIC), so that timing both measures the two algorithms.
 *   q, k, a, b [B,T,H,dk] dtype;  v [B,T,H,dv] dtype;  log_alpha [B,T,H,dk] fp32
 *   S0, S_T    [B,H,dk,dv] fp32 (NULL: zeros / skipped);  out [B,T,H,dv] dtype
 * Supported: dtype KDA_BF16 or KDA_F32, dk, dv in [1,128], dv % 4 == 0, chunk 16
 * or 32 (shared memory). Limits as kda_chunk_fwd. Not a product path.
 */
int kda_dplr_chunk_fwd(const void *q, const void *k, const void *v, const void *a,
                       const void *b, const float *log_alpha, const float *S0, void *out,
                       float *S_T, int B, int T, int H, int dk, int dv, int chunk,
                       int dtype, void *stream);

/*
 * The layer's q/k/v prologue ahead of the prefill: ShortConv followed by Swish
 * (Kimi Linear summary, es.news.hada.io/topic?id=31936, section "Configuracion
 * del modelo Kimi Linear": each head's queries, keys and values pass through
 * ShortConv and Swish; the page gives no formula). Read as a causal depthwise
 * convolution along each sequence's tokens with one W-tap filter per (head,
 * channel), no bias:
 *     y[t][h][c] = swish(sum_{j<W} weight[h][c][j] * x[t-j][h][c]),
 *     swish(u) = u / (1 + e^{-u}),
 * where x before a sequence's first token is zero (no value crosses a
 * sequence boundary). Apply it to each of q, k and v (separate filters), then
 * pass q and k un-normalised to kda_chunk_fwd_fused or kda_layer_fwd, which
 * L2-normalise them.
 *   x          [B,T,H,d] dtype, or packed [T,H,d] with cu_seqlens
 *   weight     [H,d,W]   fp32   the filter taps (caller-owned)
 *   cu_seqlens [B+1] int32 (device) or NULL: with it, B sequences packed over
 *              T tokens in all (offsets clamped to [0, T], not checked;
 *              tokens outside every sequence keep their y values); without
 *              it, B rows of T tokens
 *   y          same shape and dtype as x (written), must not alias x
 * Supported: dtype KDA_BF16 or KDA_F32, W in [1,4], d % 8 == 0. All tensors
 * 16-byte aligned (cu_seqlens 4-byte). B, T, H or d = 0 is a no-op.
 */
int kda_short_conv_swish(const void *x, const float *weight, const int32_t *cu_seqlens, void *y,
                         int B, int T, int H, int d, int W, int dtype, void *stream);

/*
 * Backward pass of kda_chunk_fwd: the gradients of a scalar loss L with respect
 * to q, k, v, log_alpha, beta and S0, given dL/d(out) and dL/d(S_T). The pages
 * print no backward pass; this is the derivative of the same recurrence, in
 * the same chunked (WY/UT) form as the prefill, visited last chunk to first.
 *
 *   q, k, v, log_alpha, beta, S0        as kda_chunk_fwd (S0 NULL means zeros)
 *   grad_out   [B,T,H,dv]  dtype        dL/d(out)
 *   grad_S_T   [B,H,dk,dv] fp32         dL/d(S_T); NULL means zeros
 *   grad_q, grad_k [B,T,H,dk] dtype     written
 *   grad_v     [B,T,H,dv]  dtype        written
 *   grad_log_alpha [B,T,H,dk] fp32      written
 *   grad_beta  [B,T,H]     fp32         written
 *   grad_S0    [B,H,dk,dv] fp32         written; NULL skips it
 *   workspace, workspace_bytes          device scratch of at least
 *                                       kda_bwd_workspace_bytes(...) bytes: the
 *                                       entry state of every 16-token chunk plus
 *                                       fp32 accumulators for grad_q and grad_k
 * Outputs must not alias inputs. Computes with fp32 states and accumulation:
 * dense products as warp-level tensor-core tiles in the 3xTF32 form, terms with
 * a pairwise decay on CUDA cores. Sums inside a CTA are in a fixed order; the
 * key-side gradients of the two 64-column value slices meet in fp32 atomics, so
 * grad_q, grad_k, grad_log_alpha and grad_beta may differ in the last bits
 * between runs.
 * T = 0 copies grad_S_T (or zeros) to grad_S0. B = 0 or H = 0 is a no-op.
 * Supported: dtype KDA_BF16 or KDA_F32, dk and dv in [1,128]; the same B*T and
 * B*H limits as kda_chunk_fwd.
 */
int kda_chunk_bwd(const void *q, const void *k, const void *v,
                  const float *log_alpha, const float *beta, const float *S0,
                  const void *grad_out, const float *grad_S_T,
                  void *grad_q, void *grad_k, void *grad_v,
                  float *grad_log_alpha, float *grad_beta, float *grad_S0,
                  int B, int T, int H, int dk, int dv, int dtype,
                  void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes kda_chunk_bwd needs for this shape (0 for empty or unsupported shapes). */
size_t kda_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype);

/*
 * Chunked prefill that allocates nothing and takes no workspace: the same
 * computation as kda_chunk_fwd_engine(KDA_ENGINE_TC_CLUSTER, ...), whose
 * scratch (the ring of per-chunk operand images) lives in a fixed device
 * array of this library. The pages have no counterpart of this call; it exists
 * for callers that cannot allocate device memory at call time, e.g. a serving
 * process whose pool allocator owns all free memory, or a plug-in inside a
 * framework that owns every allocation.
 *   Arguments as kda_chunk_fwd without the workspace; supported: bf16,
 *   dk = dv = 128, chunk = 64, B * T <= 2^31 - 1 tokens and B * H <= 2^29 - 1
 *   heads (larger problems return KDA_ERR_UNSUPPORTED).
 *   Every GPU that loads the library holds the array (29.9 MiB: a pool of 40
 *   operand rings behind an in-use bitmap) until exit. Each 4-CTA cluster (one
 *   sequence and head) claims a ring from the pool when it starts and returns
 *   it when it ends, so any number of heads fits, and calls that overlap on
 *   the GPU (other streams, other threads) claim different rings. The first
 *   call on a device looks up the array's address with that device current
 *   (again after a device reset re-creates the context); make it before any
 *   stream capture. No cudaMalloc, cudaFree or allocating library routine is
 *   called.
 */
int kda_chunk_fwd_static(const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta, const float *S0,
                         void *out, float *S_T,
                         int B, int T, int H, int dk, int dv, int chunk, int dtype,
                         void *stream);

/* Human-readable name of a kda_status code (static string). */
const char *kda_strerror(int code);

/* Detail of the last error returned on the calling host thread (static per thread). */
const char *kda_last_error_detail(void);

/*
 * Synchronises `stream` and reports whether a kernel of this library gave up
 * a bounded device-side wait since the previous call (KDA_ERR_DEVICE_TIMEOUT),
 * clearing the flag; KDA_ERR_CUDA if synchronisation failed; else KDA_OK.
 */
int kda_device_status(void *stream);

/*
 * Test hook for the give-up path of the bounded device-side waits of the
 * tensor-core prefill engine; no counterpart in the pages. Not for production
 * use and not thread-safe: a process-wide setting read at every launch. With
 * on != 0, later launches of that engine use a short wait limit and its first
 * producer CTA withholds the signal that its first chunk's operands are ready,
 * so the state-chain CTA's wait runs out. The launch then gives up without a
 * fault or a trap: every CTA stops issuing copies and MMAs, waits for those in
 * flight, and exits; kda_device_status reports KDA_ERR_DEVICE_TIMEOUT and the
 * outputs of that launch are undefined. on = 0 restores normal launches.
 * Returns the previous setting.
 */
int kda_test_inject_wait_timeout(int on);

/* ABI version of this header: major * 10000 + minor * 100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
