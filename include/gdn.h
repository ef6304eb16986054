/*
 * gdn.h — C ABI of the gated delta rule (Gated DeltaNet) library for NVIDIA B200 (sm_100a).
 *
 * What it computes.  Per value head, a d_v x d_k fp32 state S evolves token by token as
 *
 *      S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,    o_t = scale * S_t q_t
 *
 * ("L'attention hybride", section "La récurrence": alpha_t in ]0,1[ fades the whole state,
 * beta_t in ]0,1[ replaces the association bound to k_t, I is the identity; the equation itself
 * did not survive the page's extraction and is the gated delta rule written with those symbols).
 * Key/query heads are shared by groups of Hv/Hk consecutive value heads (same page, "La
 * dissymétrie 16 / 48": 16 key heads for 48 value heads; 16 for 128 in the "Max" variant): value
 * head h reads key head h / (Hv/Hk).  The state is kept in fp32 whatever the input dtype (same
 * page, "Le float32 n'est pas un détail").
 *
 * Layouts (row-major, last index contiguous, no padding, no strides):
 *   q, k        [B, T, Hk, dk]        dtype given by `dtype`
 *   v           [B, T, Hv, dv]        dtype given by `dtype`
 *   o           [B, T, Hv, dv]        dtype given by `o_dtype` (chunked forward) or `dtype`
 *   log_alpha   [B, T, Hv]  float     alpha = exp(log_alpha), expected in ]0, 1]
 *   beta        [B, T, Hv]  float     expected in [0, 1]
 *   S0, S_T, S  [B, Hv, dk, dv] float, holding S transposed: S_store[b][h][i][j] = S[j][i]
 *               (i over d_k, j over d_v; d_v contiguous)
 *
 * Pointers and ownership.  Every tensor pointer is a DEVICE pointer (cudaMalloc'd or equivalent)
 * on the device current for the calling thread, unless a comment says otherwise.  The caller owns
 * every buffer, including the device scratch ("workspace") that the chunked forward and the layer
 * need: size it with gdn_chunk_fwd_workspace_bytes / gdn_chunk_fwd_varlen_workspace_bytes /
 * gdn_layer_workspace_bytes and pass it in.  No call allocates or frees device memory.  The
 * library keeps no pointer after a call returns.  Its own device memory is part of its device
 * image, loaded with it: a 4-byte error word, and the 32 MiB scratch of gdn_layer_fwd_static.
 * Host-side state: on first use per device the tensor-core chunked forward creates two CUDA
 * streams (high and low priority) and four events and keeps them for the life of the process
 * (see gdn_chunk_fwd).
 * Outputs must not overlap inputs, except S in gdn_decode_step, which is read and written in
 * place.  Tensor pointers (q, k, v, o, z, y, states, raw projections) must be 16-byte aligned,
 * workspaces 256-byte aligned, gate and weight pointers (log_alpha, beta, conv taps, norm gain)
 * 4-byte aligned.
 *
 * Streams.  `stream` is a cudaStream_t (NULL = the legacy default stream).  Each compute call
 * validates its arguments synchronously, enqueues its kernels on `stream` and returns without
 * waiting; results are ready when the stream reaches that point.
 * CUDA graphs.  gdn_chunk_fwd, gdn_decode_step and gdn_layer_fwd can be captured into a CUDA
 * graph (stream capture on `stream`) and replayed, with the results of the eager calls (tested
 * bit for bit); the work the chunked forward forks onto the library's own streams is joined back
 * into `stream` and so captured with it.  Make one eager call of the chunked forward (or of
 * gdn_layer_fwd or gdn_prologue) per device before the first capture: it creates the library's
 * streams and events for the device.  A replay reuses the pointers and sizes of the captured call.
 *
 * Errors.  Calls return gdn_status and never abort, throw or trap.  GDN_ERR_INVALID_ARG: a null
 * required pointer, a non-positive size, Hv not a multiple of Hk, misalignment, or an
 * unsupported enum value, or a missing, misaligned or too small workspace; nothing is enqueued.
 * GDN_ERR_UNSUPPORTED: valid sizes or dtypes the library has no kernel for (dk, dv not in {16, 32,
 * 64, 128}, chunk not in {16, 32, 64}, fp32 inputs with a bf16 output); nothing enqueued.
 * GDN_ERR_CUDA: a CUDA call failed (e.g. the launch); the CUDA error is left for
 * cudaGetLastError.  GDN_ERR_TIMEOUT is reported by gdn_check_error when a kernel gave up on a
 * bounded wait (it then skipped the rest of its work; its outputs are undefined).
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so that this header needs no CUDA include. */
typedef struct CUstream_st *gdn_stream_t;

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1,
  GDN_ERR_UNSUPPORTED = 2,
  GDN_ERR_CUDA = 3,
  GDN_ERR_TIMEOUT = 4
} gdn_status;

/* Storage type of q, k, v, o (and z, y, raw projections).  Gates and states are always fp32. */
typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Kernel family for gdn_chunk_fwd_ex.  AUTO picks TCGEN05 when it supports the call
 * (bf16, dk = dv = 128, chunk = 64), else SIMT. */
typedef enum { GDN_VARIANT_AUTO = 0, GDN_VARIANT_SIMT = 1, GDN_VARIANT_TCGEN05 = 2 } gdn_variant;

/* Static string naming a status (host only, no CUDA call). */
GDN_API const char *gdn_status_string(gdn_status s);

/* Library ABI version (host only): major * 10000 + minor * 100 + patch. */
GDN_API int gdn_version(void);

/* Waits for `stream`, then reads and clears the current device's error word.  Returns
 * GDN_ERR_TIMEOUT if a kernel recorded a timed-out wait since the last check, GDN_ERR_CUDA if
 * the synchronisation failed, else GDN_OK. */
GDN_API gdn_status gdn_check_error(gdn_stream_t stream);

/*
 * Failure-detection self-test (no fault, no hang): enqueues one single-thread kernel that waits,
 * with the same bounded wait the kernels use, on a barrier that nothing completes.  After
 * `budget_cycles` SM clock cycles (1 .. 4e9, about 2 s at most) the wait gives up, the kernel
 * records the timeout bit and returns, so the next gdn_check_error on the stream reports
 * GDN_ERR_TIMEOUT (once: the call clears the bit) and the context stays usable.  This library's
 * own check that a wait which runs out is reported; the pages have no counterpart.
 *   GDN_ERR_INVALID_ARG for a budget out of range (nothing enqueued).
 */
GDN_API gdn_status gdn_wait_timeout_selftest(long long budget_cycles, gdn_stream_t stream);

/*
 * Chunked prefill forward ("Chapitre 16 - Assembler un système de type Kimi K3", 16.2: each block
 * of `chunk` tokens is processed with matrix operations and the state is handed to the next
 * block).  Computes o for all T tokens and the state after token T-1.
 *   S0   may be NULL: the zero state of a fresh request (16.1: the working state is reset for
 *        the next request).  Otherwise the state after the previous call, so that splitting a
 *        sequence over calls gives the same result as one call.
 *   o    [B, T, Hv, dv] in `o_dtype`: GDN_BF16 or GDN_F32 for bf16 inputs, GDN_F32 for fp32
 *        inputs (fp32 inputs with a bf16 o return GDN_ERR_UNSUPPORTED).
 *   S_T  may be NULL when the final state is not wanted.
 *   workspace, workspace_bytes: device scratch of at least
 *        gdn_chunk_fwd_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, dtype) bytes, 256-byte
 *        aligned (NULL and 0 when that size is 0).  Its contents are undefined after the call; it
 *        must not be used by other work until the call's kernels are done on `stream`.
 *   T    need not be a multiple of `chunk`; the ragged last block is masked.
 *   scale multiplies q (o = scale * S q).
 * Exact in real arithmetic for any chunk size; the chunk size only reorders rounding.
 * The tensor-core family (bf16, d_k = d_v = 128, chunk 64) first computes every chunk's
 * state-independent operands in a pre-pass and hands them to the recurrence through the
 * workspace (one record per (batch, value head, chunk); T up to 65535 chunks, 4,194,240 tokens,
 * else GDN_ERR_UNSUPPORTED before any work).  When B * Hv exceeds the device's SM count the
 * call runs in two parts (the last batches first) on two internal streams of the library that
 * fork from and join back into `stream`, so that the recurrence runs in one wave; the results
 * are those of one launch.  A single sequence (B = 1) of at least 256 chunks whose Hv
 * recurrences take at most half of the SMs runs in ranges of 128 chunks on the same two streams
 * (the pre-pass of the next range beside the recurrence of the current one, the state handed on
 * through two fp32 states kept in the workspace); the results are again those of one launch.
 */
GDN_API gdn_status gdn_chunk_fwd(const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta, const float *S0,
                         void *o, float *S_T, void *workspace, size_t workspace_bytes,
                         int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                         float scale, gdn_dtype dtype, gdn_dtype o_dtype,
                         gdn_stream_t stream);

/* Device scratch bytes gdn_chunk_fwd needs for these sizes (host only, no CUDA call): the
 * tensor-core family's operand hand-over, 0 for the CUDA-core family and for empty calls. */
GDN_API size_t gdn_chunk_fwd_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv,
                                     int chunk, gdn_dtype dtype);

/* gdn_chunk_fwd with an explicit kernel family.  GDN_ERR_UNSUPPORTED if the requested family has
 * no kernel for these sizes/dtype.  With GDN_VARIANT_SIMT no workspace is needed. */
GDN_API gdn_status gdn_chunk_fwd_ex(const void *q, const void *k, const void *v,
                            const float *log_alpha, const float *beta, const float *S0,
                            void *o, float *S_T, void *workspace, size_t workspace_bytes,
                            int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                            float scale, gdn_dtype dtype, gdn_dtype o_dtype,
                            gdn_variant variant, gdn_stream_t stream);

/*
 * gdn_chunk_fwd with the gates taken from the in_proj_ba outputs, computed where the pre-pass
 * loads each chunk's gates (so serving from the projections costs no extra pass over HBM):
 * beta = sigmoid(b), log_alpha = log sigmoid(a), the same definitions as gdn_gates ("L'attention
 * hybride", "Le décompte": in_proj_ba makes one beta and one alpha per value head).
 *   ba [B, T, 2*Hv] bf16: the Hv b values, then the Hv a values, of each token (2-byte aligned)
 * Other arguments as gdn_chunk_fwd (same workspace size).  Supported: the tensor-core family
 * (bf16, dk = dv = 128, chunk 64); other sizes return GDN_ERR_UNSUPPORTED.
 */
GDN_API gdn_status gdn_chunk_fwd_ba(const void *q, const void *k, const void *v, const void *ba,
                            const float *S0, void *o, float *S_T, void *workspace,
                            size_t workspace_bytes, int B, int T, int Hk, int Hv, int dk,
                            int dv, int chunk, float scale, gdn_dtype dtype,
                            gdn_dtype o_dtype, gdn_stream_t stream);

/* The family gdn_chunk_fwd would run for these sizes (host only, no CUDA call). */
GDN_API gdn_variant gdn_chunk_fwd_variant(int dk, int dv, int chunk, gdn_dtype dtype);

/* How many kernels one gdn_chunk_fwd_ex call with these arguments launches (the schedule above,
 * decided by the same code the call runs: one for the CUDA-core family; two for the tensor-core
 * family, four when a batched call is split, two per range of a long single sequence; 0 when
 * there is no token).  `sms`: the device's SM count, or 0 to read it from the current device (a
 * CUDA attribute query, nothing enqueued; with sms > 0 no CUDA call is made).  Returns -1 for
 * arguments the call would reject or if the query fails. */
GDN_API int gdn_chunk_fwd_launches(int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                           gdn_dtype dtype, gdn_variant variant, int sms);

/*
 * One decode step for N independent sequences ("Chapitre 16 ...", 16.3: read the fixed state,
 * compute the output, update the state).  q, k [N, Hk, dk]; v [N, Hv, dv] (dtype); o [N, Hv,
 * dv] (o_dtype: GDN_BF16 or GDN_F32 for bf16 inputs, GDN_F32 for fp32 inputs); log_alpha, beta
 * [N, Hv]; S [N, Hv, dk, dv] (S transposed, fp32) is read and overwritten in place with the
 * state after the token.  o_t reads the updated state.
 */
GDN_API gdn_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta, float *S, void *o,
                           int N, int Hk, int Hv, int dk, int dv, float scale,
                           gdn_dtype dtype, gdn_dtype o_dtype, gdn_stream_t stream);

/*
 * One decode step of the whole layer for N sequences, in one kernel: the prologue (causal conv of
 * 4 taps over a carried three-token history, SiLU, L2 normalisation of each q and k head), the
 * recurrence step (state in place) and the gated RMSNorm.  ("Chapitre 16 - Assembler un système
 * de type Kimi K3", 16.3: read the fixed state, compute the output, update the state; "L'attention
 * hybride", "Le décompte": conv kernel 4, swish output gate, one dv-wide norm gain; "Les briques
 * d'un réseau de neurones", 2. SiLU and 4. RMSNorm.)  It equals gdn_layer_fwd run one token at a
 * time with the conv history carried, except that q, k, v stay in fp32 between the prologue and
 * the recurrence (they never leave the chip).
 *   q_raw, k_raw [N, Hk*dk]; v_raw, z [N, Hv*dv]                        (dtype)
 *   hq_in, hk_in [N, 3, Hk*dk]; hv_in [N, 3, Hv*dv]                     (dtype) raw inputs of
 *        the three previous tokens, oldest first (zeros for a fresh request)
 *   hq_out, hk_out, hv_out: same shapes, written with the history after this token.  They must
 *        not overlap the _in buffers (swap the two sets between steps).
 *   wq, wk [Hk*dk, 4]; wv [Hv*dv, 4] float: conv taps, tap 3 on the current token
 *   log_alpha, beta [N, Hv] float; S [N, Hv, dk, dv] float (S transposed per head), in place
 *   norm_w [dv] float; y [N, Hv, dv] (dtype, output)
 *   scale multiplies q; l2_eps is added under the L2 square root, norm_eps under the RMS one.
 * dk, dv in {16, 32, 64, 128}.
 */
GDN_API gdn_status gdn_decode_layer_step(const void *q_raw, const void *k_raw, const void *v_raw,
                                 const void *z, const void *hq_in, const void *hk_in,
                                 const void *hv_in, void *hq_out, void *hk_out, void *hv_out,
                                 const float *wq, const float *wk, const float *wv,
                                 const float *log_alpha, const float *beta, float *S,
                                 const float *norm_w, void *y, int N, int Hk, int Hv, int dk,
                                 int dv, float scale, float l2_eps, float norm_eps,
                                 gdn_dtype dtype, gdn_stream_t stream);

/*
 * Chunked prefill over packed sequences of different lengths: the serving form of gdn_chunk_fwd,
 * many requests in one call, each with its own state ("Chapitre 16 - Assembler un système de type
 * Kimi K3", 16.2: a prompt in blocks with the state handed on; 16.1: the working state belongs to
 * the request).
 *   q, k [total_T, Hk, dk]; v [total_T, Hv, dv] (dtype); o [total_T, Hv, dv] (o_dtype)
 *   log_alpha, beta [total_T, Hv] float
 *   cu_seqlens [nseq + 1] int32 in device memory: sequence s is tokens cu[s] .. cu[s+1] - 1
 *        (cu[0] = 0, non-decreasing, cu[nseq] <= total_T); empty sequences are allowed.  Offsets
 *        outside [0, total_T] are clamped and a sequence longer than max_seqlen is cut there
 *        (tokens outside every sequence keep their o untouched).
 *   max_seqlen: a host-side upper bound of the lengths (it sizes the launch and the workspace)
 *   S0 [nseq, Hv, dk, dv] float or NULL (zero states); S_T [nseq, Hv, dk, dv] float or NULL
 *   workspace, workspace_bytes: at least gdn_chunk_fwd_varlen_workspace_bytes(nseq, max_seqlen,
 *        Hk, Hv, dk, dv, chunk, dtype) bytes, 256-byte aligned, as for gdn_chunk_fwd.
 * Supported: the tensor-core family (bf16 inputs, dk = dv = 128, chunk 64; o bf16 or fp32);
 * other sizes return GDN_ERR_UNSUPPORTED.
 */
GDN_API gdn_status gdn_chunk_fwd_varlen(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta, const int *cu_seqlens,
                                int nseq, int max_seqlen, const float *S0, void *o, float *S_T,
                                void *workspace, size_t workspace_bytes,
                                int total_T, int Hk, int Hv, int dk, int dv, int chunk,
                                float scale, gdn_dtype dtype, gdn_dtype o_dtype,
                                gdn_stream_t stream);

/*
 * Backward pass: gradients of L = sum <dO, o> + <dS_T, S_T>, with o and S_T those of
 * gdn_chunk_fwd on the same inputs, through the exact derivative of the token recurrence
 * ("L'attention hybride", "La récurrence": S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T)
 * + beta_t v_t k_t^T, o_t = scale S_t q_t; the pages give the layer for inference and train their
 * models, so the backward is the chain rule through that recurrence, token by token).
 *   q, k [B, T, Hk, dk]; v, dO [B, T, Hv, dv]            (dtype: GDN_F32 or GDN_BF16)
 *   log_alpha, beta [B, T, Hv] float; S0, dS_T [B, Hv, dk, dv] float holding S^T (either may be
 *        NULL: the zero state / no gradient on S_T)
 *   dq, dk [B, T, Hk, dk] float: summed over the Hv / Hk value heads of each key head
 *   dv [B, T, Hv, dv], dlog_alpha, dbeta [B, T, Hv] float; dS0 [B, Hv, dk, dv] float (nullable)
 *   workspace: gdn_bwd_workspace_bytes(...) bytes, 256-byte aligned, owned by the caller (the
 *        state every 8 tokens of every (batch, value head), and the per-slice partial outputs
 *        summed at the end); NULL is accepted when that size is 0.
 * dk == dv in {16, 32, 64, 128} (else GDN_ERR_UNSUPPORTED).  A CUDA-core kernel with a head's dv
 * columns split over 4 CTAs (d = 128; 2 at d = 64, 1 below): a forward walk keeps the
 * checkpoints, a reverse walk recomputes each state from the nearer of two kept states of its
 * 8-token segment; up to two more launches add the partial dq, dk (over each key head's value
 * heads and the slices) and dlog_alpha, dbeta (over the slices) in a fixed order, so the result
 * is reproducible bit for bit.
 * Pointer alignment: 16 bytes for dv, S0, dS_T, dS0; 4 bytes for the rest.  Errors as
 * gdn_chunk_fwd: GDN_ERR_INVALID_ARG (missing, misaligned, workspace too small) before any work.
 */
GDN_API gdn_status gdn_bwd(const void *q, const void *k, const void *v, const float *log_alpha,
                   const float *beta, const float *S0, const void *dO, const float *dS_T,
                   float *dq, float *dk, float *dv, float *dlog_alpha, float *dbeta, float *dS0,
                   void *workspace, size_t workspace_bytes, int B, int T, int Hk, int Hv,
                   int dk_, int dv_, float scale, gdn_dtype dtype, gdn_stream_t stream);

/*
 * gdn_bwd over packed sequences of different lengths: the training form of gdn_chunk_fwd_varlen,
 * each sequence with its own S0 and its own gradients ("Chapitre 16 - Assembler un système de type
 * Kimi K3", 16.1: the working state belongs to the request; the recurrence differentiated as in
 * gdn_bwd).
 *   q, k [total_T, Hk, dk]; v, dO [total_T, Hv, dv]; log_alpha, beta [total_T, Hv]
 *   cu_seqlens [nseq + 1] int32 (device), max_seqlen: as gdn_chunk_fwd_varlen
 *   S0, dS_T, dS0 [nseq, Hv, dk, dv] (each may be NULL as in gdn_bwd)
 *   dq, dk [total_T, Hk, dk]; dv [total_T, Hv, dv]; dlog_alpha, dbeta [total_T, Hv]
 *   workspace: gdn_bwd_varlen_workspace_bytes(...) bytes, 256-byte aligned.
 * Gradients of tokens outside every sequence are unspecified.  Sizes, dtypes and the
 * reproducibility of the sums as gdn_bwd; each sequence gets the gradients of gdn_bwd on it alone.
 */
GDN_API gdn_status gdn_bwd_varlen(const void *q, const void *k, const void *v,
                          const float *log_alpha, const float *beta, const int *cu_seqlens,
                          int nseq, int max_seqlen, const float *S0, const void *dO,
                          const float *dS_T, float *dq, float *dk, float *dv, float *dlog_alpha,
                          float *dbeta, float *dS0, void *workspace, size_t workspace_bytes,
                          int total_T, int Hk, int Hv, int dk_, int dv_, float scale,
                          gdn_dtype dtype, gdn_stream_t stream);

/* Device scratch bytes gdn_bwd_varlen needs (host only, no CUDA call); 0 for invalid sizes. */
GDN_API size_t gdn_bwd_varlen_workspace_bytes(int nseq, int max_seqlen, int total_T, int Hk,
                                      int Hv, int dk, int dv);

/* Kernels one gdn_bwd call with these sizes launches (host only, no CUDA call): the backward
 * kernel, plus the sums of the partial dq, dk and of dlog_alpha, dbeta where the call has them;
 * -1 for sizes the call rejects. */
GDN_API int gdn_bwd_launches(int B, int T, int Hk, int Hv, int dk, int dv);

/* Device scratch bytes gdn_bwd needs (host only, no CUDA call); 0 for invalid sizes. */
GDN_API size_t gdn_bwd_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv);

/*
 * Backward of the whole layer of gdn_layer_fwd: gradients of <dy, y> + <dS_T, S_T> for every input
 * and weight, by the chain rule through each piece ("L'attention hybride", "Les 48 couches Gated
 * DeltaNet" and "Le décompte": conv kernel 4, swish output gate, one norm gain; "Les briques d'un
 * réseau de neurones", 2. and 4.: SiLU, RMSNorm).  The forward is recomputed inside the call
 * (prologue, then the recurrence with o in fp32); the bf16 rounding of the prologue's q, k, v
 * passes the gradient unchanged.  Then the gated norm's backward (dO in fp32), gdn_bwd's work,
 * and the prologue's: L2 norm (q, k), SiLU, the 4-tap convolution.
 *   inputs as gdn_layer_fwd; dy [B, T, Hv * dv] (dy_dtype: dtype, or GDN_F32 for bf16 inputs);
 *   dS_T [B, Hv, dk, dv] float or NULL
 *   dq_raw, dk_raw [B, T, Hk * dk]; dv_raw, dz [B, T, Hv * dv]; dwq, dwk [Hk * dk, 4];
 *   dwv [Hv * dv, 4]; dlog_alpha, dbeta [B, T, Hv]; dS0 [B, Hv, dk, dv] (nullable); dnorm_w [dv]
 *   (all float outputs)
 *   workspace: gdn_layer_bwd_workspace_bytes(...) bytes, 256-byte aligned, owned by the caller.
 * dk == dv (else GDN_ERR_UNSUPPORTED); other limits as gdn_layer_fwd and gdn_bwd.  Weight
 * gradients are sums of per-CTA partial sums taken in a fixed order (reproducible bit for bit).
 * The sequence starts fresh: the conv sees zeros before token 0, as in gdn_layer_fwd (there is
 * no backward of gdn_layer_fwd_ex's carried history).  Packed sequences: gdn_layer_bwd_varlen.
 */
GDN_API gdn_status gdn_layer_bwd(const void *q_raw, const void *k_raw, const void *v_raw,
                         const void *z, const float *wq, const float *wk, const float *wv,
                         const float *log_alpha, const float *beta, const float *S0,
                         const float *norm_w, const void *dy, const float *dS_T, float *dq_raw,
                         float *dk_raw, float *dv_raw, float *dz, float *dwq, float *dwk,
                         float *dwv, float *dlog_alpha, float *dbeta, float *dS0, float *dnorm_w,
                         void *workspace, size_t workspace_bytes, int B, int T, int Hk, int Hv,
                         int dk, int dv, int chunk, float scale, float l2_eps, float norm_eps,
                         gdn_dtype dtype, gdn_dtype dy_dtype, gdn_stream_t stream);

/* Device scratch bytes gdn_layer_bwd needs (host only, no CUDA call); 0 for invalid sizes. */
GDN_API size_t gdn_layer_bwd_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv,
                                             int chunk, gdn_dtype dtype);

/*
 * gdn_layer_bwd over packed sequences of different lengths: sequence s owns rows cu_seqlens[s] ..
 * cu_seqlens[s + 1] - 1 of every token tensor (total_T rows in all, none longer than max_seqlen),
 * as gdn_layer_fwd_varlen lays them out, and starts fresh (the conv sees zeros before its first
 * token; there is no carried history).  Each sequence's gradients equal gdn_layer_bwd on that
 * sequence alone up to the order of the weight gradients' sums (per-CTA partial sums over the
 * packed tiles, taken in a fixed order).
 *   q_raw, k_raw [total_T, Hk * dk]; v_raw, z [total_T, Hv * dv]; dy [total_T, Hv * dv] (dy_dtype)
 *   log_alpha, beta [total_T, Hv]; S0, dS_T, dS0 [nseq, Hv, dk, dv] (nullable)
 *   dq_raw, dk_raw [total_T, Hk * dk]; dv_raw, dz [total_T, Hv * dv]; dlog_alpha, dbeta
 *   [total_T, Hv]; dwq, dwk [Hk * dk, 4]; dwv [Hv * dv, 4]; dnorm_w [dv] (float outputs)
 *   workspace: gdn_layer_bwd_varlen_workspace_bytes(...) bytes, 256-byte aligned, caller-owned.
 * The tensor-core shape only (bf16 inputs, dk = dv = 128, chunk 64; else GDN_ERR_UNSUPPORTED).
 * Rows in no sequence (past cu_seqlens[nseq], or cut off by max_seqlen) add nothing to the
 * weight gradients and get dz = 0; their other gradients are unspecified.  An empty sequence hands
 * dS_T on as dS0; when every sequence is empty the weight gradients are zeros.
 */
GDN_API gdn_status gdn_layer_bwd_varlen(const void *q_raw, const void *k_raw, const void *v_raw,
                         const void *z, const int *cu_seqlens, int nseq, int max_seqlen,
                         const float *wq, const float *wk, const float *wv,
                         const float *log_alpha, const float *beta, const float *S0,
                         const float *norm_w, const void *dy, const float *dS_T, float *dq_raw,
                         float *dk_raw, float *dv_raw, float *dz, float *dwq, float *dwk,
                         float *dwv, float *dlog_alpha, float *dbeta, float *dS0, float *dnorm_w,
                         void *workspace, size_t workspace_bytes, int total_T, int Hk, int Hv,
                         int dk, int dv, int chunk, float scale, float l2_eps, float norm_eps,
                         gdn_dtype dtype, gdn_dtype dy_dtype, gdn_stream_t stream);

/* Device scratch bytes gdn_layer_bwd_varlen needs (host only, no CUDA call); 0 for invalid
 * sizes. */
GDN_API size_t gdn_layer_bwd_varlen_workspace_bytes(int nseq, int max_seqlen, int total_T, int Hk,
                                                    int Hv, int dk, int dv, int chunk,
                                                    gdn_dtype dtype);

/*
 * Backward of gdn_gates: dba [rows, 2*Hv] float, the b gradients dbeta beta (1 - beta) then the a
 * gradients dlog_alpha sigmoid(-a) (d/da of log sigmoid(a)).  ba as gdn_gates (dtype).
 */
GDN_API gdn_status gdn_gates_bwd(const void *ba, const float *dlog_alpha, const float *dbeta,
                         float *dba, long long rows, int Hv, gdn_dtype dtype, gdn_stream_t stream);

/* Device scratch bytes gdn_chunk_fwd_varlen needs (host only, no CUDA call). */
GDN_API size_t gdn_chunk_fwd_varlen_workspace_bytes(int nseq, int max_seqlen, int Hk, int Hv,
                                            int dk, int dv, int chunk, gdn_dtype dtype);

/*
 * Gates from the in_proj_ba outputs, per (token, value head): beta = sigmoid(b) and
 * log_alpha = log sigmoid(a) = -softplus(-a).  ("L'attention hybride", "Le décompte": in_proj_ba
 * makes one beta and one alpha per value head and the layer counts no other gate parameter;
 * "La récurrence": alpha, beta in ]0,1[; "Les briques d'un réseau de neurones", 2.: the sigmoid
 * is the gate, softplus is log(1 + e^x).  The pages give no other parameterisation of alpha;
 * this is the plainest one that fits them.)
 *   ba [rows, 2*Hv] (dtype): the Hv b values, then the Hv a values, of each token
 *   log_alpha, beta [rows, Hv] float (outputs, the gates gdn_chunk_fwd and gdn_layer_fwd take)
 */
GDN_API gdn_status gdn_gates(const void *ba, float *log_alpha, float *beta, long long rows, int Hv,
                     gdn_dtype dtype, gdn_stream_t stream);

/*
 * Layer prologue: causal depthwise convolution with 4 taps and no bias, then SiLU, on the q, k
 * and v channels; then each q and k head is divided by sqrt(sum of squares + l2_eps).
 * ("L'attention hybride", "Le décompte": conv kernel 4 over the q, k, v channels, 4 weights per
 * channel; "Les briques d'un réseau de neurones", 2.: SiLU(x) = x sigmoid(x).)
 *   q_raw, k_raw [B, T, Hk*dk]; v_raw [B, T, Hv*dv]         (dtype)
 *   wq, wk [Hk*dk, 4]; wv [Hv*dv, 4] float: tap 3 multiplies the current token, tap 0 the token
 *        three steps back; positions before t = 0 are zeros (gdn_prologue_ex carries the
 *        previous tokens instead).
 *   q, k [B, T, Hk, dk]; v [B, T, Hv, dv]                    (dtype, outputs)
 * bf16 outputs are the exact results rounded to the nearest bf16 (ties to even): a value whose
 * rounding the fp32 computation cannot decide within its error bound is recomputed in fp64, so
 * the rounding never depends on fp32 roundoff.  Two kernels: the q and k heads run on the
 * library's high-priority stream of the device (forked from and joined back into `stream`), the
 * v heads on `stream`, so that both share the SMs; `stream` waits for both.
 */
GDN_API gdn_status gdn_prologue(const void *q_raw, const void *k_raw, const void *v_raw,
                        const float *wq, const float *wk, const float *wv,
                        void *q, void *k, void *v,
                        int B, int T, int Hk, int Hv, int dk, int dv, float l2_eps,
                        gdn_dtype dtype, gdn_stream_t stream);

/*
 * gdn_prologue continuing a sequence: the convolution at tokens 0, 1, 2 reads the raw inputs of
 * the three tokens before the call from a carried history instead of zeros, so that a sequence
 * run in pieces gets the outputs of one run ("Chapitre 16 - Assembler un système de type Kimi
 * K3", 16.2: prefill in blocks, the state handed from block to block; the conv's three inputs are
 * part of that state, as in gdn_decode_layer_step).
 *   hq_in, hk_in [B, 3, Hk*dk]; hv_in [B, 3, Hv*dv] (dtype, 16-byte aligned): the raw inputs of
 *        the three previous tokens, oldest first; NULL means zeros (a fresh sequence).
 * Everything else as gdn_prologue.
 */
GDN_API gdn_status gdn_prologue_ex(const void *q_raw, const void *k_raw, const void *v_raw,
                           const void *hq_in, const void *hk_in, const void *hv_in,
                           const float *wq, const float *wk, const float *wv,
                           void *q, void *k, void *v,
                           int B, int T, int Hk, int Hv, int dk, int dv, float l2_eps,
                           gdn_dtype dtype, gdn_stream_t stream);

/*
 * Output gate: y = o / sqrt(mean(o^2) + eps) * w (.) SiLU(z) for each row of dv values
 * ("L'attention hybride": swish output gate and one normalisation gain of 128 shared by all
 * heads; "Les briques d'un réseau de neurones", 4.: RMSNorm).
 *   o, z, y [rows, dv] (dtype); w [dv] float.
 */
GDN_API gdn_status gdn_out_norm(const void *o, const void *z, const float *w, void *y,
                        long long rows, int dv, float eps, gdn_dtype dtype,
                        gdn_stream_t stream);

/*
 * Whole layer between the projections: gdn_prologue -> gdn_chunk_fwd -> gdn_out_norm.
 *   q_raw, k_raw [B, T, Hk*dk]; v_raw, z [B, T, Hv*dv] (dtype); wq, wk, wv conv taps as in
 *   gdn_prologue; log_alpha, beta [B, T, Hv]; S0 nullable; norm_w [dv];
 *   y [B, T, Hv, dv] (y_dtype, output: GDN_BF16 or GDN_F32 for bf16 inputs, GDN_F32 for fp32
 *   inputs); S_T nullable (output).
 *   workspace: device scratch of at least gdn_layer_workspace_bytes(...) bytes, 256-byte
 *   aligned, or NULL when that size is 0.  Its contents are undefined after the call.
 */
GDN_API gdn_status gdn_layer_fwd(const void *q_raw, const void *k_raw, const void *v_raw,
                         const void *z, const float *wq, const float *wk, const float *wv,
                         const float *log_alpha, const float *beta, const float *S0,
                         const float *norm_w, void *y, float *S_T,
                         void *workspace, size_t workspace_bytes,
                         int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                         float scale, float l2_eps, float norm_eps,
                         gdn_dtype dtype, gdn_dtype y_dtype, gdn_stream_t stream);

/*
 * gdn_layer_fwd continuing a sequence (prefill in pieces, or prefill followed by
 * gdn_decode_layer_step): the conv reads a carried history of the three previous tokens' raw
 * inputs, and the history after the call can be written out.  Run in pieces, with S0 = the
 * previous piece's S_T and the history passed on, a sequence gets the outputs of one run (bit for
 * bit when each piece but the last is a multiple of `chunk` tokens long; otherwise the pieces'
 * chunk boundaries differ and the results differ by rounding).  ("Chapitre 16 - Assembler un
 * système de type Kimi K3", 16.2 and 16.3: the state handed from block to block, then read and
 * updated by decode; the conv's inputs are part of it.)
 *   hq_in, hk_in [B, 3, Hk*dk]; hv_in [B, 3, Hv*dv] (dtype): raw inputs of the three tokens
 *        before the call, oldest first; NULL means zeros (a fresh sequence).
 *   hq_out, hk_out, hv_out: same shapes (dtype), written with the raw inputs of the last three
 *        tokens of [history; this call's tokens], the history gdn_decode_layer_step or the next
 *        piece takes; NULL skips it.  They must not overlap the _in buffers or any input.
 * History pointers are 16-byte aligned.  Everything else as gdn_layer_fwd (same workspace size).
 */
GDN_API gdn_status gdn_layer_fwd_ex(const void *q_raw, const void *k_raw, const void *v_raw,
                            const void *z, const void *hq_in, const void *hk_in,
                            const void *hv_in, const float *wq, const float *wk, const float *wv,
                            const float *log_alpha, const float *beta, const float *S0,
                            const float *norm_w, void *y, float *S_T, void *hq_out,
                            void *hk_out, void *hv_out, void *workspace, size_t workspace_bytes,
                            int B, int T, int Hk, int Hv, int dk, int dv, int chunk, float scale,
                            float l2_eps, float norm_eps, gdn_dtype dtype, gdn_dtype y_dtype,
                            gdn_stream_t stream);

/*
 * The whole layer over packed requests of different lengths: the serving form of
 * gdn_layer_fwd_ex, many requests in one call, each with its own state and conv history
 * ("Chapitre 16 - Assembler un système de type Kimi K3", 16.1-16.2: the working state belongs
 * to the request; a prompt in blocks with the state handed on).
 *   q_raw, k_raw [total_T, Hk*dk]; v_raw, z [total_T, Hv*dv] (dtype); y [total_T, Hv, dv]
 *        (y_dtype); log_alpha, beta [total_T, Hv] float
 *   cu_seqlens [nseq + 1] int32 in device memory, max_seqlen: as gdn_chunk_fwd_varlen (request s
 *        is tokens cu[s] .. cu[s+1] - 1; empty requests allowed; offsets clamped); the conv of a
 *        request never reads another request's tokens.
 *   hq_in, hk_in [nseq, 3, Hk*dk]; hv_in [nseq, 3, Hv*dv] (dtype) or NULL (fresh requests);
 *        hq_out, hk_out, hv_out: same shapes or NULL, as gdn_layer_fwd_ex, per request
 *   S0, S_T [nseq, Hv, dk, dv] float, each may be NULL (zero states / not written)
 *   workspace: gdn_layer_fwd_varlen_workspace_bytes(...) bytes, 256-byte aligned.
 * y of tokens outside every request is unspecified.  Supported: bf16 inputs, dk = dv = 128,
 * chunk 64 (y bf16 or fp32); other sizes return GDN_ERR_UNSUPPORTED.  Each request gets the
 * results of gdn_layer_fwd_ex on it alone.
 */
GDN_API gdn_status gdn_layer_fwd_varlen(const void *q_raw, const void *k_raw, const void *v_raw,
                                const void *z, const int *cu_seqlens, int nseq, int max_seqlen,
                                const void *hq_in, const void *hk_in, const void *hv_in,
                                const float *wq, const float *wk, const float *wv,
                                const float *log_alpha, const float *beta, const float *S0,
                                const float *norm_w, void *y, float *S_T, void *hq_out,
                                void *hk_out, void *hv_out, void *workspace,
                                size_t workspace_bytes, int total_T, int Hk, int Hv, int dk,
                                int dv, int chunk, float scale, float l2_eps, float norm_eps,
                                gdn_dtype dtype, gdn_dtype y_dtype, gdn_stream_t stream);

/* Device scratch bytes gdn_layer_fwd_varlen needs (host only, no CUDA call); 0 for sizes it does
 * not support. */
GDN_API size_t gdn_layer_fwd_varlen_workspace_bytes(int nseq, int max_seqlen, int total_T,
                                            int Hk, int Hv, int dk, int dv, int chunk,
                                            gdn_dtype dtype);

/* Scratch bytes gdn_layer_fwd needs for these sizes (host only, no CUDA call); 0 if none. */
GDN_API size_t gdn_layer_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                                 gdn_dtype dtype);

/* Size of the device scratch that the library carries for gdn_layer_fwd_static: 32 MiB. */
#define GDN_LAYER_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* gdn_layer_fwd_static: the same layer as gdn_layer_fwd, for callers that cannot hand it a
 * workspace.  A program that has no device allocator of its own (plain C linking only this
 * library), or one that must not allocate device memory while it runs the layer (an allocation
 * can synchronise the device and stall other streams), calls this instead: it allocates and frees
 * nothing.  The pages describe no such call; it belongs to this library only.
 *
 *   Arguments, layouts, results and errors are those of gdn_layer_fwd without `workspace` and
 *   `workspace_bytes`.  The scratch is GDN_LAYER_STATIC_SCRATCH_BYTES of device memory built into
 *   the library (one per device); sizes for which gdn_layer_workspace_bytes(...) exceeds it return
 *   GDN_ERR_UNSUPPORTED before any work (about 380 tokens at Hk=16, Hv=48, d=128, bf16).
 *   The first call on a device looks the scratch's device address up (cudaGetSymbolAddress on
 *   the current device, which must be the device of every pointer and of `stream`) and keeps it;
 *   that lookup allocates nothing, but make the first call on each device before any stream
 *   capture starts.  Nothing in the scratch needs to start at zero.
 *   All calls on one device share the one scratch: two calls whose GPU work can overlap (on
 *   streams not ordered with each other) race on it and give wrong results.  Order them.
 */
GDN_API gdn_status gdn_layer_fwd_static(const void *q_raw, const void *k_raw, const void *v_raw,
                         const void *z, const float *wq, const float *wk, const float *wv,
                         const float *log_alpha, const float *beta, const float *S0,
                         const float *norm_w, void *y, float *S_T,
                         int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                         float scale, float l2_eps, float norm_eps,
                         gdn_dtype dtype, gdn_dtype y_dtype, gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
