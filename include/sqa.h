/*
 * sqa.h - C ABI of the Sparse Query Attention hot path for NVIDIA B200 (sm_100a).
 *
 * Sparse Query Attention keeps the key/value sharing of Grouped Query
 * Attention but lowers the number of *query* heads: H_q query heads attend,
 * and each of the H_kv key/value heads is shared by G = H_q / H_kv
 * consecutive query heads (query head h reads key/value head h / G).  Score
 * and context FLOPs therefore scale with H_q instead of the full head count H.
 *   - "ReactiveAI/GQA-Ref-Micro" model card, introduction (SQA as an
 *     extension of GQA that reduces query heads);
 *   - "Sparse Query Attention (SQA): A Computationally Efficient Attention
 *     Mechanism with Query Heads Reduction", abstract (FLOPs fall in
 *     proportion to the query-head reduction; pre-training, fine-tuning and
 *     encoder workloads; 32k-200k token sequences);
 *   - "ReactiveAI/xSMQAT-m" model card, note on model size (query and output
 *     projections shrink to width H_q * d_head).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The
 *    library allocates no device memory and keeps no per-call state; on the
 *    host it caches driver entry points and, per device, kernel and cluster
 *    size, how many thread-block clusters run at once (queried once).
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL means the legacy default stream).  Nothing synchronises except
 *    sqa_device_status().  Kernels are launched as programmatic dependents
 *    of the previous kernel on the stream: they may start their set-up
 *    while it finishes but touch no global memory before the kernels of
 *    earlier calls have completed, so stream order holds for every buffer,
 *    as with ordinary launches.  (Inside one call, a kernel that reads
 *    nothing its predecessor writes, dQ after dK/dV or the second of two
 *    forward launches over one problem, starts its work early and waits
 *    for that predecessor before it exits.)
 *  - Layouts are dense, row-major, with the last index contiguous:
 *      Q, O, dO, dQ : [B, N, H_q,  d_head]
 *      K, V, dK, dV : [B, N, H_kv, d_head]
 *      LSE          : [B, H_q, N]  (fp32, natural log of the softmax sum)
 *    so O viewed as [B*N, H_q*d_head] is the input of the output projection.
 *  - Tensor pointers must be 16-byte aligned.
 *  - Invalid arguments return SQA_ERR_INVALID_ARG and launch nothing; shapes
 *    the kernels do not handle return SQA_ERR_UNSUPPORTED; a failed launch
 *    returns SQA_ERR_CUDA.
 *  - Device-side waits are bounded.  A wait that runs out records
 *    SQA_ERR_TIMEOUT in a device status word (the kernel then winds down and
 *    returns); sqa_device_status() reports and clears it.
 */
#ifndef SQA_H_
#define SQA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQA_OK = 0,
  SQA_ERR_INVALID_ARG = 1,
  SQA_ERR_UNSUPPORTED = 2,
  SQA_ERR_CUDA = 3,
  SQA_ERR_TIMEOUT = 4
} sqa_status_t;

typedef enum { SQA_DT_F32 = 0, SQA_DT_BF16 = 1 } sqa_dtype_t;

/*
 * sqa_attn_fwd - attention core forward, fp32 output.
 *   O[b,t,h,:] = sum_u softmax_u(scale * <Q[b,t,h,:], K[b,u,j,:]>) V[b,u,j,:],
 *   j = h / (H_q / H_kv); with causal != 0 only keys u <= t take part.
 * q, k, v : bf16, layouts above.   out : fp32 [B, N, H_q * d_head].
 * Requirements: B, N >= 1; 1 <= H_kv <= H_q; H_q % H_kv == 0;
 * d_head in {16, 32, 64, 128} (else SQA_ERR_UNSUPPORTED); scale finite.
 */
sqa_status_t sqa_attn_fwd(const void* q, const void* k, const void* v, void* out,
                          int B, int N, int H_q, int H_kv, int d_head, int causal,
                          float scale, void* stream);

/*
 * sqa_attn_fwd_ex - as sqa_attn_fwd, with the output dtype chosen by
 * out_dtype (SQA_DT_F32 or SQA_DT_BF16) and, when lse != NULL, the
 * per-row log-sum-exp of the scaled scores written to lse [B, H_q, N] fp32
 * (natural log; what sqa_attn_bwd needs).
 */
sqa_status_t sqa_attn_fwd_ex(const void* q, const void* k, const void* v, void* out,
                             sqa_dtype_t out_dtype, float* lse,
                             int B, int N, int H_q, int H_kv, int d_head, int causal,
                             float scale, void* stream);

/*
 * sqa_attn_bwd_workspace_size - bytes of device workspace sqa_attn_bwd needs
 * for this shape (the per-row dot products D = rowsum(dO * O), fp32).
 * Returns 0 for invalid shapes.
 */
size_t sqa_attn_bwd_workspace_size(int B, int N, int H_q, int H_kv, int d_head);

/*
 * sqa_attn_bwd - gradient of the attention core (the training step the
 * pages' throughput claims are about).
 * Inputs : q, k, v (bf16), out = the forward output O (dtype o_dtype),
 *          dout = dL/dO (bf16, [B,N,H_q,d_head]),
 *          lse  = the forward's log-sum-exp [B,H_q,N] fp32.
 * Outputs: dq [B,N,H_q,d], dk and dv [B,N,H_kv,d] in grad_dtype (F32 or
 *          BF16).  dk and dv of key/value head j are summed over the G query
 *          heads of group j.  All three are fully overwritten.
 * workspace: device buffer of at least sqa_attn_bwd_workspace_size() bytes,
 *          owned by the caller, 16-byte aligned; contents on entry ignored.
 */
sqa_status_t sqa_attn_bwd(const void* q, const void* k, const void* v,
                          const void* out, sqa_dtype_t o_dtype,
                          const void* dout, const float* lse,
                          void* dq, void* dk, void* dv, sqa_dtype_t grad_dtype,
                          int B, int N, int H_q, int H_kv, int d_head, int causal,
                          float scale, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * sqa_attn_fwd_cross - cross / memory attention: N_q query tokens attend,
 * without a mask, to N_kv key/value tokens of another sequence (a memory
 * state, an encoder's output).  "ReactiveAI/GQA-Ref-Micro" model card,
 * closing outlook: the Reactive Transformer's memory attention, designed with
 * shared key/value heads, is to take SQA variants as well; "Sparse Query
 * Attention ...", "Built on by" (Reactive Transformer).
 * Layouts: q, out [B, N_q, H_q, d_head]; k, v [B, N_kv, H_kv, d_head] bf16;
 *   lse [B, H_q, N_q] fp32 or NULL.
 * Otherwise as sqa_attn_fwd_ex with causal = 0: N_q, N_kv >= 1, any pair
 * (N_kv may be shorter or longer than N_q).  sqa_attn_fwd_ex(..., N, ...)
 * equals sqa_attn_fwd_cross(..., N_q = N, N_kv = N, ...) non-causal.
 * Unmasked problems with few query tiles (d_head = 128) may run as clusters
 * of CTAs that split the key range and merge their partial rows in a fixed
 * order: the result does not change from run to run.
 */
sqa_status_t sqa_attn_fwd_cross(const void* q, const void* k, const void* v, void* out,
                                sqa_dtype_t out_dtype, float* lse,
                                int B, int N_q, int N_kv, int H_q, int H_kv, int d_head,
                                float scale, void* stream);

/*
 * sqa_attn_bwd_cross - gradient of sqa_attn_fwd_cross.  Arguments as
 * sqa_attn_bwd with causal = 0 and the two lengths apart: q, out, dout, dq
 * [B, N_q, H_q, d]; k, v, dk, dv [B, N_kv, H_kv, d]; lse [B, H_q, N_q].
 * The workspace is sqa_attn_bwd_workspace_size(B, N_q, H_q, H_kv, d_head)
 * bytes (it holds per-query-row values only).  Unmasked problems with few key
 * tiles (dK/dV) or few query tiles (dQ) may run as clusters of CTAs that
 * split the other sequence and sum their partial gradients in a fixed order:
 * the gradients do not change from run to run, and no workspace is added.
 */
sqa_status_t sqa_attn_bwd_cross(const void* q, const void* k, const void* v,
                                const void* out, sqa_dtype_t o_dtype,
                                const void* dout, const float* lse,
                                void* dq, void* dk, void* dv, sqa_dtype_t grad_dtype,
                                int B, int N_q, int N_kv, int H_q, int H_kv, int d_head,
                                float scale, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * sqa_attn_fwd_window - sliding-window (local) SQA: query t attends only to
 * the keys u with t - window_left <= u <= t + window_right (and u < N).
 * Spatially sparse attention of this kind is what the GQA-Ref-Micro model
 * card (results paragraph) sets SQA beside; the paper's "Builds on" list
 * includes Longformer.  The query-head reduction and the band combine: the
 * cost is 4 * B * H_q * P_w * d FLOPs, P_w = number of visible (t, u) pairs.
 * Common forms: a causal window of W keys is (W - 1, 0); a symmetric local
 * window is (w, w).  A side of N or more is unbounded, so (N, 0) is the
 * causal mask and (N, N) no mask.  Key tiles outside every row's band are
 * skipped, not masked.
 * Self-attention only (K/V have N tokens); window_left, window_right >= 0
 * (else SQA_ERR_INVALID_ARG).  Layouts, dtypes and lse as sqa_attn_fwd_ex.
 */
sqa_status_t sqa_attn_fwd_window(const void* q, const void* k, const void* v, void* out,
                                 sqa_dtype_t out_dtype, float* lse,
                                 int B, int N, int H_q, int H_kv, int d_head,
                                 int window_left, int window_right, float scale, void* stream);

/*
 * sqa_attn_bwd_window - gradient of sqa_attn_fwd_window (same window);
 * arguments otherwise as sqa_attn_bwd, workspace from
 * sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d_head).
 */
sqa_status_t sqa_attn_bwd_window(const void* q, const void* k, const void* v,
                                 const void* out, sqa_dtype_t o_dtype,
                                 const void* dout, const float* lse,
                                 void* dq, void* dk, void* dv, sqa_dtype_t grad_dtype,
                                 int B, int N, int H_q, int H_kv, int d_head,
                                 int window_left, int window_right, float scale,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * sqa_attn_decode - decoding against a key/value cache.  Autoregressive
 * inference is the memory-bound regime ("Sparse Query Attention (SQA): ...",
 * abstract: its latency is bound by memory bandwidth, which MQA/GQA address
 * by sharing K/V): each step streams the cache once, so SQA's fewer query
 * heads cut arithmetic but not bytes; the kernel is built to stream the cache
 * at HBM speed.
 * Inputs : q [B, n_new, H_q, d_head] bf16, the queries of the last n_new
 *          tokens of each sequence;
 *          k_cache, v_cache [B, L_max, H_kv, d_head] bf16, of which the first
 *          cache_lens[b] tokens of sequence b are valid, the new tokens' own
 *          keys/values included; entries past cache_lens[b] are never read;
 *          cache_lens: DEVICE int32 [B], n_new <= cache_lens[b] <= L_max.
 * Outputs: out [B, n_new, H_q, d_head] (out_dtype), lse [B, H_q, n_new] fp32
 *          (natural log) or NULL.  Token i of sequence b sits at position
 *          cache_lens[b] - n_new + i and sees keys 0 .. that position.
 * workspace: sqa_attn_decode_workspace_size() bytes (0 when the cache is
 *          processed as one chunk per sequence; workspace may then be NULL).
 * Requirements: g * n_new <= 128 where g is the largest power of two dividing
 * H_q / H_kv (else SQA_ERR_UNSUPPORTED); other rules as sqa_attn_fwd.  A
 * cache length outside [n_new, L_max] cannot be checked on the host: the
 * kernel clamps it into range and sqa_device_status() then reports
 * SQA_ERR_INVALID_ARG.
 */
size_t sqa_attn_decode_workspace_size(int B, int n_new, int H_q, int H_kv, int d_head, int L_max);

sqa_status_t sqa_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                             const int* cache_lens, void* out, sqa_dtype_t out_dtype, float* lse,
                             int B, int n_new, int H_q, int H_kv, int d_head, int L_max,
                             float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * sqa_attn_fwd_packed - the forward on a packed QKV buffer, the output of one
 * fused input projection with the concatenated weight [Wq; Wk; Wv]
 * ((H_q + 2 H_kv) * d_head rows): qkv [B, N, H_q + 2 H_kv, d_head] bf16,
 * holding per token the H_q query heads, then the H_kv key heads, then the
 * H_kv value heads.  SQA narrows exactly this projection (query and output
 * projections of width H_q * d_head: "ReactiveAI/xSMQAT-m" model card, note
 * on model size), so one GEMM produces all three operands.
 * out [B, N, H_q, d_head] (out_dtype) and lse [B, H_q, N] (or NULL) are
 * dense, as in sqa_attn_fwd_ex; every other argument and rule as there.
 * The result equals sqa_attn_fwd_ex on the three heads' slices copied out.
 */
sqa_status_t sqa_attn_fwd_packed(const void* qkv, void* out, sqa_dtype_t out_dtype, float* lse,
                                 int B, int N, int H_q, int H_kv, int d_head, int causal,
                                 float scale, void* stream);

/*
 * sqa_attn_bwd_packed - gradient of sqa_attn_fwd_packed: dqkv
 * [B, N, H_q + 2 H_kv, d_head] in grad_dtype, laid out as qkv (dQ heads,
 * then dK, then dV), so the input projection's backward is one GEMM for dX
 * and one for the concatenated weight gradient.  out, dout [B, N, H_q, d]
 * and lse [B, H_q, N] are dense; workspace as sqa_attn_bwd.  Every entry of
 * dqkv is overwritten.
 */
sqa_status_t sqa_attn_bwd_packed(const void* qkv, const void* out, sqa_dtype_t o_dtype,
                                 const void* dout, const float* lse,
                                 void* dqkv, sqa_dtype_t grad_dtype,
                                 int B, int N, int H_q, int H_kv, int d_head, int causal,
                                 float scale, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * sqa_attn_bwd_static - sqa_attn_bwd without a caller-supplied workspace.
 * (Library plumbing; the paper has no counterpart.)
 *
 * For callers that cannot allocate device memory themselves: code handed
 * only input and output pointers by a host framework that owns the GPU's
 * memory (a plugin or custom-op interface), or services that forbid any
 * allocation once they are running.  The scratch the backward needs (the
 * per-row D and LSE*log2(e) values) lives instead in one fixed device array
 * inside this library, SQA_BWD_STATIC_SCRATCH_BYTES in size, which every GPU
 * that loads the library holds until the process exits.
 *
 * Arguments, layouts and results are those of sqa_attn_bwd.  The call
 * allocates nothing (no cudaMalloc/cudaFree, no allocating library routine).
 * Shapes whose workspace (sqa_attn_bwd_workspace_size) exceeds
 * SQA_BWD_STATIC_SCRATCH_BYTES return SQA_ERR_UNSUPPORTED and launch nothing.
 * The first call on a device looks up the array's device address (with that
 * device current); make that first call before any stream capture.  The
 * address belongs to the device's context: after a cudaDeviceReset the next
 * call finds a new context and looks the address up again (so, again, not
 * inside a stream capture).  All
 * calls share the one array: calls that overlap on the GPU (different
 * streams, or different host threads, on the same device) race on it, so
 * serialise them.  The array keeps the previous call's contents; the
 * backward overwrites every entry it reads, so nothing needs clearing.
 */
#define SQA_BWD_STATIC_SCRATCH_BYTES (16u << 20)

sqa_status_t sqa_attn_bwd_static(const void* q, const void* k, const void* v,
                                 const void* out, sqa_dtype_t o_dtype,
                                 const void* dout, const float* lse,
                                 void* dq, void* dk, void* dv, sqa_dtype_t grad_dtype,
                                 int B, int N, int H_q, int H_kv, int d_head, int causal,
                                 float scale, void* stream);

/*
 * sqa_proj - one reduced-width projection, Y[M, Nout] = X[M, K] W[Nout, K]^T
 * (+ bias), the Q/K/V projections (Nout = H_q*d_head or H_kv*d_head) and the
 * output projection (K = H_q*d_head).  X and W are bf16 (W in nn.Linear
 * layout); bias is NULL or fp32 [Nout]; Y is y_dtype (F32 or BF16).
 * Requirements: M, K, Nout >= 1; K % 16 == 0; Nout % 16 == 0.
 */
sqa_status_t sqa_proj(const void* x, const void* w, const float* bias, void* y,
                      sqa_dtype_t y_dtype, int M, int K, int Nout, void* stream);

/*
 * sqa_gemm - the general projection contraction, used for the backward of
 * the projections of an SQA layer (dX = dY W, dW = dY^T X) as well as the
 * forward sqa_proj is a special case of:
 *     C[M, N] (+)= sum_k A(m, k) B(n, k)  (+ bias[n])
 * Operands are read as stored, no transpose through memory:
 *   A(m, k) = a[m * K + k]  (SQA_K_CONTIGUOUS)  or  a[k * M + m]  (SQA_MN_CONTIGUOUS)
 *   B(n, k) = b[n * K + k]  (SQA_K_CONTIGUOUS, nn.Linear weight layout)
 *                        or  b[k * N + n]  (SQA_MN_CONTIGUOUS)
 * a, b bf16; c row-major [M, N] in c_dtype; bias NULL or fp32 [N].
 * accumulate != 0 adds into the existing C (fp32 C only).
 * Products with few output tiles and a long K (weight gradients, K = tokens)
 * split K over clusters of CTAs and sum the partial tiles in a fixed order:
 * C does not change from run to run, and no workspace is needed.
 * Requirements: M, N, K >= 1; K % 16 == 0; N % 16 == 0; M % 16 == 0 when A
 * is MN-contiguous.  Examples (y = x W^T, x [M, K], W [N, K]):
 *   forward  y  = sqa_gemm(x, K_CONTIGUOUS, W, K_CONTIGUOUS)            (M, N, K)
 *   input    dx = sqa_gemm(dy, K_CONTIGUOUS, W, MN_CONTIGUOUS)          (M, K, N)
 *   weight   dW = sqa_gemm(dy, MN_CONTIGUOUS, x, MN_CONTIGUOUS)         (N, K, M)
 */
typedef enum { SQA_K_CONTIGUOUS = 0, SQA_MN_CONTIGUOUS = 1 } sqa_layout_t;

sqa_status_t sqa_gemm(const void* a, sqa_layout_t a_layout, const void* b, sqa_layout_t b_layout,
                      const float* bias, void* c, sqa_dtype_t c_dtype, int accumulate,
                      int M, int N, int K, void* stream);

/*
 * sqa_device_status - synchronises `stream`, then returns SQA_ERR_TIMEOUT if
 * any kernel of this library on the current device gave up a bounded wait
 * since the last call, else SQA_ERR_INVALID_ARG if sqa_attn_decode met a
 * cache length outside [n_new, L_max] (and clears the record either way),
 * SQA_ERR_CUDA if the stream reports an error, else SQA_OK.
 */
sqa_status_t sqa_device_status(void* stream);

/*
 * sqa_selftest_wait_timeout - exercises the bounded-wait failure path on the
 * GPU without faulting anything: launches one warp that waits on a barrier
 * nothing arrives on, gives up after timeout_ms (1..10000) and records
 * SQA_ERR_TIMEOUT in the device status word, then returns normally.  A later
 * sqa_device_status() reports (and clears) it; the context stays usable.
 * Returns SQA_ERR_INVALID_ARG for an out-of-range timeout.
 */
sqa_status_t sqa_selftest_wait_timeout(int timeout_ms, void* stream);

/* Static, human-readable name of a status code. */
const char* sqa_status_string(sqa_status_t status);

/* Library version, "major.minor.patch". */
const char* sqa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SQA_H_ */
