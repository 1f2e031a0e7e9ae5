/*
 * libsqa -- full-sequence attention with decoupled query / key-value head
 * counts on NVIDIA B200 (sm_100a).
 *
 * The operation (definitions restated from the pages this library follows):
 *
 *   Query head i in [0, H_q) reads key/value group g(i) = floor(i * H_kv / H_q),
 *   so contiguous blocks of query heads share one group. G = H is multi-head
 *   attention, G = 1 multi-query attention, 1 < G < H grouped-query attention
 *   (GQA explainer, "MHA・MQA・GQAの関係" equations and head-to-group diagram).
 *   Sparse Query Attention uses fewer query heads than the base head count,
 *   which cuts the score and value FLOPs in proportion ("Sparse Query Attention
 *   (SQA)", abstract). The attention of one head is
 *     out[t] = sum_u softmax_u(scale * q[t] . k[u]) v[u]
 *   over all keys u, or over u <= t when causal (the GQA module's
 *   scaled_dot_product_attention(..., is_causal=True)).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are caller-owned DEVICE pointers to contiguous bf16 data,
 *     16-byte aligned. The library never frees or keeps them.
 *   - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy default
 *     stream) and return after the work is enqueued.
 *   - Argument errors are detected on the host before anything is launched
 *     and returned as an sqa_status; nothing is written in that case.
 *   - Device-side failures (a bounded wait inside a kernel that ran out) are
 *     recorded in a per-device status word and reported by sqa_device_status().
 *   - The library allocates no device memory per call; the layer takes a
 *     caller-provided workspace.
 *   - Thread-safe; each call may target any device (the current one is used).
 *   - Per device, the first call looks up and keeps device addresses (the
 *     status word, the static scratch array) and kernel attributes. They
 *     belong to that device's primary context: do not call the library again
 *     after cudaDeviceReset() or another teardown of that context in the same
 *     process.
 */
#ifndef SQA_H
#define SQA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQA_OK = 0,
  SQA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, bad scale */
  SQA_ERR_UNSUPPORTED = 2,  /* valid request the library does not implement (e.g. d_head other than 64/128) */
  SQA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  SQA_ERR_TIMEOUT = 4,      /* a kernel wait exceeded its limit (device status) */
  SQA_ERR_WORKSPACE = 5,    /* workspace too small or misaligned */
  SQA_ERR_BOUNDS = 6        /* debug build only: a device bounds check failed (device status) */
} sqa_status;

/*
 * Attention core.
 *   q   [B, N, H_q,  d_head]   (the [B, T, H, d] view of the GQA module)
 *   k   [B, N, H_kv, d_head]
 *   v   [B, N, H_kv, d_head]
 *   out [B, N, H_q,  d_head]   written in full
 * Requirements: B, N >= 1; 1 <= H_kv <= H_q; d_head in {64, 128};
 * scale finite and > 0 (1/sqrt(d_head) gives the SDPA default); causal in {0,1}.
 * Arithmetic: bf16 inputs, fp32 accumulation and softmax, bf16 output.
 * Returns SQA_OK once the kernel is enqueued.
 */
int sqa_attn_fwd(const void* q, const void* k, const void* v, void* out,
                 int B, int N, int H_q, int H_kv, int d_head,
                 int causal, float scale, void* stream);

/*
 * sqa_attn_fwd that also writes the row log-sum-exp the backward pass needs:
 *   lse [B, H_q, N] fp32, DEVICE, 16-byte aligned, written in full:
 *   lse[b,i,t] = ln sum_u exp(scale * q[b,t,i,:] . k[b,u,g(i),:]) over the
 *   same keys as the forward. Other arguments, requirements and results as
 *   sqa_attn_fwd.
 */
int sqa_attn_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                     int B, int N, int H_q, int H_kv, int d_head,
                     int causal, float scale, void* stream);

/*
 * Attention for a contiguous block of query rows: the rows at global
 * positions q_offset .. q_offset + N_q - 1 of a sequence of N_k tokens,
 * against all N_k keys (causal: key u visible iff u <= q_offset + t). This is
 * the per-rank step of sequence sharding, where each rank owns a block of
 * query positions and gathers every key and value.
 *   q   [B, N_q, H_q,  d_head]  (the block's query rows)
 *   k   [B, N_k, H_kv, d_head]
 *   v   [B, N_k, H_kv, d_head]
 *   out [B, N_q, H_q,  d_head]  written in full
 * Requirements as sqa_attn_fwd, plus N_q >= 1, q_offset >= 0 and
 * q_offset + N_q <= N_k. Results equal rows q_offset .. q_offset + N_q - 1 of
 * sqa_attn_fwd over the whole sequence.
 */
int sqa_attn_fwd_rows(const void* q, const void* k, const void* v, void* out,
                      int B, int N_q, int N_k, int q_offset, int H_q, int H_kv, int d_head,
                      int causal, float scale, void* stream);

/*
 * Number of kernel launches sqa_attn_fwd enqueues for these sizes on the
 * current device: 1, or 2 when the pairs of query tiles left for a partial last
 * wave of non-causal work run in a second launch whose clusters of two CTAs
 * split each pair's keys. 0 for invalid sizes or when the device cannot be
 * queried. For accounting (counting launches); nothing is enqueued.
 */
int sqa_attn_fwd_grids(int B, int N, int H_q, int H_kv, int d_head, int causal);

/*
 * Bytes of device workspace sqa_attn_bwd needs (two fp32 [B, H_q] x N row
 * arrays, rows padded to a multiple of 4 floats). Returns 0 for invalid sizes.
 */
size_t sqa_attn_bwd_workspace_bytes(int B, int N, int H_q);

/*
 * Attention backward: the gradients of sum(out * dout) with respect to q, k
 * and v, the training-time pass of the attention core (Sparse Query Attention
 * targets pre-training and fine-tuning: "Sparse Query Attention (SQA)",
 * abstract). With P = softmax(scale * q_i k_g^T) and
 * D[t] = sum_c dout[t,c] * out[t,c]:
 *   dq_i = scale * (P * (dout_i v_g^T - D)) k_g
 *   dk_g = scale * sum over heads i of group g of (P * (dout_i v_g^T - D))^T q_i
 *   dv_g = sum over heads i of group g of P^T dout_i
 * so every query head adds its share to its group's key/value gradient.
 *   q, k, v, out  as sqa_attn_fwd (out = that call's result for q, k, v)
 *   dout [B, N, H_q, d_head] bf16 upstream gradient
 *   lse  [B, H_q, N] fp32 from sqa_attn_fwd_lse on the same q, k, causal, scale
 *   dq   [B, N, H_q, d_head]  bf16, written in full
 *   dk, dv [B, N, H_kv, d_head] bf16, written in full (no accumulation into
 *        what they held)
 *   workspace: device memory of at least sqa_attn_bwd_workspace_bytes(B, N,
 *        H_q), 256-byte aligned; scratch, overwritten.
 * Requirements as sqa_attn_fwd. Arithmetic: P recomputed in fp32 from lse,
 * P and dS rounded to bf16 as tensor-core operands, fp32 accumulation.
 * SQA_ERR_WORKSPACE for a missing, misaligned or short workspace.
 */
int sqa_attn_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv,
                 void* workspace, size_t workspace_bytes,
                 int B, int N, int H_q, int H_kv, int d_head,
                 int causal, float scale, void* stream);

/*
 * Bytes of device workspace sqa_decode_fwd needs (fp32 partial results of
 * the split key ranges). Returns 0 for invalid sizes.
 */
size_t sqa_decode_workspace_bytes(int B, int N, int H_q, int H_kv, int d_head);

/*
 * Decode step: one new token per sequence attends to its whole K/V cache
 * (the autoregressive step the GQA explainer motivates, "背景と動機" and its
 * KV-cache table; every query head of a group reads the same cached K/V):
 *   out[b,i,:] = sum_u softmax_u(scale * q[b,i,:] . k_cache[b,u,g(i),:]) v_cache[b,u,g(i),:]
 * over all u in [0, N), g(i) = floor(i * H_kv / H_q). The new token's own K/V
 * are expected to be in the cache already (it is the last row of causal
 * attention over the cache).
 *   q        [B, H_q, d_head] bf16
 *   k_cache  [B, N, H_kv, d_head] bf16 (the layout of sqa_attn_fwd's k)
 *   v_cache  [B, N, H_kv, d_head] bf16
 *   out      [B, H_q, d_head] bf16, written in full
 *   workspace: device memory of at least sqa_decode_workspace_bytes(...),
 *              256-byte aligned; scratch, overwritten.
 * Requirements: B, N >= 1; 1 <= H_kv <= H_q; d_head in {64, 128}; scale
 * finite and > 0. Arithmetic: bf16 inputs, fp32 scores, softmax and sums, P
 * rounded to bf16 for the P.V product, bf16 output.
 * Errors: SQA_ERR_INVALID_ARG for bad pointers, sizes or scale;
 * SQA_ERR_UNSUPPORTED for other head sizes; SQA_ERR_WORKSPACE for a null,
 * misaligned or short workspace. Enqueues two kernels on `stream`: the split
 * pass and the merge, the merge as a programmatic dependent launch of the
 * split (it starts early and waits on the device for the split to finish).
 */
int sqa_decode_fwd(const void* q, const void* k_cache, const void* v_cache, void* out,
                   void* workspace, size_t workspace_bytes,
                   int B, int N, int H_q, int H_kv, int d_head, float scale, void* stream);

/*
 * Bytes of device workspace sqa_layer_fwd needs (Q, K, V and the merged
 * attention output, each 256-byte aligned). Returns 0 for invalid sizes.
 */
size_t sqa_layer_workspace_bytes(int B, int N, int d_model, int H_q, int H_kv, int d_head);

/*
 * Attention layer forward (the GQA explainer's module, "PyTorchでのGQA実装",
 * with H_q query heads and H_kv key/value groups, no biases):
 *   Q = x Wq^T, K = x Wk^T, V = x Wv^T   viewed [B, N, H, d_head]
 *   A = attention(Q, K, V)               merged back to [B, N, H_q * d_head]
 *   out = A Wo^T
 *   x   [B, N, d_model]
 *   Wq  [H_q * d_head,  d_model]   (nn.Linear weight layout [out, in])
 *   Wk  [H_kv * d_head, d_model]
 *   Wv  [H_kv * d_head, d_model]
 *   Wo  [d_model, H_q * d_head]
 *   out [B, N, d_model]
 *   workspace: device memory of at least sqa_layer_workspace_bytes(...),
 *   256-byte aligned; its contents are scratch and are overwritten.
 * Requirements: as sqa_attn_fwd, plus d_model >= 8 and d_model % 8 == 0.
 * Q, K and V are stored in bf16 between the kernels, as is A.
 */
int sqa_layer_fwd(const void* x, const void* Wq, const void* Wk, const void* Wv, const void* Wo,
                  void* out, void* workspace, size_t workspace_bytes,
                  int B, int N, int d_model, int H_q, int H_kv, int d_head,
                  int causal, float scale, void* stream);

/*
 * Size of the library's own per-device scratch array used by
 * sqa_layer_fwd_static_ws (64 MiB; every device that loads the library holds
 * it until the process exits).
 */
#define SQA_STATIC_WORKSPACE_BYTES (64u << 20)

/*
 * sqa_layer_fwd without a caller-provided workspace. The pages have no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory -- a framework that owns all device memory through its own
 * allocator and budget, or a plugin interface that passes the library only
 * input and output buffers. The caller still provides x, the weights and out;
 * the layer's Q/K/V/attention scratch lives in one library-owned array of
 * SQA_STATIC_WORKSPACE_BYTES per device. Nothing is allocated per call.
 *   - Same arguments, layouts, arithmetic and results as sqa_layer_fwd.
 *   - Returns SQA_ERR_WORKSPACE, without launching anything, when
 *     sqa_layer_workspace_bytes(B, N, d_model, H_q, H_kv, d_head) exceeds
 *     SQA_STATIC_WORKSPACE_BYTES (e.g. B*N*(2*H_q + 2*H_kv)*d_head*2 bytes
 *     above 64 MiB); SQA_ERR_INVALID_ARG for sizes sqa_layer_fwd rejects.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - All calls on a device share the one array, and it keeps the previous
 *     call's contents. Calls whose kernels overlap on the GPU (different
 *     streams, or host threads without ordering) race on it: order them on one
 *     stream.
 */
int sqa_layer_fwd_static_ws(const void* x, const void* Wq, const void* Wk, const void* Wv, const void* Wo,
                            void* out, int B, int N, int d_model, int H_q, int H_kv, int d_head,
                            int causal, float scale, void* stream);

/*
 * Plain projection y[M, N_out] = x[M, K] W[N_out, K]^T (bf16 in, fp32
 * accumulate, bf16 out): the layer's linear step exposed on its own.
 * Requirements: M >= 1, K >= 8, K % 8 == 0, N_out >= 8, N_out % 8 == 0.
 */
int sqa_linear_fwd(const void* x, const void* W, void* y, long long M, int K, int N_out, void* stream);

/*
 * Synchronises `stream`, then returns and clears the current device's status
 * word: SQA_OK, or SQA_ERR_TIMEOUT if any kernel gave up on a wait since the
 * last call. SQA_ERR_CUDA if the synchronisation itself failed.
 */
int sqa_device_status(void* stream);

/*
 * Upper limit (nanoseconds) on each wait inside the kernels of later calls on
 * this device; 0 restores the default (2 s). Returns the previous value.
 */
unsigned long long sqa_set_wait_limit_ns(unsigned long long ns);

/*
 * Diagnostic: launches one warp that waits on a shared-memory barrier nothing
 * ever completes, through the same bounded wait the kernels use, with the
 * given limit (nanoseconds, 1e3..1e10). Synchronises `stream` and returns the
 * status the device recorded -- SQA_ERR_TIMEOUT when the bound works -- and
 * clears it. Shows that a stuck wait ends with a status instead of a hang.
 */
int sqa_check_wait_timeout(unsigned long long limit_ns, void* stream);

/*
 * Diagnostic: the exp2 the attention kernels evaluate on the FMA pipe for part
 * of the softmax (the rest uses the hardware ex2 unit), next to CUDA's exp2f.
 * For i in [0, n): poly[i] = that polynomial 2^x[i], ref[i] = exp2f(x[i]).
 * The polynomial: x clamped at -125, x = n + f with n = round(x) and
 * f in [-1/2, 1/2], 2^f from a degree-3 polynomial with minimum maximum
 * relative error on [-1/2, 1/2] (7.5e-5), 2^n added into the exponent field.
 * x, poly, ref: DEVICE fp32 arrays, 4-byte aligned; 1 <= n <= 2^31.
 * SQA_ERR_INVALID_ARG otherwise. Asynchronous on `stream`.
 */
int sqa_check_exp2_poly(const float* x, float* poly, float* ref, long long n, void* stream);

/*
 * Diagnostic of the debug build's device bounds checks (built with
 * SQA_DEBUG_BOUNDS: every kernel checks its tile coordinates and global
 * indices and records SQA_ERR_BOUNDS in the device status word instead of
 * making the access). Launches one thread that evaluates a failing check with
 * no memory access behind it, synchronises `stream`, and returns and clears
 * the device status: SQA_ERR_BOUNDS from a debug build, SQA_OK from a release
 * build (where the checks are compiled away).
 */
int sqa_check_bounds_report(void* stream);

/* Human-readable name of a status code (static string). */
const char* sqa_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int sqa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SQA_H */
