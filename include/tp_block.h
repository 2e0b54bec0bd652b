/*
 * tp_block.h -- C ABI of the tensor-parallel transformer block on one B200.
 *
 * The block is the Megatron-style split of a transformer layer (xingyuzhitong.com
 * "Tensor vs Pipeline Parallelism", section "Tensor parallelism: split inside each
 * layer"; drpranayjha.com "AI Infrastructure series, Part 5", section "How does
 * tensor parallelism split a layer?"; aidolsgroup.com glossary "Tensor
 * Parallelism", section "Full definition"):
 *
 *   - the first linear (MLP up-projection, or the fused QKV projection split by
 *     heads) is split by its output features into t shards (column-parallel);
 *   - an elementwise activation (tanh GeLU) follows on the MLP;
 *   - the second linear (MLP down-projection, or the attention output
 *     projection) is split by its input features into the same t shards
 *     (row-parallel); every shard yields a full-size partial, and the partials
 *     are summed -- the step the pages call the all-reduce.
 *
 * Here all t shards are logical shards on one GPU.  The all-reduce is a
 * deterministic on-chip sum of the t partials inside the row-parallel kernel's
 * epilogue: partial s is accumulated from zero over its own input-feature
 * slice, the partials are added in ascending shard order in fp32, then the bias
 * once, then one rounding to bf16.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *   - Element type: bfloat16, passed as raw 16-bit patterns (tp_bf16).
 *     Arithmetic: bf16 x bf16 products accumulated in fp32; bias, GeLU and the
 *     shard sum in fp32; one round-to-nearest-even to bf16 on output.
 *   - Weights are stored [out_features, in_features] row-major (the layer
 *     computes x @ weight.T with weight shaped (out, in), iloveeagents.com
 *     section "Example").  Activations are [tokens, features] row-major.
 *   - Every pointer is caller-owned DEVICE memory on the current CUDA device,
 *     16-byte aligned.  The library never allocates, frees or synchronises:
 *     the work is enqueued asynchronously on `stream` and the call returns.
 *     Inputs must stay valid and outputs untouched until the stream reaches
 *     the work.  Outputs must not alias inputs.
 *   - Sizes: T >= 1 tokens (any value); every feature dimension (K, N, H, F)
 *     a positive multiple of 64.
 *   - tp_degree t >= 1 must divide the dimension it splits; for the
 *     row-parallel split the shard width (K / t) must be a multiple of 64; for
 *     attention t must divide both head counts (xingyuzhitong.com section
 *     "What the serving engines expose"; drpranayjha.com section "What do
 *     people get wrong?": 64 heads split 2, 4 or 8 ways, not 3 or 6).
 *   - Errors: argument checks run before any CUDA call; on failure the entry
 *     point returns a tp_status != TP_OK and enqueues nothing.  A failing
 *     CUDA call returns TP_ERR_CUDA.  No exception crosses the ABI.
 *   - Kernels never wait without bound: a wait that runs past its limit
 *     (about one second) records a device-side error and the kernel returns;
 *     tp_device_error_check() reports it as TP_ERR_DEVICE_TIMEOUT.
 *   - Results are bit-identical across repeated calls with the same
 *     arguments, whatever the order of other work on the device.
 *
 * `tp_stream_t` is the same type as cudaStream_t (NULL = the legacy default
 * stream).
 */
#ifndef TP_BLOCK_H_
#define TP_BLOCK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t tp_bf16;
typedef struct CUstream_st* tp_stream_t;

typedef enum tp_status {
  TP_OK = 0,
  TP_ERR_NULL = 1,            /* a required pointer is NULL                          */
  TP_ERR_ALIGN = 2,           /* a pointer is not 16-byte aligned                    */
  TP_ERR_SHAPE = 3,           /* T < 1, or a feature size not a positive multiple of 64 */
  TP_ERR_TP_DEGREE = 4,       /* t < 1, or t does not divide what it splits          */
  TP_ERR_WORKSPACE = 5,       /* workspace NULL or smaller than required             */
  TP_ERR_UNSUPPORTED = 6,     /* unknown activation code or option                   */
  TP_ERR_CUDA = 7,            /* a CUDA runtime / driver call failed                 */
  TP_ERR_DEVICE_TIMEOUT = 8   /* a kernel's bounded wait ran out (see above)         */
} tp_status;

typedef enum tp_act {
  TP_ACT_NONE = 0,            /* identity                                            */
  TP_ACT_GELU_TANH = 1        /* 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3)))     */
} tp_act;

/*
 * Column-parallel linear (+ bias, + activation).
 *   out[T, N] = act(x[T, K] @ w[N, K]^T + b[N])
 * Shard s of t owns output features [s N/t, (s+1) N/t) and computes them from
 * the whole of x with no exchange (iloveeagents.com section "Detail", the TP=2
 * diagram, and section "Example"); the shards' outputs side by side are `out`.
 *   x    [T, K]  activations                    (read)
 *   w    [N, K]  weight, output-feature major    (read)
 *   b    [N]     bias, or NULL for none          (read)
 *   out  [T, N]  result                          (written)
 *   act  a tp_act value
 * Requires N % t == 0.  Returns TP_OK or an error as described above.
 */
tp_status tp_colpar_gemm_gelu(const tp_bf16* x, const tp_bf16* w, const tp_bf16* b,
                              int T, int K, int N, int tp_degree, int act,
                              tp_bf16* out, tp_stream_t stream);

/*
 * Row-parallel linear with the fused shard sum (the all-reduce).
 *   P_s      = h[:, K_s] @ w[:, K_s]^T,  K_s = [s K/t, (s+1) K/t), each from zero
 *   out[T,N] = ((P_0 + P_1) + ... + P_{t-1}) + b
 * (xingyuzhitong.com section "Tensor parallelism: split inside each layer": the
 * second linear layer is split by rows and the partial results are combined by
 * an all-reduce.)
 *   h    [T, K]  activations (the column-parallel output)  (read)
 *   w    [N, K]  weight                                     (read)
 *   b    [N]     bias added once after the sum, or NULL     (read)
 *   out  [T, N]  result                                     (written)
 * Requires K % t == 0 and (K / t) % 64 == 0.
 */
tp_status tp_rowpar_gemm_reduce(const tp_bf16* h, const tp_bf16* w, const tp_bf16* b,
                                int T, int K, int N, int tp_degree,
                                tp_bf16* out, tp_stream_t stream);

/*
 * Bytes of workspace tp_mlp_forward needs for T tokens and FFN width F: the
 * bf16 activation h[T, F] between the two layers, rounded up to 256 bytes.
 * Returns 0 for T < 1 or F < 1.
 */
size_t tp_mlp_workspace_bytes(int T, int F);

/*
 * The tensor-parallel MLP block:
 *   h   = act(x @ w1^T + b1)                      column-parallel, shards of F/t
 *   out = sum_s h[:, F_s] @ w2[:, F_s]^T + b2      row-parallel, the same shards
 * (xingyuzhitong.com section "Tensor parallelism: split inside each layer";
 * drpranayjha.com section "How does tensor parallelism split a layer?").
 * Column shard s of w1 feeds exactly row shard s of w2, so the activation
 * needs no exchange; only the final partials are summed.
 *   x  [T, H], w1 [F, H], b1 [F] or NULL, w2 [H, F], b2 [H] or NULL  (read)
 *   out [T, H]                                                      (written)
 *   workspace: device memory of at least tp_mlp_workspace_bytes(T, F) bytes,
 *   16-byte aligned, holding h between the two kernels; its contents on
 *   return are unspecified.
 * Requires F % t == 0 and (F / t) % 64 == 0.
 */
tp_status tp_mlp_forward(const tp_bf16* x, const tp_bf16* w1, const tp_bf16* b1,
                         const tp_bf16* w2, const tp_bf16* b2,
                         int T, int H, int F, int tp_degree, int act,
                         tp_bf16* out, void* workspace, size_t workspace_bytes,
                         tp_stream_t stream);

/*
 * The attention block's two projections, split by heads.
 *   qkv_out[T, (nq + 2 nkv) d] = x @ w_qkv^T + b_qkv     column-parallel
 *   out[T, H] = sum_s ctx[:, G_s] @ w_o[:, G_s]^T + b_o  row-parallel
 * Shard s owns query heads [s nq/t, (s+1) nq/t) and key-value heads
 * [s nkv/t, (s+1) nkv/t) (attention heads distributed among the GPUs,
 * xingyuzhitong.com section "Tensor parallelism: split inside each layer");
 * G_s are the context columns of its query heads, (nq/t) d wide.  The
 * attention core between the projections is not part of this library: `ctx`
 * is the per-head context supplied by the caller.
 *   x      [T, H]                 w_qkv [(nq + 2 nkv) d, H], columns ordered
 *                                 Q heads | K heads | V heads, each d wide
 *   b_qkv  [(nq + 2 nkv) d] or NULL
 *   ctx    [T, nq d]              w_o   [H, nq d]       b_o [H] or NULL
 *   qkv_out[T, (nq + 2 nkv) d]    out   [T, H]          (written)
 * Requires t | nq, t | nkv, ((nq / t) d) % 64 == 0 and (nq + 2 nkv) d % 64 == 0.
 * Key-value heads are not replicated when t > nkv: such t is rejected.
 */
tp_status tp_attn_proj_forward(const tp_bf16* x, const tp_bf16* w_qkv, const tp_bf16* b_qkv,
                               const tp_bf16* ctx, const tp_bf16* w_o, const tp_bf16* b_o,
                               int T, int H, int n_q_heads, int n_kv_heads, int head_dim,
                               int tp_degree, tp_bf16* qkv_out, tp_bf16* out,
                               tp_stream_t stream);

/*
 * Bytes of workspace tp_mlp_backward needs: three [T, F] bf16 activations (the
 * pre-activation z, its gradient dz and h = act(z)), each rounded up to 256
 * bytes.  Returns 0 for T < 1 or F < 1.
 */
size_t tp_mlp_backward_workspace_bytes(int T, int F);

/*
 * Backward pass of the tensor-parallel MLP block (tp_mlp_forward) for an
 * upstream gradient dy = dL/dy.  The split needs two more all-reduces per layer
 * in the backward pass (xingyuzhitong.com "Tensor vs Pipeline Parallelism",
 * section "Tensor parallelism: split inside each layer"); for the MLP the one
 * that carries data is the sum over shards of the input gradient, since every
 * column shard used all of x.  dy reaches every shard whole, and each weight
 * gradient stays on the shard that owns the weight:
 *   z    = x w1^T + b1                      (recomputed, column-parallel)
 *   dz   = (dy w2) * act'(z),  h = act(z)    shard s: columns F_s, no exchange
 *   dx   = ((dz[:,F_0] w1[F_0,:] + dz[:,F_1] w1[F_1,:]) + ...)   fused shard sum,
 *          each partial from zero, ascending shard order
 *   dw1  = dz^T x [F, H],   dw2 = dy^T h [H, F]   (contractions over tokens)
 *   db1  = sum over tokens of dz [F],  db2 = sum over tokens of dy [H]
 * Arithmetic: bf16 operands, fp32 accumulation; z, dz and h are rounded to
 * bf16 once, in the workspace; every output is rounded once to bf16.
 *   x [T, H], w1 [F, H], b1 [F] or NULL, w2 [H, F], dy [T, H]    (read)
 *   dx [T, H], dw1 [F, H], dw2 [H, F]                           (written)
 *   db1 [F], db2 [H]: written unless NULL
 *   workspace: at least tp_mlp_backward_workspace_bytes(T, F) bytes, 16-byte
 *   aligned; on return it holds z, dz and h (in that order, each in its
 *   256-byte-rounded slot).
 * Requires F % t == 0 and (F / t) % 64 == 0; T >= 1 is arbitrary.
 */
tp_status tp_mlp_backward(const tp_bf16* x, const tp_bf16* w1, const tp_bf16* b1,
                          const tp_bf16* w2, const tp_bf16* dy,
                          int T, int H, int F, int tp_degree, int act,
                          tp_bf16* dx, tp_bf16* dw1, tp_bf16* db1, tp_bf16* dw2, tp_bf16* db2,
                          void* workspace, size_t workspace_bytes, tp_stream_t stream);

/*
 * Bytes of workspace tp_attn_decode needs for T new tokens after `past` cached
 * ones (the per-chunk partial results); 0 for unsupported arguments.  A
 * function of the sizes only.
 */
size_t tp_attn_decode_workspace_bytes(int T, int past, int n_q_heads, int n_kv_heads,
                                      int head_dim);

/*
 * The attention core between the two projections of tp_attn_proj_forward, for
 * decode: T new tokens of one sequence attend over its key-value cache.
 * Attention heads are distributed among the tensor-parallel shards, each with
 * its share of the KV cache, so the core needs no exchange (xingyuzhitong.com
 * "Tensor vs Pipeline Parallelism", section "Tensor parallelism: split inside
 * each layer"; drpranayjha.com "AI Infrastructure series, Part 5", section "How
 * does tensor parallelism split a layer?"): shard s owns query heads
 * [s nq/t, (s+1) nq/t), key-value heads [s nkv/t, (s+1) nkv/t) and their cache
 * rows.  On one GPU the shards are head groups of one grid.
 *   1. the new tokens' keys and values (columns K and V of qkv) are written
 *      into the cache at positions [past, past + T);
 *   2. ctx[i, h d .. h d + d) = sum_j p_j v_j over keys j <= past + i of
 *      key-value head g = h / (nq / nkv), with p = softmax_j(q_i,h . k_j / sqrt(d))
 *      (causal, grouped-query; no positional rotation is applied here).
 * Arithmetic: bf16 q, k, v; scores, maxima and sums in fp32; the softmax
 * weights are rounded to bf16 for the weighted sum of v (fp32 accumulate) and
 * their row sum is taken from the rounded weights; the keys are processed in
 * chunks whose partial results are merged in a fixed order, so the
 * result is bit-identical from run to run and does not depend on the GPU.
 *   qkv      [T, (nq + 2 nkv) d]  tp_attn_proj_forward's qkv_out   (read)
 *   k_cache  [nkv, max_len, d]    rows [0, past) hold the cached keys;
 *                                 rows [past, past + T) are written
 *   v_cache  [nkv, max_len, d]    likewise for values
 *   ctx      [T, nq d]            the input of the output projection (written)
 *   workspace: at least tp_attn_decode_workspace_bytes(...) bytes, 16-byte
 *   aligned; contents on return unspecified.
 * Requires head_dim == 128 (else TP_ERR_UNSUPPORTED), nq / nkv in {1, 2, 4,
 * 8, 16} (else TP_ERR_UNSUPPORTED), past + T <= max_len (else TP_ERR_SHAPE),
 * and t dividing both head counts (else TP_ERR_TP_DEGREE).  Calls that
 * overlap on the GPU must not share a workspace or a cache.
 */
tp_status tp_attn_decode(const tp_bf16* qkv, tp_bf16* k_cache, tp_bf16* v_cache, int T, int past,
                         int max_len, int n_q_heads, int n_kv_heads, int head_dim, int tp_degree,
                         tp_bf16* ctx, void* workspace, size_t workspace_bytes,
                         tp_stream_t stream);

/*
 * The same attention core as tp_attn_decode (same sharding, same causal
 * grouped-query operation, same cache update), for many new tokens at once: a
 * prompt (past = 0) or a chunk of one appended after `past` cached tokens.
 * The queries of one head fill 128-row tiles; each tile streams the keys and
 * values it may see once, with a running softmax, and needs no workspace.
 *   1. the new tokens' keys and values (columns K and V of qkv) are written
 *      into the cache at positions [past, past + T);
 *   2. ctx[i, h d .. h d + d) = sum_j p_j v_j over keys j <= past + i of
 *      key-value head h / (nq / nkv), p = softmax_j(q_i,h . k_j / sqrt(d)).
 * Arithmetic: bf16 q, k, v; scores, maxima and sums in fp32; the softmax
 * weights are rounded to bf16 for the weighted sum of v (fp32 accumulate) and
 * their row sum is taken from the fp32 weights before that rounding.  The
 * running maximum is raised only when a block of 128 keys exceeds it by more
 * than a factor 2^8, so the weights lie in [0, 2^8] before normalisation.
 * The key blocks of a row are visited in ascending order by one CTA, so the
 * result is bit-identical from run to run.
 *   qkv      [T, (nq + 2 nkv) d]  tp_attn_proj_forward's qkv_out   (read)
 *   k_cache  [nkv, max_len, d]    rows [0, past) hold the cached keys;
 *                                 rows [past, past + T) are written
 *   v_cache  [nkv, max_len, d]    likewise for values
 *   ctx      [T, nq d]            the input of the output projection (written)
 * Requires head_dim == 128 (else TP_ERR_UNSUPPORTED), nq a multiple of nkv and
 * past + T <= max_len (else TP_ERR_SHAPE), and t dividing both head counts
 * (else TP_ERR_TP_DEGREE).  Calls that overlap on the GPU must not share a
 * cache.
 */
tp_status tp_attn_prefill(const tp_bf16* qkv, tp_bf16* k_cache, tp_bf16* v_cache, int T,
                          int past, int max_len, int n_q_heads, int n_kv_heads, int head_dim,
                          int tp_degree, tp_bf16* ctx, tp_stream_t stream);

/*
 * The sequence-parallel region after a row-parallel linear: residual add and
 * RMSNorm, token shard by token shard.  Sequence parallelism splits the parts
 * of a layer that tensor parallelism leaves whole (normalisation, dropout)
 * along the sequence inside the tensor-parallel group (drpranayjha.com "AI
 * Infrastructure series, Part 5", section "What about MoE models and very long
 * prompts?"): the row-parallel all-reduce becomes a reduce-scatter that leaves
 * shard s the summed rows of its tokens [s T/t, (s+1) T/t), the shard adds
 * the residual stream and normalises its rows, and an all-gather returns every
 * token for the next column-parallel linear.  On one GPU tp_rowpar_gemm_reduce
 * has already summed every row (the reduce-scatter and the all-gather together
 * are that all-reduce), so this call is the per-shard region itself:
 *   r_out = residual + y
 *   n_out = r / sqrt(mean_j r_j^2 + eps) * gamma      (RMSNorm of each token row)
 * Arithmetic: fp32 from the bf16 inputs; n is computed from the fp32 r; each
 * output is rounded once to bf16; the sum of squares is taken in a fixed order.
 *   y [T, H] (the row-parallel output), residual [T, H], gamma [H]  (read)
 *   r_out [T, H], n_out [T, H]                                       (written)
 *   eps >= 0 (1e-5 for Llama-shaped models)
 * Requires T % t == 0 (equal token shards; else TP_ERR_TP_DEGREE) and H a
 * positive multiple of 64.  Dropout is the identity at inference and is not
 * applied.
 */
tp_status tp_sp_add_rmsnorm(const tp_bf16* y, const tp_bf16* residual, const tp_bf16* gamma,
                            int T, int H, int tp_degree, float eps, tp_bf16* r_out,
                            tp_bf16* n_out, tp_stream_t stream);

/*
 * Largest activation h[T, F] (T * F * 2 bytes) that tp_mlp_forward_noalloc can
 * hold: 4 MiB, e.g. 64 tokens at F = 28672 or 2048 tokens at F = 1024.
 */
#define TP_NOALLOC_SCRATCH_BYTES (4u * 1024u * 1024u)

/*
 * tp_mlp_forward for callers that cannot allocate device memory.
 *
 * The reference pages have no counterpart of this call; it exists for the
 * callers of this library that cannot obtain scratch memory: plugin hosts
 * that hand a kernel library only its input and output buffers (no workspace,
 * no allocator), processes whose device memory is wholly owned by another
 * allocator, and latency-critical loops that must not take cudaMalloc's
 * implicit device synchronisation.
 *
 * Same arguments, arithmetic and results as tp_mlp_forward, minus the
 * workspace: h lives in one TP_NOALLOC_SCRATCH_BYTES array in the library's
 * own device memory (a static __device__ array, held by every GPU that loads
 * the library until the process exits).  The call allocates nothing and calls
 * no allocating routine.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture on the device.
 *   - Every call on a device shares the one array.  Calls that may overlap
 *     on the GPU (different streams, or other host threads) race on it and
 *     must be ordered by the caller.  h is fully written before it is read,
 *     so nothing needs clearing between calls.
 * Returns TP_ERR_WORKSPACE, before any CUDA call, if T * F * 2 exceeds
 * TP_NOALLOC_SCRATCH_BYTES; otherwise the errors of tp_mlp_forward, and
 * TP_ERR_CUDA if the array's address cannot be obtained.
 */
tp_status tp_mlp_forward_noalloc(const tp_bf16* x, const tp_bf16* w1, const tp_bf16* b1,
                                 const tp_bf16* w2, const tp_bf16* b2,
                                 int T, int H, int F, int tp_degree, int act,
                                 tp_bf16* out, tp_stream_t stream);

/*
 * 8-bit weights (decode).  In decode every token reads every weight, so the
 * weight bytes set the time per token; the pages' example reads a 70B model
 * in 8-bit (drpranayjha.com "AI Infrastructure series, Part 5", section
 * "Reason 2: one user's answers are too slow").  These calls take each weight
 * as FP8 E4M3 bytes (the OCP "E4M3FN" encoding: sign, 4 exponent bits with
 * bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN) with one fp32
 * scale per output row:
 *   W[n, k] = w_scale[n] * e4m3(w8[n, k])
 * and otherwise compute exactly what the bf16 calls compute with that W:
 * bf16 activations, fp32 accumulation (every E4M3 value is a bf16 value, so
 * the products are the bf16 kernel's), the scale applied to the fp32 sum of
 * each output before bias and activation.
 *   w8       [N, K] (w1: [F, H], w2: [H, F]) bytes, row-major, 16-byte aligned
 *   w_scale  [N] fp32 (s1: [F], s2: [H]), 16-byte aligned
 * Other arguments, checks and errors as tp_colpar_gemm_gelu,
 * tp_rowpar_gemm_reduce and tp_mlp_forward.  These calls always use the
 * weight-streaming kernel: T <= 128 (else TP_ERR_UNSUPPORTED); row-parallel
 * calls whose shards would not fit two per streaming CTA also return
 * TP_ERR_UNSUPPORTED (none of t <= 8 at the 70B shapes).  tp_mlp_forward_w8
 * checks both layers' splits before it launches anything, so such a return
 * leaves the workspace and out untouched.
 */
tp_status tp_colpar_gemm_gelu_w8(const tp_bf16* x, const uint8_t* w8, const float* w_scale,
                                 const tp_bf16* b, int T, int K, int N, int tp_degree, int act,
                                 tp_bf16* out, tp_stream_t stream);

tp_status tp_rowpar_gemm_reduce_w8(const tp_bf16* h, const uint8_t* w8, const float* w_scale,
                                   const tp_bf16* b, int T, int K, int N, int tp_degree,
                                   tp_bf16* out, tp_stream_t stream);

tp_status tp_mlp_forward_w8(const tp_bf16* x, const uint8_t* w1, const float* s1,
                            const tp_bf16* b1, const uint8_t* w2, const float* s2,
                            const tp_bf16* b2, int T, int H, int F, int tp_degree, int act,
                            tp_bf16* out, void* workspace, size_t workspace_bytes,
                            tp_stream_t stream);

/* A short English description of a status code (static storage). */
const char* tp_status_string(tp_status status);

/*
 * Text of the last CUDA runtime / driver error that made an entry point
 * return TP_ERR_CUDA on the calling host thread ("no CUDA error recorded"
 * if none).  The string lives in thread-local storage until the next call.
 */
const char* tp_last_cuda_error(void);

/*
 * Synchronises the current device, then reads and clears the library's
 * device-side error word.  Returns TP_ERR_DEVICE_TIMEOUT if any kernel of
 * this library ran out a bounded wait since the last check, TP_ERR_CUDA if the
 * synchronisation itself failed, TP_OK otherwise.
 */
tp_status tp_device_error_check(void);

/*
 * Diagnostic (not part of the block): makes the library's bounded wait run out
 * on purpose, so a caller or a test can check the timeout path without a fault
 * or a hang.  Launches one CTA on `stream` in which two roles wait on barriers
 * that nothing arrives on: the first with a limit of `limit_us` microseconds,
 * the second with the library's normal limit (about one second) but sharing
 * the CTA's abort flag, so it must give up as soon as the first one has.
 *   limit_us  1 .. 1000000
 *   result    device int[3], 16-byte aligned (written): what the two waits
 *             returned (1 = completed, 0 = gave up; both are 0), and the
 *             nanoseconds the second wait took
 * After the kernel, tp_device_error_check() returns TP_ERR_DEVICE_TIMEOUT once
 * and clears the error word.  Returns TP_ERR_NULL, TP_ERR_ALIGN or
 * TP_ERR_UNSUPPORTED (limit out of range) before any launch, TP_ERR_CUDA if
 * the launch fails.
 */
tp_status tp_diag_bounded_wait(unsigned int limit_us, int* result, tp_stream_t stream);

/*
 * Token count at or below which a call takes the weight-streaming (decode)
 * kernels instead of the tiled (prefill) kernels.  `max_tokens` in [0, 128];
 * 0 sends every call to the tiled kernels.  Process-wide; returns
 * TP_ERR_UNSUPPORTED for values outside the range.  The default is 128.
 */
tp_status tp_set_decode_max_tokens(int max_tokens);
int tp_get_decode_max_tokens(void);


/*
 * Launch options, process-wide, a bitwise OR of:
 *   TP_OPT_PDL             launch with programmatic dependent launch, so a
 *                          kernel's set-up (barriers, tensor memory, descriptor
 *                          prefetch) overlaps the tail of the preceding kernel
 *                          on the stream.  Activations are read and outputs
 *                          written only after that kernel has completed.  On by
 *                          default.
 *   TP_OPT_STATIC_WEIGHTS  with TP_OPT_PDL: a kernel may also start reading its
 *                          weights (w, w1, w2, w_qkv, w_o) before the preceding
 *                          kernel on the stream has completed.  Set it only when
 *                          no kernel that may run just before a call writes that
 *                          call's weights -- e.g. inference with weights loaded
 *                          once.  Off by default.
 * Returns TP_ERR_UNSUPPORTED for unknown bits (and changes nothing).
 */
#define TP_OPT_PDL 1u
#define TP_OPT_STATIC_WEIGHTS 2u
tp_status tp_set_launch_options(unsigned int flags);
unsigned int tp_get_launch_options(void);

/*
 * The launch the weight-streaming kernel makes for one linear layer, computed
 * for a device with `sms` multiprocessors and `max_smem` bytes of opt-in
 * shared memory per block.  Host arithmetic only: no device is touched, so it
 * also runs without a GPU.
 *   T, K, N     tokens, input features, output features of the layer
 *   row_shards  1 for a column-parallel layer, t for a row-parallel one
 *               (t must divide K into multiples of 64)
 *   w8          nonzero for 8-bit weights (the *_w8 calls)
 * Fills *plan and returns TP_OK; TP_ERR_UNSUPPORTED when the streaming kernel
 * does not take the layer (T > 128, no cluster shape, or an 8-bit split with
 * more than two shards per CTA: the bf16 calls then use the tiled kernel, the
 * *_w8 calls return TP_ERR_UNSUPPORTED); TP_ERR_NULL for a NULL plan;
 * TP_ERR_SHAPE or TP_ERR_TP_DEGREE for bad sizes.  Whether a bf16 call
 * streams at all also depends on tp_set_decode_max_tokens.
 */
typedef struct {
  int grid_x;           /* 128-row weight tiles (the grid is grid_x x cluster CTAs) */
  int cluster;          /* CTAs per thread-block cluster, splitting K */
  int jsplit;           /* CTAs that share one shard's K-slice */
  int shards_per_cta;   /* row-parallel shards one CTA sums */
  int stages;           /* depth of the shared-memory ring */
  int kblocks_per_box;  /* 64-column k-blocks per TMA box */
  int stage_bytes;      /* bytes of one ring stage */
  int smem_bytes;       /* dynamic shared memory per CTA */
  int l2_ahead;         /* boxes sent to L2 before the wait on the preceding grid */
} tp_stream_plan_t;
tp_status tp_stream_plan(int T, int K, int N, int row_shards, int w8, int sms, int max_smem,
                         tp_stream_plan_t* plan);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* TP_BLOCK_H_ */
