/*
 * libdma — C ABI of the B200 (sm_100a) hot path of Doge's Dynamic Mask Attention.
 *
 * Source of the method: the page "Transformers 中的 Doge 小语言模型完全指南：
 * 动态掩码注意力（DMA）与跨域 MoE（CDMoE）架构解析与实战" (blog.gitcode.com), section
 * "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码" (written [DMA] below; its
 * forward-chain steps are [DMA step 3] and [DMA step 4]) and section
 * "DogeConfig 全参数详解" ([Config]).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them, and keeps no per-call state.
 *   - bf16 tensors are passed as `const void*` and hold IEEE bfloat16 values.
 *   - Layouts are dense row-major, innermost dimension last:
 *       q (prefill)   [B, L, Hq, d]        q (decode) [B, Hq, d]
 *       k, v          [B, L, Hkv, d]       caches     [B, Lk, Hkv, d]
 *       out           same layout as q
 *       W_dt          [Hkv*d, Hkv] float32, input-major: x[g] = sum_c v_flat[c] * W_dt[c, g],
 *                     with v_flat[h'*d + e] = v[h', e] (head-major flattening); no bias
 *       A             [Hkv] float32
 *       dt            [B, Hkv, L] float32
 *       lengths       [B] int32 valid lengths (right padding), or NULL = all full
 *   - GQA: query head h reads kv head g = h / (Hq / Hkv).
 *   - Every pointer must be 16-byte aligned.  Supported: d in {64, 128},
 *     Hkv in {1, 2, 4, 8, 16}, Hq a multiple of Hkv with Hq/Hkv <= 8,
 *     L (or Lk) in [1, 2^20], keep_window_size >= 1 (at most 8192 whenever
 *     the key length exceeds it), an sm_100 device.
 *   - Calls are asynchronous on `stream` and ordered after the work enqueued on
 *     it before them.  Some of a call's kernels are launched with programmatic
 *     dependent launch: they may become resident while the previous kernel on
 *     the stream finishes, but they wait for it to complete before reading any
 *     input, so stream order holds for every pointer passed in.
 *   - Calls return a status at once; they only
 *     fail synchronously on argument errors and launch errors.  Faults found
 *     on the device (a length outside [1, Lk], a bounded wait that gave up) are
 *     recorded in the workspace's status word; read them with dma_check().
 *   - A workspace must be zeroed once before its first use.  Its first 256
 *     bytes are a header: the status word at byte 0 (kernels only ever set
 *     it) and, at bytes 64-71, a work-item counter of the d = 128 prefill
 *     attention, which every such call leaves at zero when it ends.
 *   - Calls on different streams must use different workspaces.
 */
#ifndef DMA_H_
#define DMA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DMA_API __attribute__((visibility("default")))
#else
#define DMA_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* dma_stream_t;

typedef enum {
  DMA_OK = 0,
  DMA_ERR_INVALID_ARG = 1, /* NULL pointer, non-positive size, Hq % Hkv != 0, misaligned pointer */
  DMA_ERR_UNSUPPORTED = 2, /* shape outside the supported set, or not an sm_100 device */
  DMA_ERR_WORKSPACE = 3,   /* workspace smaller than dma_workspace_size() */
  DMA_ERR_CUDA = 4,        /* a CUDA call failed; dma_last_cuda_error() has the code */
  DMA_ERR_TIMEOUT = 5,     /* a bounded device wait gave up (reported by dma_check) */
  DMA_ERR_BAD_LENGTH = 6,  /* a lengths[b] outside [1, Lk] (reported by dma_check; clamped) */
  DMA_ERR_BAD_POSITION = 7 /* a prologue token outside the cache (reported by dma_check; not written) */
} dma_status_t;

/*
 * Workspace bytes needed by one call.  Prefill geometry: Lq == Lk == L.
 * Decode geometry: Lq == 1, Lk = cache length.  Returns 0 for any other
 * geometry or unsupported sizes.
 */
DMA_API size_t dma_workspace_size(int B, int Lq, int Lk, int Hq, int Hkv, int d, int keep_window_size);

/*
 * S1, [DMA step 3]: dt = exp(A * softplus(dt_proj(value_states))), in float32.
 *   v       [B, L, Hkv, d] bf16 value states
 *   W_dt    [Hkv*d, Hkv] float32, A [Hkv] float32
 *   dt_out  [B, Hkv, L] float32 (written)
 */
DMA_API dma_status_t dma_dt_scores(const void* v, const float* W_dt, const float* A, int B, int L, int Hkv, int d,
                           float* dt_out, dma_stream_t stream);

/*
 * S2, [DMA step 3] prepare_dynamic_mask: for every (b, g, query row) the kept
 * key set.  A row sees the keys a causal mask and the padding leave it (query
 * row i of a prefill sees keys j <= i, j < len_b; the decode query sits at
 * position len_b - 1 and sees keys j < len_b).  When Lk > keep_window_size the
 * row keeps its keep_window_size best keys by dt (ties: lower key index);
 * otherwise it keeps every key it sees.
 *   dt           [B, Hkv, Lk] float32
 *   Lq           Lk (prefill geometry) or 1 (decode geometry)
 *   tau_out      [B, Hkv, Lq] uint64 or NULL.  tau = (bits(dt[j*]) << 32) | (0xFFFFFFFF - j*)
 *                for the row's worst kept key j* when the top-k is active and the row
 *                sees more than keep_window_size keys, else 0.  A seen key j is kept
 *                iff (bits(dt[j]) << 32 | (0xFFFFFFFF - j)) >= tau.
 *   bitmask_out  [B, Hkv, Lq, ceil(Lk/32)] uint32 or NULL: bit (j % 32) of word j / 32
 *                is 1 iff key j is kept.  Expanded from the compact plan the
 *                attention kernels read (debug/test use; it is Lq*Lk bits).
 *   workspace    dma_workspace_size(B, Lq, Lk, Hkv, Hkv, 64, keep_window_size) bytes
 *                or more; on return it holds the compact plan (the block map the
 *                attention kernels read), laid out as below.
 *
 * Compact plan layout in the workspace.  Offsets are in bytes; each array
 * starts at the next multiple of 256 after the previous one ends; the first
 * 256 bytes are the header (status word at offset 0).
 *   Prefill geometry (Lq == Lk == L), n_rt = ceil(L / 128) row tiles,
 *   tiles = B * Hkv * n_rt ordered ((b * Hkv + g) * n_rt + t),
 *   cap = roundup(L > w ? min(w + 127, L) : L, 128):
 *     dt     [B, Hkv, L]        float32   (written by dma_forward_prefill when dt_in is NULL)
 *     tau    [B, Hkv, L]        uint64    row thresholds (as tau_out)
 *     idx    [tiles, cap]       int32     the keys any row of the tile keeps: first
 *                                         those every row keeps, then the others (in
 *                                         index order when no row needs the top-k;
 *                                         otherwise the order inside a class is free)
 *     bias   [tiles, cap]       float32   dt of the listed key
 *     span   [tiles, cap]       uint32    lo | hi << 16: the tile rows [lo, hi) keeping it
 *     counts [tiles]            int32 x2  (n_full, n_total): entries [0, n_full) are kept
 *                                         by every row; entries from n_total up to the
 *                                         next multiple of 128 are padding (span 0)
 *     kbase  [tiles, cap / 128] int32     j0 when 128-entry block k lists exactly
 *                                         j0, j0+1, ..., else -1
 *   Decode geometry (Lq == 1), cap = roundup(min(Lk, w), 128):
 *     dt [B, Hkv, Lk] float32, tau [B, Hkv] uint64, idx [B, Hkv, cap] int32 (the
 *     kept keys, in any order), bias [B, Hkv, cap] float32, count [B, Hkv] int32, then the
 *     split-K partials of dma_decode_step.
 */
DMA_API dma_status_t dma_build_mask(const float* dt, const int32_t* lengths, int B, int Hkv, int Lq, int Lk,
                            int keep_window_size, uint64_t* tau_out, uint32_t* bitmask_out, void* workspace,
                            size_t ws_bytes, dma_stream_t stream);

/*
 * S1 + S2 + S3, [DMA steps 3-4]: prefill attention with the dynamic mask.
 * For query head h of kv group g and row i:
 *   out[b, i, h, :] = sum_j p_j v[b, j, g, :],
 *   p = softmax_fp32(scale * q[b, i, h, :] . k[b, j, g, :] + dt[b, g, j]) over the kept keys j.
 *   dt_in   [B, Hkv, L] float32 or NULL; when given, S1 is skipped and dt_in is used.
 *   scale   normally d^-0.5 ([DMA step 4]); must lie in [1e-20, 1e20] (the kernel adds the
 *           bias through the tensor core as dt / scale), else DMA_ERR_INVALID_ARG.
 *   out     [B, L, Hq, d] bf16 (written; rows i >= len_b are computed with the same rule).
 */
DMA_API dma_status_t dma_forward_prefill(const void* q, const void* k, const void* v, const float* W_dt, const float* A,
                                 const int32_t* lengths, int B, int L, int Hq, int Hkv, int d, int keep_window_size,
                                 float scale, const float* dt_in, void* out, void* workspace, size_t ws_bytes,
                                 dma_stream_t stream);

/*
 * As dma_forward_prefill, and also writes each query row's softmax
 * normaliser for a later dma_backward_prefill:
 *   lse_out  [B, Hq, L] float32 (16-byte aligned; written): log2 of the sum over
 *            the row's kept keys of 2^((q.k * scale + dt) * log2(e)), i.e. the
 *            natural log-sum-exp times log2(e); 0 for a row that keeps no key.
 */
DMA_API dma_status_t dma_forward_prefill_lse(const void* q, const void* k, const void* v, const float* W_dt,
                                             const float* A, const int32_t* lengths, int B, int L, int Hq, int Hkv,
                                             int d, int keep_window_size, float scale, const float* dt_in, void* out,
                                             float* lse_out, void* workspace, size_t ws_bytes, dma_stream_t stream);

/*
 * S4, [DMA step 3 closing paragraph, step 4]: one decode step.  dt is computed
 * over the whole cached value states, the query at position len_b - 1 keeps
 * its keep_window_size best cached keys, and attends to them as above.
 *   q       [B, Hq, d] bf16;  k_cache, v_cache [B, Lk, Hkv, d] bf16 (hold the current token)
 *   dt_in   [B, Hkv, Lk] float32 or NULL
 *   out     [B, Hq, d] bf16
 */
DMA_API dma_status_t dma_decode_step(const void* q, const void* k_cache, const void* v_cache, const float* W_dt,
                             const float* A, const int32_t* lengths, int B, int Lk, int Hq, int Hkv, int d,
                             int keep_window_size, float scale, const float* dt_in, void* out, void* workspace,
                             size_t ws_bytes, dma_stream_t stream);

/*
 * Prologue, [DMA steps 1-2]: the steps of the attention forward between the
 * projections and the dynamic mask, for L new tokens per sequence.  Q and K
 * each pass an RMSNorm over head_dim (q_norm / k_norm: Llama's RMSNorm, which
 * the page says Doge reuses) and then the rotary position embedding (Llama's
 * pairing of channel i with channel i + d/2); K and V are appended to the
 * cache (past_key_values.update).  For token t of sequence b, pos = positions[b] + t:
 *   y_c        = w_c * x_c / sqrt(mean over the d channels of x^2 + eps)
 *   a_i        = pos * rope_theta^(-2i/d),  i < d/2
 *   out_i      = y_i cos a_i - y_{i+d/2} sin a_i
 *   out_{i+d/2} = y_{i+d/2} cos a_i + y_i sin a_i
 * computed in float32 (angles in double precision) and rounded once to bf16.
 *   q, k, v        [B, L, Hq, d], [B, L, Hkv, d], [B, L, Hkv, d] bf16 projected states
 *   q_norm_w, k_norm_w  [d] float32 RMSNorm weights;  eps: rms_norm_eps ([Config]: 1e-6)
 *   rope_theta     > 1 (the page gives no default; Llama's is 10000)
 *   positions      [B] int32 (device): cache row of each sequence's first new token
 *   q_out          [B, L, Hq, d] bf16 (written)
 *   k_cache, v_cache [B, Lmax, Hkv, d] bf16: rows positions[b] .. positions[b] + L - 1
 *                  are written (normalised and rotated K; V as given); other rows untouched
 *   workspace      >= 256 bytes, zeroed once: its status word records a token whose
 *                  cache row lies outside [0, Lmax) (DMA_ERR_BAD_POSITION via dma_check);
 *                  such a token's q_out row is still written, its cache rows are not.
 * Supported: d in {64, 128}, Hq a multiple of Hkv, Hkv <= 16, Hq / Hkv <= 8.
 */
DMA_API dma_status_t dma_prologue(const void* q, const void* k, const void* v, const float* q_norm_w,
                                  const float* k_norm_w, float eps, float rope_theta, const int32_t* positions,
                                  int B, int L, int Lmax, int Hq, int Hkv, int d, void* q_out, void* k_cache,
                                  void* v_cache, void* workspace, size_t ws_bytes, dma_stream_t stream);

/*
 * Backward of S1 + S2 + S3 ([DMA step 3] closing paragraph: dt is learnt end
 * to end from the value states; [DMA step 4]).  The top-k selection has no
 * gradient: each row's kept set is held fixed, and the gradient reaches dt
 * through the kept keys' bias.  For the loss sum(out * dout):
 *   dP = dO V^T, D_i = dO_i . O_i, dS = P (dP - D),
 *   dq = scale dS K, dk = scale dS^T Q, dv = P^T dO + (dt path),
 *   d_dt[b, g, j] = sum over the group's heads and rows of dS[., j],
 *   dt = exp(A softplus(x)), x = v_flat W_dt:
 *   dA = sum d_dt dt softplus(x), dx = d_dt dt A sigmoid(x),
 *   dW_dt = v_flat^T dx, dv_flat += dx W_dt^T.
 * Arguments as dma_forward_prefill, plus:
 *   out      [B, L, Hq, d] bf16: the forward's output for the same inputs
 *   dout     [B, L, Hq, d] bf16: the gradient of the loss with respect to out
 *   lse_in   [B, Hq, L] float32 or NULL: the forward's row normalisers
 *            (dma_forward_prefill_lse); when NULL they are recomputed (one more
 *            pass over every row tile's kept keys).
 *   dq       [B, L, Hq, d] bf16 (written);  dk, dv [B, L, Hkv, d] bf16 (written)
 *   d_dt     [B, Hkv, L] float32 (written) or NULL
 *   dW_dt    [Hkv*d, Hkv] float32 (written);  dA [Hkv] float32 (written)
 *   dt_in    as in the forward (NULL: dt computed from W_dt and A); the dt chain
 *            always starts from W_dt and A, which are required.
 *   workspace  dma_backward_workspace_size(...) bytes, zeroed once (status word first).
 * The accumulations (dk, dv, d_dt, dW_dt, dA) add float32 partial sums in an
 * unspecified order, so results may differ in the last bits between calls.
 */
DMA_API size_t dma_backward_workspace_size(int B, int L, int Hq, int Hkv, int d, int keep_window_size);
DMA_API dma_status_t dma_backward_prefill(const void* q, const void* k, const void* v, const float* W_dt,
                                          const float* A, const int32_t* lengths, int B, int L, int Hq, int Hkv,
                                          int d, int keep_window_size, float scale, const float* dt_in,
                                          const void* out, const void* dout, const float* lse_in, void* dq,
                                          void* dk, void* dv, float* d_dt, float* dW_dt, float* dA, void* workspace,
                                          size_t ws_bytes, dma_stream_t stream);

/*
 * CDMoE routing ([CDMoE], section "跨域 MoE（CDMoE）" of the same page): the
 * routed experts of the Cross Domain Mixture of Experts for T tokens.
 * router_gate maps each hidden state to 2K logits (K = num_keys =
 * floor(sqrt(num_experts))): columns [0, K) are domain x, [K, 2K) domain y.
 * Each domain keeps its top_k best keys (ties: lower key index); pair (a, b)
 * of the two kept sets scores s_x[a] + s_y[b] (float32) and names expert
 * a * K + b; the token keeps the top_k best pairs (ties: lower expert index),
 * weights them by the softmax of their scores, and adds
 *   out = sum_e w_e * silu(h . down_embed[e]) * up_embed[e].
 *   h            [T, hidden] bf16 hidden states
 *   W_router     [2K, hidden] bf16 router_gate weight (the Linear layout: one row per logit), no bias
 *   down_embed, up_embed  [num_experts, hidden] bf16 expert tables
 *   num_experts  K * K with K in {16, 32, 64, 128};  top_k in [1, min(K, 64)]
 *   hidden       a multiple of 64, at most 8192
 *   logits_in    [T, 2K] float32 or NULL: when given, the router GEMM is skipped
 *   out          [T, hidden] bf16 (written): the routed part, to be added to the shared expert's output
 *   experts_out, scores_out  [T, top_k] int32 / float32 or both NULL: the kept experts, best first
 *   workspace    dma_cdmoe_workspace_size(T, num_experts) bytes, zeroed once (status word first)
 */
DMA_API size_t dma_cdmoe_workspace_size(int T, int num_experts);
DMA_API dma_status_t dma_cdmoe_forward(const void* h, const void* W_router, const void* down_embed,
                                       const void* up_embed, int T, int hidden, int num_experts, int top_k,
                                       const float* logits_in, void* out, int32_t* experts_out, float* scores_out,
                                       void* workspace, size_t ws_bytes, dma_stream_t stream);

/*
 * Incremental decode with cached dt.  dt is one linear projection per cached
 * token followed by exp(A * softplus(.)) ([DMA step 3]), so a token's dt never
 * changes once it is cached: this pair of calls keeps dt and each (b, g)'s
 * kept set in a caller-owned decode state and, per step, takes in only the
 * tokens cached since the previous step (compute their dt; append while fewer
 * than keep_window_size keys are kept, else replace the worst kept key when
 * the new one ranks higher).  The output of a step equals dma_decode_step's
 * for the same caches and lengths; the per-step cost no longer includes the
 * scan of the whole value cache.
 *
 *   dma_decode_state_size  bytes of a decode state for this geometry (0 when
 *                          unsupported, as dma_workspace_size).
 *   dma_decode_state_init  dt over every cached token (lengths[b] of them) and
 *                          the full top-keep_window_size selection; clears the
 *                          state's status word.  The state (16-byte aligned
 *                          device memory, state_bytes >= the size above)
 *                          then belongs to these calls until the caller frees
 *                          it; dma_check(state) reports its status word.
 *   dma_decode_step_cached  one decode step: lengths[b] may grow by any number
 *                          of tokens since the previous call (the new tokens'
 *                          K and V already in the caches); a length outside
 *                          [1, Lk] or below the previous one is reported as
 *                          DMA_ERR_BAD_LENGTH through dma_check and that
 *                          sequence's state is left unchanged.  Arguments
 *                          as dma_decode_step.  Calls on one state must be
 *                          ordered (one stream).
 */
DMA_API size_t dma_decode_state_size(int B, int Lk, int Hq, int Hkv, int d, int keep_window_size);
DMA_API dma_status_t dma_decode_state_init(const void* v_cache, const float* W_dt, const float* A,
                                           const int32_t* lengths, int B, int Lk, int Hq, int Hkv, int d,
                                           int keep_window_size, void* state, size_t state_bytes,
                                           dma_stream_t stream);
DMA_API dma_status_t dma_decode_step_cached(const void* q, const void* k_cache, const void* v_cache,
                                            const float* W_dt, const float* A, const int32_t* lengths, int B,
                                            int Lk, int Hq, int Hkv, int d, int keep_window_size, float scale,
                                            void* out, void* state, size_t state_bytes, dma_stream_t stream);

/*
 * dma_decode_step without a caller-provided workspace (the pages have no
 * counterpart: this is a calling convention of this library).
 *
 * For callers that cannot allocate device memory themselves, for example code
 * embedded in a framework that owns all device memory through its own pool
 * and forbids raw cudaMalloc (which synchronises the device and fragments that
 * pool), or plain C callers without a device allocator.  Inputs and outputs are
 * still the caller's (same arguments and layouts as dma_decode_step); the
 * scratch lives in a 64 MiB array inside this library's device memory, which
 * every GPU that loads the library holds until the process exits.  This entry
 * point calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Returns DMA_ERR_WORKSPACE when the step needs more than 64 MiB of scratch,
 *     i.e. when dma_workspace_size(B, 1, Lk, Hq, Hkv, d, keep_window_size)
 *     exceeds 64 MiB (roughly B * Hkv * Lk above 15.7 million cached keys).
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress, with the device current); make that first
 *     call before any stream capture.  The address is cached per device and
 *     context: after the device's context is destroyed and made anew
 *     (cudaDeviceReset), the next call looks it up again, and that call too
 *     belongs before any stream capture.
 *   - Arguments are checked exactly as dma_decode_step checks them before
 *     anything is enqueued; a rejected call enqueues nothing.
 *   - Every call on every stream shares the one array and it keeps the last
 *     call's contents; calls that overlap on the GPU race, so serialise them
 *     (one stream, or events).  The status word is cleared at the start of
 *     each call; device-side faults are not reported back by this entry point
 *     (lengths are still clamped), so use dma_decode_step with a workspace and
 *     dma_check when you need that report.
 */
DMA_API dma_status_t dma_decode_step_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                             const float* W_dt, const float* A, const int32_t* lengths, int B, int Lk,
                                             int Hq, int Hkv, int d, int keep_window_size, float scale,
                                             const float* dt_in, void* out, dma_stream_t stream);

/*
 * Synchronises `stream`, then returns the status recorded in the workspace by
 * the device (DMA_OK if none).  clear != 0 resets the word afterwards.
 */
DMA_API dma_status_t dma_check(void* workspace, int clear, dma_stream_t stream);

/*
 * Profiling aid.  events: caller-owned cudaEvent_t handles (created with
 * timing enabled), n >= 4, or NULL to stop.  While set, on the calling host
 * thread, dma_forward_prefill and dma_decode_step record events[0] before
 * their first kernel, events[1] after S1 (dt), events[2] after S2 (selection)
 * and events[3] after the attention, all on the call's stream.  The library
 * keeps only the pointer; the caller keeps the array alive while it is set.
 */
DMA_API dma_status_t dma_set_stage_events(void* const* events, int n);

/*
 * Diagnostic (no counterpart on the pages): exercises the bounded-wait path
 * every kernel of this library uses.  One device thread waits on a barrier
 * that nothing completes; after the library's wait limit (about one second)
 * it gives up and records a timeout in the workspace's status word, which
 * dma_check() then reports as DMA_ERR_TIMEOUT.  workspace: at least 256
 * bytes, 16-byte aligned, zeroed before use.  Nothing faults or hangs.
 */
DMA_API dma_status_t dma_selftest_wait(void* workspace, dma_stream_t stream);

/* Human-readable name of a status. Never NULL. */
DMA_API const char* dma_status_string(dma_status_t status);

/* The cudaError_t of the last DMA_ERR_CUDA returned on this thread (0 if none). */
DMA_API int dma_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DMA_H_ */
