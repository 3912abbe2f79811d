"""CPU oracle for Doge's Dynamic Mask Attention (DMA) hot path.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its Python binding) never calls it, and this module imports
nothing from the product package.

Everything here is a plain, slow, obviously-correct restatement of what the
pages define, computed in numpy float64 (except where noted: the per-key score
is handed on as float32, which is the precision the kernels and the dynamic
mask use).  There is no blocking, fusion or reordering beyond what the
definitions state.

Source cited throughout (the only page that defines DMA):
  "Transformers 中的 Doge 小语言模型完全指南：动态掩码注意力（DMA）与跨域 MoE（CDMoE）
   架构解析与实战" (blog.gitcode.com), written below as [Guide].
  [Guide §DMA.3]  section "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码",
                  forward chain step 3 (dt_proj, exp(A*softplus), prepare_dynamic_mask,
                  top-k + scatter above keep_window_size).
  [Guide §DMA.4]  same section, step 4 (scores scaled by head_dim**-0.5, fp32 softmax,
                  additive attn_mask).
  [Guide §DMA.init] same section, closing paragraph (A initialised with zeros).
  [Guide §Config] section "DogeConfig 全参数详解" (num_key_value_heads, attention_bias=False,
                  keep_window_size=2048, sliding_window=None -> full causal mask).

Readings taken where the pages are silent:
  * dt_proj input is the per-token value row flattened head-major
    (index h'*d + e) and projected to H_kv outputs; no bias (attention_bias=False).
  * causal and padding masking are merged into the mask BEFORE the top-k, so a
    row keeps the keep_window_size best keys among the keys it may see.
  * ties in the top-k go to the lower key index.
  * "exceeds keep_window_size" is strict: Lk > w triggers the top-k.
  * the dt bias is added after scaling: s = scale * q.k + dt.
  * GQA: query head h reads kv head g = h // (H_q / H_kv).
  * min_dtype is bf16's lowest finite value.
  * padded query rows (i >= len_b) are computed with the same formula.
  * the decode query sits at position len_b - 1 and the cache holds it.

Parity status of each function (pins live in tests/test_oracle_pins.py):
  softplus, dt_scores            pinned (closed forms, worked example, flatten-order probe)
  dynamic_mask_rows, kept_mask   pinned (brute-force rank count, closed forms, invariants,
                                  torch.topk on tie-free rows)
  thresholds                     pinned (rebuilds kept_mask exactly)
  attention_rows, prefill        pinned (float64 SDPA, closed forms)
  prefill_rows                   pinned (float64 SDPA with a brute-force rank-count mask,
                                  n_rep 1-3, padding, ties, scattered rows)
  decode_step                    pinned (float64 SDPA, closed forms)
  rms_norm                       pinned (hand example, unit mean square, scale invariance)
  rope_angles, rope              pinned (2-D closed form, complex-number form, relative
                                  position, composition, identity at position 0)
  prologue                       pinned (pair lengths show norm-then-rotate, position 0 is
                                  the plain norm, relative-position invariance under a
                                  shifted offset, untouched cache rows, V appended as is)
  cdmoe_logits                   pinned (float64 matmul against explicit index loops)
  cdmoe_route                    pinned (brute force over all K*K experts on tie-free logits,
                                  closed form on constant logits, torch.topk per domain)
  prefill_backward               pinned (float64 torch.autograd of an independent forward,
                                  central finite differences, planted mistakes)
  cdmoe_experts, cdmoe           pinned (one expert = silu(h.d) u, equal scores = plain mean,
                                  linearity in up_embed, a hand-worked two-expert example)
"""
from __future__ import annotations

import numpy as np

# bf16's lowest finite value, exactly representable in float32 and float64.
MIN_DTYPE = -3.3895313892515355e38


# --------------------------------------------------------------------------
# S1: per-key score  dt = exp(A * softplus(dt_proj(value_states)))   [Guide §DMA.3]
# --------------------------------------------------------------------------

def softplus(x):
    """softplus(x) = log(1 + exp(x)), written in the overflow-free form
    max(x, 0) + log1p(exp(-|x|)) (same value, float64)."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def dt_scores64(v, W, A):
    """Float64 per-key score [Guide §DMA.3].

    v : [B, L, H_kv, d] value states (any float dtype; bf16 values pass exactly)
    W : [H_kv*d, H_kv] dt_proj weight, input-major (x = v_flat @ W), no bias
    A : [H_kv] one learnable scalar per kv head
    returns dt64 [B, H_kv, L] float64
    """
    v = np.asarray(v, dtype=np.float64)
    B, L, Hkv, d = v.shape
    W = np.asarray(W, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    assert W.shape == (Hkv * d, Hkv) and A.shape == (Hkv,)
    v_flat = v.reshape(B, L, Hkv * d)            # head-major: column h'*d + e
    x = v_flat @ W                               # [B, L, H_kv]   dt_proj(value_states)
    dt = np.exp(A[None, None, :] * softplus(x))  # exp(A * softplus(.))
    return np.ascontiguousarray(dt.transpose(0, 2, 1))


def dt_scores(v, W, A):
    """dt rounded to float32, the precision the mask is built in: [B, H_kv, L]."""
    return dt_scores64(v, W, A).astype(np.float32)


# --------------------------------------------------------------------------
# S2: dynamic mask   [Guide §DMA.3, prepare_dynamic_mask]
# --------------------------------------------------------------------------

def _valid_limit(row, len_b, Lq, Lk):
    """Number of leading keys row `row` may see: causal (query position
    row + Lk - Lq, so prefill row i sees keys <= i) and padding (keys >= len_b
    are never seen).  For decode (Lq == 1) this is len_b: the query sits at
    position len_b - 1 and sees every valid cached key."""
    return min(row + (Lk - Lq) + 1, len_b)


def dynamic_mask_rows(dt_row, len_b, Lq, Lk, w, rows):
    """Additive mask rows for one (batch, kv head) [Guide §DMA.3].

    dt_row : [Lk] float32 per-key score of this kv head
    rows   : iterable of query rows
    Each mask row starts as dt broadcast over the query rows; keys the row may
    not see (causal or padding) are set to MIN_DTYPE; then, when Lk exceeds w,
    only the w largest entries of the row are kept (ties: lower key index first,
    a stable sort of the negated row) and every other entry becomes MIN_DTYPE.
    returns float64 [len(rows), Lk]
    """
    dt_row = np.asarray(dt_row, dtype=np.float32).astype(np.float64)
    rows = list(rows)
    out = np.full((len(rows), Lk), MIN_DTYPE, dtype=np.float64)
    for r, i in enumerate(rows):
        lim = _valid_limit(i, len_b, Lq, Lk)
        m = np.full(Lk, MIN_DTYPE, dtype=np.float64)
        m[:lim] = dt_row[:lim]
        if Lk > w:
            order = np.argsort(-m, kind="stable")
            keep = np.zeros(Lk, dtype=bool)
            keep[order[:w]] = True
            m[~keep] = MIN_DTYPE
        out[r] = m
    return out


def kept_mask(dt, lengths, Lq, Lk, w):
    """Boolean kept-key mask [B, H_kv, Lq, Lk] (small shapes only)."""
    dt = np.asarray(dt, dtype=np.float32)
    B, Hkv, _ = dt.shape
    out = np.zeros((B, Hkv, Lq, Lk), dtype=bool)
    for b in range(B):
        for g in range(Hkv):
            m = dynamic_mask_rows(dt[b, g], int(lengths[b]), Lq, Lk, w, range(Lq))
            out[b, g] = m > MIN_DTYPE
    return out


def composite_key(dt_value, j):
    """Total order used for the top-k: float32 bits of dt in the high word
    (dt >= 0, so its bit pattern orders like the value), 0xFFFFFFFF - j in the
    low word (so the lower index ranks higher on equal dt)."""
    bits = int(np.asarray(dt_value, dtype=np.float32).view(np.uint32))
    return (bits << 32) | (0xFFFFFFFF - int(j))


def threshold_row(dt_row, len_b, Lq, Lk, w, i):
    """tau of one query row (see thresholds)."""
    lim = _valid_limit(i, len_b, Lq, Lk)
    if Lk > w and lim > w:
        order = np.argsort(-np.asarray(dt_row[:lim], dtype=np.float64), kind="stable")
        j = int(order[w - 1])
        return composite_key(dt_row[j], j)
    return 0


def thresholds(dt, lengths, Lq, Lk, w):
    """Row thresholds tau [B, H_kv, Lq] as uint64.

    tau = composite key of the w-th best visible key when Lk > w and the row
    sees more than w keys; else 0 (every visible key kept).  Key j is kept in a
    row iff it is visible and composite_key(dt[j], j) >= tau.
    """
    dt = np.asarray(dt, dtype=np.float32)
    B, Hkv, _ = dt.shape
    tau = np.zeros((B, Hkv, Lq), dtype=np.uint64)
    for b in range(B):
        for g in range(Hkv):
            for i in range(Lq):
                tau[b, g, i] = threshold_row(dt[b, g], int(lengths[b]), Lq, Lk, w, i)
    return tau


# --------------------------------------------------------------------------
# S3: attention with the additive mask   [Guide §DMA.4]
# --------------------------------------------------------------------------

def attention_rows(q_rows, K, V, mask_rows, scale):
    """softmax(scale * q K^T + mask) V for a block of query rows, float64.

    q_rows [n, d], K [Lk, d], V [Lk, d], mask_rows [n, Lk] -> [n, d]
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    s = scale * (q_rows @ K.T) + mask_rows
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V


def prefill_rows(q, k, v, dt, lengths, w, scale, b, h, rows):
    """Output rows of one (batch b, query head h) of the prefill path.

    q [B, L, H_q, d], k/v [B, L, H_kv, d], dt [B, H_kv, L] float32.
    """
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    g = h // (Hq // Hkv)                                   # GQA group [Guide §Config]
    rows = list(rows)
    M = dynamic_mask_rows(dt[b, g], int(lengths[b]), L, L, w, rows)
    return attention_rows(np.asarray(q[b, rows, h, :], dtype=np.float64),
                          k[b, :, g, :], v[b, :, g, :], M, scale)


def prefill(q, k, v, W, A, lengths, w, scale, dt=None, row_block=1024):
    """Whole prefill forward: dt (unless given) -> dynamic mask -> attention.

    Returns float64 [B, L, H_q, d].  dt, when given, is float32 [B, H_kv, L].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if dt is None:
        dt = dt_scores(v, W, A)
    dt = np.asarray(dt, dtype=np.float32)
    n_rep = Hq // Hkv
    out = np.empty((B, L, Hq, d), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            for r0 in range(0, L, row_block):
                rows = range(r0, min(L, r0 + row_block))
                M = dynamic_mask_rows(dt[b, g], int(lengths[b]), L, L, w, rows)
                for r in range(n_rep):
                    h = g * n_rep + r
                    out[b, r0:r0 + len(rows), h, :] = attention_rows(
                        q[b, r0:r0 + len(rows), h, :], k[b, :, g, :], v[b, :, g, :], M, scale)
    return out


# --------------------------------------------------------------------------
# S4: one decode step over a KV cache   [Guide §DMA.3 last paragraph, §DMA.4]
# --------------------------------------------------------------------------

def decode_step(q, k_cache, v_cache, W, A, lengths, w, scale, dt=None, batches=None):
    """One query per sequence against its cache.

    q [B, H_q, d]; k_cache / v_cache [B, Lk, H_kv, d]; the query sits at
    position len_b - 1 and the cache already holds it.  dt is computed over the
    whole cached value states (all Lk positions; positions >= len_b are masked).
    Returns float64 [len(batches), H_q, d] (all batches by default).
    """
    B, Hq, d = q.shape
    Lk, Hkv = k_cache.shape[1], k_cache.shape[2]
    n_rep = Hq // Hkv
    batches = range(B) if batches is None else list(batches)
    out = np.empty((len(batches), Hq, d), dtype=np.float64)
    for ob, b in enumerate(batches):
        vb = np.asarray(v_cache[b], dtype=np.float64)            # [Lk, H_kv, d]
        kb = np.asarray(k_cache[b], dtype=np.float64)
        if dt is None:
            dtb = dt_scores(vb[None], W, A)[0]                   # [H_kv, Lk] float32
        else:
            dtb = np.asarray(dt[b], dtype=np.float32)
        for g in range(Hkv):
            M = dynamic_mask_rows(dtb[g], int(lengths[b]), 1, Lk, w, [0])
            for r in range(n_rep):
                h = g * n_rep + r
                out[ob, h, :] = attention_rows(np.asarray(q[b, h][None, :], dtype=np.float64),
                                               kb[:, g, :], vb[:, g, :], M, scale)[0]
    return out


# --------------------------------------------------------------------------
# Prologue: q_norm / k_norm, rotary position embedding, KV-cache append
#   [Guide §DMA.1-2]  section "动态掩码注意力（DMA）", forward-chain steps 1 and 2:
#                     after q_proj/k_proj/v_proj, Q and K each pass an RMSNorm
#                     over head_dim (q_norm / k_norm), then the rotary position
#                     embedding (apply_rotary_pos_emb); with a cache, K and V
#                     are appended to it (past_key_values.update).
#   [Guide §Modules]  section "从源码理解两大核心模块": RMSNorm and RoPE are the
#                     Llama implementations; [Guide §Residual] DogeRMSNorm is the
#                     T5-style norm (learnable elementwise scale, variance in fp32).
#   [Guide §Config]   rms_norm_eps = 1e-6; rope_parameters (rope_theta) has no
#                     default on the page.
# Readings taken where the pages are silent:
#   * RMSNorm: y = w * x / sqrt(mean(x^2) + eps) over the d channels of one head.
#   * RoPE (the Llama convention): channel i < d/2 pairs with channel i + d/2;
#     the pair is rotated by the angle pos * theta^(-2i/d):
#       (a, b) -> (a cos - b sin, b cos + a sin).
#   * token t of sequence b sits at position positions[b] + t, and is written to
#     the cache row of that position.
#   * norm first, then rotation (the order of step 1); V is appended unchanged.
# --------------------------------------------------------------------------

def rms_norm(x, w, eps):
    """RMSNorm over the last axis, float64: w * x / sqrt(mean(x^2) + eps)."""
    x = np.asarray(x, dtype=np.float64)
    ms = (x * x).mean(axis=-1, keepdims=True)
    return np.asarray(w, dtype=np.float64) * (x / np.sqrt(ms + eps))


def rope_angles(pos, d, theta):
    """Rotation angles [len(pos), d/2]: pos * theta^(-2i/d), float64."""
    i = np.arange(d // 2, dtype=np.float64)
    inv_freq = np.power(float(theta), -2.0 * i / d)
    return np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]


def rope(x, pos, theta):
    """Rotary embedding of x [..., n, H, d] at positions pos [n] (Llama pairing)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = rope_angles(pos, d, theta)                   # [n, d/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a, b = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def prologue(q, k, v, q_norm_w, k_norm_w, eps, theta, positions, k_cache, v_cache):
    """Steps 1-2 of the attention forward for new tokens.

    q [B, L, H_q, d], k / v [B, L, H_kv, d] projected states; q_norm_w / k_norm_w [d];
    positions [B] cache offset of each sequence's first new token;
    k_cache / v_cache [B, Lmax, H_kv, d] (not modified).
    Returns (q_out [B, L, H_q, d], k_cache_out, v_cache_out) in float64, the
    caches with rows positions[b] .. positions[b] + L - 1 replaced.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, L = q.shape[:2]
    kc = np.array(k_cache, dtype=np.float64, copy=True)
    vc = np.array(v_cache, dtype=np.float64, copy=True)
    q_out = np.empty_like(q)
    for b in range(B):
        pos = int(positions[b]) + np.arange(L)
        q_out[b] = rope(rms_norm(q[b], q_norm_w, eps), pos, theta)
        kc[b, pos] = rope(rms_norm(k[b], k_norm_w, eps), pos, theta)
        vc[b, pos] = v[b]
    return q_out, kc, vc


# --------------------------------------------------------------------------
# CDMoE routing   [Guide §CDMoE]  section "跨域 MoE（CDMoE）：在稠密 checkpoint 上“叠加”稀疏专家"
#   router_gate maps the hidden state to num_keys * 2 logits; a top-k runs on
#   each of the two domains x and y (num_keys = floor(sqrt(num_experts)));
#   their Cartesian product gives the expert indices; the experts are rows of
#   two embedding tables (down_embed, up_embed [num_experts, hidden_size]):
#   looked up and applied to the hidden state as down-projection -> activation
#   -> up-projection, added to the shared expert's output.
#   [Guide §Config]  num_experts = 16384, num_experts_per_tok = 64 (the top-k),
#   hidden_act = "silu", mlp_bias = False, norm_topk_prob = False.
# Readings taken where the pages are silent:
#   * logits [T, 2K]: columns [0, K) are domain x, [K, 2K) domain y; no bias.
#   * each domain keeps its k = num_experts_per_tok best keys (ties: lower key
#     index); the product pair (a, b) scores s_x[a] + s_y[b] (float32 sum, the
#     precision the logits are handed on in) and names expert a * K + b; the
#     token keeps the k best of the k * k pairs (ties: lower expert index).
#   * routing weights: softmax over the k kept scores (norm_topk_prob = False
#     adds no further scaling).
#   * expert e contributes weight_e * silu(h . down_embed[e]) * up_embed[e].
# --------------------------------------------------------------------------

def cdmoe_logits(h, W_router):
    """router_gate: h [T, hidden] @ W_router [hidden, 2K], float64."""
    return np.asarray(h, dtype=np.float64) @ np.asarray(W_router, dtype=np.float64)


def _topk_stable(vals, k):
    """Indices of the k largest values, larger first, ties to the lower index."""
    order = np.argsort(-np.asarray(vals, dtype=np.float64), kind="stable")
    return order[:k]


def cdmoe_route(logits, k):
    """Expert indices [T, k] (int64) and scores [T, k] (float32) from float32
    router logits [T, 2K]: top-k per domain, then the k best of their product."""
    logits = np.asarray(logits, dtype=np.float32)
    T, twoK = logits.shape
    K = twoK // 2
    experts = np.empty((T, k), dtype=np.int64)
    scores = np.empty((T, k), dtype=np.float32)
    for t in range(T):
        lx, ly = logits[t, :K], logits[t, K:]
        ix = _topk_stable(lx, k)
        iy = _topk_stable(ly, k)
        cand_s = (lx[ix][:, None] + ly[iy][None, :]).astype(np.float32).ravel()   # float32 sums
        cand_e = (ix[:, None] * K + iy[None, :]).ravel()
        # best score first; equal scores: lower expert index first
        order = np.lexsort((cand_e, -cand_s.astype(np.float64)))[:k]
        experts[t] = cand_e[order]
        scores[t] = cand_s[order]
    return experts, scores


def cdmoe_experts(h, experts, scores, down_embed, up_embed):
    """Routed output [T, hidden], float64: sum over the kept experts of
    softmax(scores)_e * silu(h . down_embed[e]) * up_embed[e]."""
    h = np.asarray(h, dtype=np.float64)
    D = np.asarray(down_embed, dtype=np.float64)
    U = np.asarray(up_embed, dtype=np.float64)
    out = np.empty_like(h)
    for t in range(h.shape[0]):
        s = np.asarray(scores[t], dtype=np.float64)
        wts = np.exp(s - s.max())
        wts = wts / wts.sum()
        a = D[experts[t]] @ h[t]                  # down-projection: one scalar per expert
        act = a / (1.0 + np.exp(-a))              # silu
        out[t] = (wts * act) @ U[experts[t]]      # up-projection
    return out


def cdmoe(h, W_router, down_embed, up_embed, k, logits=None):
    """Routed CDMoE output [T, hidden] (float64), experts [T, k], scores [T, k].
    logits, when given, are the float32 router logits [T, 2K] to route on."""
    if logits is None:
        logits = cdmoe_logits(h, W_router).astype(np.float32)
    experts, scores = cdmoe_route(logits, k)
    return cdmoe_experts(h, experts, scores, down_embed, up_embed), experts, scores


# --------------------------------------------------------------------------
# Backward of the prefill path, the kept-key selection held fixed
#   [Guide §DMA.3] the closing paragraph: dt comes from the cached value
#   states, so the training stage learns end to end which history tokens to
#   mask; [Guide] the architecture list's item 1 (training uses self-attention
#   tied to the value states).
# Readings taken where the pages are silent:
#   * the top-k is a selection, not a function with a gradient: the kept set
#     of every row is held fixed, and gradients flow through the dt values of
#     the kept keys (masked entries are constants);
#   * the float32 rounding of dt for the mask passes gradients unchanged.
# For L = sum(out * dout):
#   dP = dO V^T, D_i = dO_i . O_i, dS = P (dP - D), dQ = scale dS K,
#   dK = scale dS^T Q, dV = P^T dO (+ the dt path below),
#   d_dt[g, j] = sum over the group's heads and rows of dS[., j];
#   dt = exp(A softplus(x)):  dA = sum d_dt dt softplus(x),
#   dx = d_dt dt A sigmoid(x),  dW = v_flat^T dx,  dV_flat += dx W^T.
# --------------------------------------------------------------------------

def prefill_backward(q, k, v, W, A, lengths, w, scale, dout, dt_fixed=None):
    """Gradients of sum(prefill(...) * dout), float64.

    Returns dq [B,L,Hq,d], dk [B,L,Hkv,d], dv [B,L,Hkv,d] (attention and dt
    paths), d_dt [B,Hkv,L], dW [Hkv*d, Hkv], dA [Hkv].  dt_fixed, when given,
    is the float32 dt the mask is built from (the kernels' own dt): the
    selection and bias use it, while the dt chain still starts from W and A.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    n_rep = Hq // Hkv
    # forward quantities of the dt chain  [Guide §DMA.3]
    x = v.reshape(B, L, Hkv * d) @ W                       # [B, L, Hkv]
    sp = softplus(x)
    dt64 = np.exp(A[None, None, :] * sp)                   # [B, L, Hkv]
    dt32 = dt64.transpose(0, 2, 1).astype(np.float32) if dt_fixed is None else np.asarray(dt_fixed, np.float32)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    d_dt = np.zeros((B, Hkv, L))
    for b in range(B):
        for g in range(Hkv):
            M = dynamic_mask_rows(dt32[b, g], int(lengths[b]), L, L, w, range(L))    # [L, L]
            Kg, Vg = k[b, :, g, :], v[b, :, g, :]
            for r in range(n_rep):
                h = g * n_rep + r
                Q, dO = q[b, :, h, :], dout[b, :, h, :]
                s = scale * (Q @ Kg.T) + M
                s = s - s.max(axis=1, keepdims=True)
                P = np.exp(s)
                P = P / P.sum(axis=1, keepdims=True)
                O = P @ Vg
                dP = dO @ Vg.T
                Dr = (dO * O).sum(axis=1, keepdims=True)
                dS = P * (dP - Dr)
                dq[b, :, h, :] = scale * (dS @ Kg)
                dk[b, :, g, :] += scale * (dS.T @ Q)
                dv[b, :, g, :] += P.T @ dO
                d_dt[b, g, :] += dS.sum(axis=0)
    ddt = d_dt.transpose(0, 2, 1)                          # [B, L, Hkv]
    dA = (ddt * dt64 * sp).sum(axis=(0, 1))
    sig = 1.0 / (1.0 + np.exp(-x))
    dx = ddt * dt64 * A[None, None, :] * sig               # [B, L, Hkv]
    v_flat = v.reshape(B * L, Hkv * d)
    dW = v_flat.T @ dx.reshape(B * L, Hkv)
    dv += (dx.reshape(B * L, Hkv) @ W.T).reshape(B, L, Hkv, d)
    return dq, dk, dv, d_dt, dW, dA
