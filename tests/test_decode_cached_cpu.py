"""Pins for the incremental decode (cached dt), on the oracle alone.

The cached-dt decode rests on two facts, both checked here against the
oracle's own definitions:

1. dt of a cached token depends on that token's value states only (page
   "Transformers 中的 Doge 小语言模型完全指南", section "动态掩码注意力（DMA）：从缓存
   value states 生成稀疏掩码", step 3: one linear projection per token, then
   exp(A * softplus(.))), so dt over a prefix of the cache equals the prefix
   of dt over the whole cache (up to float64 rounding of the matrix product),
   and changing other tokens leaves a token's dt unchanged;
2. the decode query's kept set over a growing cache (top keep_window_size
   by dt, ties to the lower index) is obtained by inserting each new key and
   evicting the current worst when the new key ranks higher: checked against
   the oracle's full selection at every length, on rows with forced ties.
"""
import numpy as np

from oracle import dma_oracle as oracle


def test_dt_of_a_token_ignores_the_rest_of_the_cache():
    rng = np.random.default_rng(5)
    B, L, Hkv, d = 2, 37, 3, 8
    v = rng.standard_normal((B, L, Hkv, d))
    W = rng.normal(0.0, 0.3, size=(Hkv * d, Hkv))
    A = rng.uniform(-2.0, -0.1, size=Hkv)
    full = oracle.dt_scores64(v, W, A)
    # equal up to the last bits of the float64 matrix product (its blocking
    # depends on the matrix size)
    for n in (1, 5, 36):
        np.testing.assert_allclose(oracle.dt_scores64(v[:, :n], W, A), full[..., :n], rtol=1e-13, atol=0)
    # changing every other token leaves token j's dt unchanged
    j = 11
    v2 = rng.standard_normal(v.shape)
    v2[:, j] = v[:, j]
    np.testing.assert_allclose(oracle.dt_scores64(v2, W, A)[..., j], full[..., j], rtol=1e-13, atol=0)
    assert not np.allclose(oracle.dt_scores64(v2, W, A)[..., j + 1], full[..., j + 1])


def _incremental_kept(dt_row, w):
    """Kept set after each length 1..len(dt_row), by insert / evict-the-worst."""
    kept = []
    out = []
    for j in range(len(dt_row)):
        ck = oracle.composite_key(dt_row[j], j)
        if len(kept) < w:
            kept.append((ck, j))
        else:
            worst = min(kept)
            if ck > worst[0]:
                kept.remove(worst)
                kept.append((ck, j))
        out.append(sorted(j for _, j in kept))
    return out


def test_insert_and_evict_equals_full_selection_at_every_length():
    rng = np.random.default_rng(9)
    for trial in range(40):
        Lk = int(rng.integers(1, 60))
        w = int(rng.integers(1, 20))
        if trial % 3 == 0:   # forced ties
            dt_row = rng.choice(np.array([0.25, 0.5, 0.75, 1.0], np.float32), size=Lk)
        else:
            dt_row = rng.uniform(0.01, 1.0, size=Lk).astype(np.float32)
        inc = _incremental_kept(dt_row, w)
        for n in range(1, Lk + 1):
            m = oracle.kept_mask(dt_row[None, None, :], np.array([n]), 1, Lk, w)[0, 0, 0]
            assert sorted(np.nonzero(m)[0].tolist()) == inc[n - 1], (trial, n)


def test_evicted_keys_never_return():
    # the structure the update relies on: the kept set at length n+1 lies in
    # the kept set at length n plus the new key
    rng = np.random.default_rng(13)
    dt_row = rng.uniform(0.0, 1.0, size=80).astype(np.float32)
    w = 7
    prev = None
    for n in range(1, 81):
        kept = set(np.nonzero(oracle.kept_mask(dt_row[None, None, :], np.array([n]), 1, 80, w)[0, 0, 0])[0])
        if prev is not None:
            assert kept <= prev | {n - 1}
        prev = kept
