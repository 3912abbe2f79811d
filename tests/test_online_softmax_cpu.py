"""The prefill attention's softmax procedure, checked on the CPU.

Page "Transformers 中的 Doge 小语言模型完全指南", section
"动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", step 4: softmax in float32
over scale * q.k + dt, masked keys weighted 0, times V.  The attention kernel
computes it tile by tile (128 keys) with a lazily rescaled running maximum:
  - the maximum m (log2 units) moves only when a tile's maximum exceeds it by
    more than 2^8, and O and the running sum l are then scaled by 2^(m_old - m);
  - p = 2^(x - m) with x = log2(e) * (scale q.k + dt), so p may reach 2^8;
  - l sums the float32 p, P = bf16(p) enters the float32 accumulation of
    P V, and the output is O / l rounded to bf16.
This test restates that procedure in numpy (float32, explicit bf16 rounding)
and compares it with the float64 softmax attention.  Score patterns force
rescales, drifts just under the threshold, large dynamic ranges, and
leading tiles that are entirely masked.
"""
import numpy as np

LOG2E = 1.4426950408889634
THRESHOLD = 8.0
TILE = 128


def bf16(x):
    """Round float32 values to bfloat16 (nearest even), returned as float32."""
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16
    return b.astype(np.uint32).view(np.float32)


def kernel_row(s_row, v):
    """One query row: s_row = scale * q.k + dt per key (-inf where masked),
    v [keys, d] bf16-exact values.  Returns the bf16 output row."""
    m = np.float32(-np.inf)
    l = np.float32(0.0)
    o = np.zeros(v.shape[1], np.float32)
    for t0 in range(0, len(s_row), TILE):
        x = (s_row[t0:t0 + TILE] * LOG2E).astype(np.float32)
        tmax = np.float32(x.max())
        m_new = max(m, tmax)
        with np.errstate(invalid="ignore"):
            grows = (m_new - m) > THRESHOLD   # False while both are -inf
        if grows:
            alpha = np.float32(np.exp2(np.float64(m) - np.float64(m_new)))
            m = m_new
            l = np.float32(l * alpha)
            o = (o * alpha).astype(np.float32)
        nm = np.float32(0.0) if m == -np.inf else -m
        p = np.exp2((x + nm).astype(np.float64)).astype(np.float32)
        l = np.float32(l + p.sum(dtype=np.float32))
        o = (o + (bf16(p)[:, None] * v[t0:t0 + TILE]).sum(axis=0, dtype=np.float32)).astype(np.float32)
    return bf16(o / l)


def reference_row(s_row, v):
    s = np.asarray(s_row, np.float64)
    e = np.exp(s - s[np.isfinite(s)].max())
    e[~np.isfinite(s)] = 0.0
    return (e / e.sum()) @ v.astype(np.float64)


def _case(rng, n_keys, d, pattern):
    v = bf16(rng.standard_normal((n_keys, d)).astype(np.float32))
    s = rng.normal(0.0, 2.0, n_keys)
    n_tiles = (n_keys + TILE - 1) // TILE
    if pattern == "rising":          # each tile's maximum far above the last: a rescale per tile
        s += np.repeat(np.arange(n_tiles) * 9.0, TILE)[:n_keys]
    elif pattern == "drift":         # just under the threshold per tile, so m stays stale
        s += np.repeat(np.arange(n_tiles) * 5.0, TILE)[:n_keys]
    elif pattern == "wide":          # a wide dynamic range inside one row
        s *= 8.0
    elif pattern == "masked_head":   # the first tiles see no key at all
        s[: min(n_keys - 1, 2 * TILE)] = -np.inf
    elif pattern == "sparse":        # scattered masked keys
        s[rng.random(n_keys) < 0.6] = -np.inf
        s[rng.integers(0, n_keys)] = 0.0
    return s.astype(np.float32), v


def test_lazy_rescaled_softmax_matches_float64_attention():
    rng = np.random.default_rng(11)
    worst_max, errs = 0.0, []
    for pattern in ("plain", "rising", "drift", "wide", "masked_head", "sparse"):
        for n_keys in (1, 100, 128, 300, 1024):
            s, v = _case(rng, n_keys, 64, pattern)
            got = kernel_row(s, v)
            want = reference_row(s, v)
            err = np.abs(got.astype(np.float64) - want)
            worst_max = max(worst_max, float(err.max()))
            errs.append(float(err.mean()))
    # the same bars as every GPU parity test
    assert worst_max <= 2e-2, worst_max
    assert np.mean(errs) <= 2e-3, np.mean(errs)


def test_a_rescale_that_forgets_the_sum_is_caught():
    """The procedure with l left unscaled on a rescale fails the bars on a row
    whose first tile keeps real weight after the rescale: 128 keys at x = 0,
    then one key 9 log2 units higher (the rest of its tile masked)."""
    rng = np.random.default_rng(12)
    v = bf16(rng.standard_normal((2 * TILE, 64)).astype(np.float32))
    s = np.full(2 * TILE, -np.inf, np.float32)
    s[:TILE] = 0.0
    s[TILE] = np.float32(9.0 / LOG2E)

    def broken(s_row, vv):
        m, l, o = np.float32(-np.inf), np.float32(0.0), np.zeros(vv.shape[1], np.float32)
        for t0 in range(0, len(s_row), TILE):
            x = (s_row[t0:t0 + TILE] * LOG2E).astype(np.float32)
            m_new = max(m, np.float32(x.max()))
            with np.errstate(invalid="ignore"):
                if (m_new - m) > THRESHOLD:
                    alpha = np.float32(np.exp2(np.float64(m) - np.float64(m_new)))
                    m = m_new
                    o = (o * alpha).astype(np.float32)      # l is not scaled: the planted mistake
            p = np.exp2((x - m).astype(np.float64)).astype(np.float32)
            l = np.float32(l + p.sum(dtype=np.float32))
            o = (o + (bf16(p)[:, None] * vv[t0:t0 + TILE]).sum(axis=0, dtype=np.float32)).astype(np.float32)
        return bf16(o / l)

    want = reference_row(s, v)
    assert np.abs(kernel_row(s, v) - want).max() <= 2e-2
    assert np.abs(broken(s, v) - want).max() > 2e-2
