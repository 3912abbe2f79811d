"""The decode attention's split-K procedure, checked on the CPU.

The decode step attends one query to its kept keys (page "Transformers 中的
Doge 小语言模型完全指南", section "动态掩码注意力（DMA）：从缓存 value states
生成稀疏掩码", step 4: scale * q.k + dt, float32 softmax, times V).  The kernel
splits the kept list into 128-key chunks.  Each chunk writes an
unnormalised partial: o = sum 2^(x - m) v, its maximum m and sum l, with
x = log2(e) * (scale q.k + dt) and padding entries at -inf.  A second kernel
merges the partials with weights 2^(m - M), M the largest m, and writes
bf16(sum w o / sum w l).  This test restates that procedure in float32 and
compares it with float64 softmax attention.  A planted mistake (partials
merged without their weights) must fail the same bars.
"""
import numpy as np

LOG2E = 1.4426950408889634
CHUNK = 128


def bf16(x):
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16
    return b.astype(np.uint32).view(np.float32)


def partials(s, v):
    out = []
    for c0 in range(0, len(s), CHUNK):
        x = (s[c0:c0 + CHUNK] * LOG2E).astype(np.float32)
        m = np.float32(x.max())
        p = np.zeros_like(x) if m == -np.inf else np.exp2((x - m).astype(np.float64)).astype(np.float32)
        out.append(((p[:, None] * v[c0:c0 + CHUNK]).sum(axis=0, dtype=np.float32), m, p.sum(dtype=np.float32)))
    return out


def combine(parts, weighted=True):
    M = max(m for _, m, _ in parts)
    num = np.zeros_like(parts[0][0])
    den = np.float32(0.0)
    for o, m, l in parts:
        if m == -np.inf:
            continue
        wgt = np.float32(np.exp2(np.float64(m) - np.float64(M))) if weighted else np.float32(1.0)
        num = (num + wgt * o).astype(np.float32)
        den = np.float32(den + wgt * l)
    return bf16(num / den)


def reference(s, v):
    s = np.asarray(s, np.float64)
    e = np.exp(s - s[np.isfinite(s)].max())
    e[~np.isfinite(s)] = 0.0
    return (e / e.sum()) @ v.astype(np.float64)


def _case(rng, n, pad, spread):
    v = bf16(rng.standard_normal((n + pad, 128)).astype(np.float32))
    s = (rng.normal(0.0, 1.0, n + pad) * spread).astype(np.float32)
    s[n:] = -np.inf                     # list padding up to the chunk multiple
    return s, v


def test_split_partials_merge_to_float64_attention():
    rng = np.random.default_rng(31)
    worst, means = 0.0, []
    for n in (1, 5, 127, 128, 129, 1000, 2048):
        pad = (-n) % CHUNK
        for spread in (0.5, 3.0, 12.0):
            s, v = _case(rng, n, pad, spread)
            err = np.abs(combine(partials(s, v)).astype(np.float64) - reference(s, v))
            worst = max(worst, float(err.max()))
            means.append(float(err.mean()))
    assert worst <= 2e-2 and np.mean(means) <= 2e-3, (worst, np.mean(means))


def test_partials_merged_without_weights_are_caught():
    rng = np.random.default_rng(32)
    s, v = _case(rng, 2048, 0, 3.0)
    s[:CHUNK] += 6.0   # one chunk far above the others
    want = reference(s, v)
    assert np.abs(combine(partials(s, v)) - want).max() <= 2e-2
    assert np.abs(combine(partials(s, v), weighted=False) - want).max() > 2e-2
