"""The three-term bf16 split used by the tensor-core paths, checked on the CPU.

Two kernels feed float32 operands through bf16 tensor-core inputs by
splitting each value c into hi = bf16(c), mid = bf16(c - hi) and
lo = bf16(c - hi - mid), all roundings to nearest even:
  - the attention kernel's dt bias: c = dt / scale in three extra key columns,
    each multiplied by 1 from the query's extra columns, so the float32
    accumulation adds hi + mid + lo to scale^-1 * (scale q.k), and scale * S =
    scale q.k + dt (page "Transformers 中的 Doge 小语言模型完全指南", section
    "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", step 4);
  - the dt kernel's weights: W = W_hi + W_mid + W_lo in three column groups,
    each a bf16 x bf16 product accumulated in float32 (same section, step 3).
For those products and sums to reproduce float32 arithmetic, the three terms
must add back to c exactly: 8 + 8 + 8 significant bits cover float32's 24.
This test restates the split and checks exact reconstruction over the ranges
the kernels see, plus float32 edge values.
"""
import numpy as np


def bf16(x):
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16
    return b.astype(np.uint32).view(np.float32)


def split3(c):
    c = np.asarray(c, np.float32)
    hi = bf16(c)
    r1 = (c - hi).astype(np.float32)
    mid = bf16(r1)
    lo = bf16((r1 - mid).astype(np.float32))
    return hi, mid, lo


def _reconstruct(hi, mid, lo):
    # the tensor core multiplies each term by 1 exactly and accumulates in
    # float32; with non-overlapping terms every partial sum is exact
    return ((hi.astype(np.float32) + mid) + lo).astype(np.float32)


def test_bias_split_is_exact_over_dt_over_scale():
    rng = np.random.default_rng(3)
    for d in (64, 128):
        scale = np.float32(d ** -0.5)
        dt = np.concatenate([rng.uniform(0.0, 1.0, 200_000), rng.uniform(1e-30, 1e-3, 20_000),
                             np.array([0.0, 1.0, np.float32(0.5) ** 20])]).astype(np.float32)
        c = (dt / scale).astype(np.float32)
        hi, mid, lo = split3(c)
        assert np.array_equal(_reconstruct(hi, mid, lo), c)


def test_weight_split_is_exact_over_normal_weights():
    rng = np.random.default_rng(4)
    w = np.concatenate([rng.normal(0.0, 0.02, 300_000), rng.normal(0.0, 3.0, 50_000),
                        np.array([0.0, -0.0, 1e-20, -1e-20, 1e20, np.float32(np.finfo(np.float32).max) / 4])])
    w = w.astype(np.float32)
    hi, mid, lo = split3(w)
    assert np.array_equal(_reconstruct(hi, mid, lo), w)
    # and the terms shrink: each is at most 2^-8 of the one before (bf16 keeps 8 significant bits)
    nz = hi != 0
    assert np.all(np.abs(mid[nz]) <= np.abs(hi[nz]) * 2.0 ** -8)


def test_two_terms_would_not_be_enough():
    # a plausible shortcut (hi + mid only) loses float32 bits: the split needs three terms
    rng = np.random.default_rng(5)
    c = rng.uniform(0.0, 11.4, 10_000).astype(np.float32)
    hi, mid, _ = split3(c)
    two = (hi + mid).astype(np.float32)
    assert np.count_nonzero(two != c) > 1000
