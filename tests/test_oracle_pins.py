"""Pins for the CPU oracle: each checks it against something other than itself
(closed forms, a hand-worked example, brute force on tiny inputs, invariants
the method implies, and float64 library routines).

Cited page: "Transformers 中的 Doge 小语言模型完全指南" ([Guide]); sections as in
the oracle's header.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import MIN_DTYPE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# reusable pin checks (they take the oracle functions as arguments, so
# test_oracle_mutations.py can show that planted mistakes fail them)
# ----------------------------------------------------------------------------

def check_dt_worked_example(dt_scores64):
    """Hand-worked example from tests/golden/dt_worked_example.txt [Guide §DMA.3]."""
    v = np.zeros((1, 2, 2, 2))
    v[0, 0, 0, 0] = 1.0
    v[0, 0, 1, 1] = 2.0
    W = np.zeros((4, 2))
    W[0, 0] = 0.5
    W[3, 0] = 0.25
    A = np.array([-1.0, -2.0])
    dt = dt_scores64(v, W, A)
    rows = [l.split() for l in open(os.path.join(GOLDEN, "dt_worked_example.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 4
    for g, t, val in rows:
        assert dt[0, int(g), int(t)] == pytest.approx(float(val), rel=1e-15, abs=0)


def check_dt_sigmoid_closed_form(dt_scores64, seed=0):
    """A = -1  =>  dt = exp(-log(1+e^x)) = 1/(1+e^x);  A = -2  =>  its square.
    x is formed by explicit index arithmetic over (head, channel)."""
    rng = np.random.default_rng(seed)
    B, L, Hkv, d = 2, 5, 2, 3
    v = rng.standard_normal((B, L, Hkv, d))
    W = rng.standard_normal((Hkv * d, Hkv)) * 0.7
    A = np.array([-1.0, -2.0])
    dt = dt_scores64(v, W, A)
    for b in range(B):
        for j in range(L):
            for g in range(Hkv):
                x = 0.0
                for hp in range(Hkv):
                    for e in range(d):
                        x += v[b, j, hp, e] * W[hp * d + e, g]
                sig = 1.0 / (1.0 + math.exp(x))
                want = sig if g == 0 else sig * sig
                assert dt[b, g, j] == pytest.approx(want, rel=1e-12)


def check_dt_flatten_order(dt_scores64):
    """One-hot probe: v nonzero only at (head 1, channel 2) and W nonzero only
    at input row 1*d + 2 -> only x[g] for that column moves.  A transposed
    flatten (channel-major) would read another W row."""
    Hkv, d = 3, 4
    v = np.zeros((1, 1, Hkv, d))
    v[0, 0, 1, 2] = 1.5
    W = np.zeros((Hkv * d, Hkv))
    W[1 * d + 2, 2] = 2.0        # x[g=2] = 3
    A = np.array([-1.0, -1.0, -1.0])
    dt = dt_scores64(v, W, A)
    assert dt[0, 0, 0] == pytest.approx(0.5, rel=1e-15)
    assert dt[0, 1, 0] == pytest.approx(0.5, rel=1e-15)
    assert dt[0, 2, 0] == pytest.approx(1.0 / (1.0 + math.exp(3.0)), rel=1e-14)


def brute_kept(dt_row, len_b, Lq, Lk, w, i):
    """Kept set of row i by counting ranks, straight from the definition:
    visible key j is kept iff fewer than w visible keys beat it (higher dt, or
    equal dt and lower index); when Lk <= w every visible key is kept."""
    q_pos = i + (Lk - Lq)
    vis = [j for j in range(Lk) if j <= q_pos and j < len_b]
    if Lk <= w:
        return set(vis)
    kept = set()
    for j in vis:
        beats = sum(1 for k in vis if dt_row[k] > dt_row[j] or (dt_row[k] == dt_row[j] and k < j))
        if beats < w:
            kept.add(j)
    return kept


def check_mask_brute_force(kept_mask, seed=0, trials=60):
    rng = np.random.default_rng(seed)
    for t in range(trials):
        Lk = int(rng.integers(1, 17))
        decode = (t % 4 == 3)
        Lq = 1 if decode else Lk
        B, Hkv = 2, 2
        # few distinct values -> many exact ties
        vals = rng.choice(np.array([0.25, 0.5, 0.5, 0.75, 1.0, 0.125], dtype=np.float32),
                          size=(B, Hkv, Lk))
        lengths = rng.integers(1, Lk + 1, size=B)
        for w in range(1, 17):
            km = kept_mask(vals, lengths, Lq, Lk, w)
            for b in range(B):
                for g in range(Hkv):
                    for i in range(Lq):
                        got = set(np.nonzero(km[b, g, i])[0].tolist())
                        assert got == brute_kept(vals[b, g], int(lengths[b]), Lq, Lk, w, i), (t, w, b, g, i)


# ----------------------------------------------------------------------------
# S1 pins
# ----------------------------------------------------------------------------

def test_dt_worked_example():
    check_dt_worked_example(oracle.dt_scores64)


def test_dt_A_zero_is_exactly_one():
    # [Guide §DMA.init]: A starts at zeros, so dt = exp(0) = 1 for every key.
    rng = np.random.default_rng(1)
    v = rng.standard_normal((2, 7, 3, 4))
    W = rng.standard_normal((12, 3))
    dt = oracle.dt_scores(v, W, np.zeros(3))
    assert dt.dtype == np.float32 and np.all(dt == 1.0)


def test_dt_sigmoid_closed_form():
    check_dt_sigmoid_closed_form(oracle.dt_scores64)


def test_dt_flatten_order():
    check_dt_flatten_order(oracle.dt_scores64)


def test_softplus_extremes():
    # softplus(x) -> x for large x, -> e^x for very negative x, ln 2 at 0.
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-16)
    assert oracle.softplus(800.0) == 800.0
    assert oracle.softplus(-800.0) == 0.0
    assert oracle.softplus(-30.0) == pytest.approx(math.exp(-30.0), rel=1e-12)


# ----------------------------------------------------------------------------
# S2 pins
# ----------------------------------------------------------------------------

def test_mask_brute_force_with_ties():
    check_mask_brute_force(oracle.kept_mask)


def test_mask_kept_count_and_monotone_eviction():
    rng = np.random.default_rng(3)
    B, Hkv, L = 3, 2, 96
    dt = rng.random((B, Hkv, L)).astype(np.float32)
    dt[:, :, ::7] = dt[:, :, 3:4]            # some exact ties
    lengths = np.array([96, 50, 1])
    for w in (1, 5, 17, 64, 95, 96, 200):
        km = oracle.kept_mask(dt, lengths, L, L, w)
        for b in range(B):
            for i in range(L):
                nvis = min(i + 1, int(lengths[b]))
                want = min(w, nvis)
                assert np.all(km[b, :, i].sum(axis=-1) == want)
                if i + 1 < L:
                    # kept(i+1) is inside kept(i) plus the new key i+1
                    extra = km[b, :, i + 1] & ~km[b, :, i]
                    extra[:, min(i + 1, L - 1)] = False
                    assert not extra.any()


def test_mask_closed_forms_monotone_dt():
    L, w = 40, 6
    inc = np.arange(1, L + 1, dtype=np.float32)[None, None, :] / L
    dec = inc[:, :, ::-1].copy()
    const = np.ones((1, 1, L), dtype=np.float32)      # A = 0
    lengths = np.array([L])
    km_inc = oracle.kept_mask(inc, lengths, L, L, w)[0, 0]
    km_dec = oracle.kept_mask(dec, lengths, L, L, w)[0, 0]
    km_const = oracle.kept_mask(const, lengths, L, L, w)[0, 0]
    for i in range(L):
        # increasing scores: the causal sliding window of the last w keys
        window = np.zeros(L, bool)
        window[max(0, i - w + 1):i + 1] = True
        assert np.array_equal(km_inc[i], window)
        # decreasing or constant scores: the first min(w, i+1) keys
        first = np.zeros(L, bool)
        first[:min(w, i + 1)] = True
        assert np.array_equal(km_dec[i], first)
        assert np.array_equal(km_const[i], first)


def test_mask_window_at_least_length_is_causal_padding():
    rng = np.random.default_rng(4)
    L = 33
    dt = rng.random((2, 3, L)).astype(np.float32)
    lengths = np.array([33, 20])
    for w in (L, L + 5):
        km = oracle.kept_mask(dt, lengths, L, L, w)
        for b in range(2):
            causal = np.tril(np.ones((L, L), bool))
            causal[:, int(lengths[b]):] = False
            assert np.array_equal(km[b, 0], causal) and np.array_equal(km[b, 2], causal)


def test_mask_matches_torch_topk_without_ties():
    rng = np.random.default_rng(5)
    L, w = 70, 9
    dt = (rng.permutation(L).astype(np.float32) + 1.0)[None, None, :] / 128.0
    lengths = np.array([L])
    M = oracle.dynamic_mask_rows(dt[0, 0], L, L, L, w, range(L))
    for i in range(L):
        row = torch.full((L,), -1.0, dtype=torch.float64)
        row[:i + 1] = torch.from_numpy(dt[0, 0, :i + 1].astype(np.float64))
        k = min(w, i + 1)
        top = set(torch.topk(row, k).indices.tolist())
        assert set(np.nonzero(M[i] > MIN_DTYPE)[0].tolist()) == top
        assert np.all(M[i][M[i] > MIN_DTYPE] == dt[0, 0][sorted(top)])


def test_thresholds_rebuild_mask_and_are_monotone():
    rng = np.random.default_rng(6)
    B, Hkv, L = 2, 2, 80
    dt = rng.choice(np.array([0.1, 0.2, 0.3, 0.4], np.float32), size=(B, Hkv, L))
    lengths = np.array([80, 41])
    for w in (1, 7, 30, 80):
        tau = oracle.thresholds(dt, lengths, L, L, w)
        km = oracle.kept_mask(dt, lengths, L, L, w)
        for b in range(B):
            for g in range(Hkv):
                assert np.all(np.diff(tau[b, g].astype(np.float64)) >= 0)
                for i in range(L):
                    lim = min(i + 1, int(lengths[b]))
                    rebuilt = np.array([j < lim and oracle.composite_key(dt[b, g, j], j) >= int(tau[b, g, i])
                                        for j in range(L)])
                    assert np.array_equal(rebuilt, km[b, g, i])


# ----------------------------------------------------------------------------
# S3 / S4 pins (float64 SDPA is an independent library routine)
# ----------------------------------------------------------------------------

def _rand_qkv(rng, B, L, Hq, Hkv, d):
    q = rng.standard_normal((B, L, Hq, d))
    k = rng.standard_normal((B, L, Hkv, d))
    v = rng.standard_normal((B, L, Hkv, d))
    return q, k, v


def _sdpa(q, k, v, add_mask, scale):
    """torch SDPA in float64; q [B,L,Hq,d], k/v [B,Lk,Hkv,d], add_mask [B,Hq,L,Lk] or None."""
    n_rep = q.shape[2] // k.shape[2]
    Q = torch.from_numpy(q).permute(0, 2, 1, 3)
    K = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(n_rep, dim=1)
    V = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(n_rep, dim=1)
    m = None if add_mask is None else torch.from_numpy(add_mask)
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=m, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def test_prefill_dense_A_zero_equals_causal_gqa_sdpa():
    rng = np.random.default_rng(7)
    B, L, Hq, Hkv, d = 2, 24, 4, 2, 8
    q, k, v = _rand_qkv(rng, B, L, Hq, Hkv, d)
    W = rng.standard_normal((Hkv * d, Hkv)) * 0.02
    out = oracle.prefill(q, k, v, W, np.zeros(Hkv), np.array([L, L]), w=L, scale=d ** -0.5)
    n_rep = Hq // Hkv
    Q = torch.from_numpy(q).permute(0, 2, 1, 3)
    K = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(n_rep, dim=1)
    V = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(n_rep, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=d ** -0.5)
    np.testing.assert_allclose(out, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)


def test_prefill_dense_bias_and_padding_equals_sdpa_additive_mask():
    rng = np.random.default_rng(8)
    B, L, Hq, Hkv, d = 2, 20, 6, 3, 8
    q, k, v = _rand_qkv(rng, B, L, Hq, Hkv, d)
    W = rng.standard_normal((Hkv * d, Hkv)) * 0.3
    A = np.array([-2.0, -0.5, -1.0])
    lengths = np.array([20, 13])
    dt = oracle.dt_scores(v, W, A)
    out = oracle.prefill(q, k, v, W, A, lengths, w=L + 3, scale=0.37)
    add = np.full((B, Hq, L, L), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(L):
                n = min(i + 1, int(lengths[b]))
                add[b, h, i, :n] = dt[b, g, :n]
    np.testing.assert_allclose(out, _sdpa(q, k, v, add, 0.37), rtol=1e-12, atol=1e-12)


def test_prefill_window_one_copies_best_value_row():
    rng = np.random.default_rng(9)
    B, L, Hq, Hkv, d = 1, 30, 2, 1, 5
    q, k, v = _rand_qkv(rng, B, L, Hq, Hkv, d)
    dt = rng.choice(np.array([0.3, 0.6, 0.9], np.float32), size=(B, Hkv, L))
    out = oracle.prefill(q, k, v, None, None, np.array([L]), w=1, scale=0.125, dt=dt)
    for i in range(L):
        best = max(range(i + 1), key=lambda j: (dt[0, 0, j], -j))
        for h in range(Hq):
            np.testing.assert_allclose(out[0, i, h], v[0, best, 0], rtol=0, atol=1e-15)


def test_prefill_zero_scale_is_dt_weighted_mean():
    # scale = 0 leaves softmax(dt) over the kept keys: weights e^{dt_j} / sum.
    rng = np.random.default_rng(10)
    B, L, Hq, Hkv, d = 1, 26, 2, 2, 4
    q, k, v = _rand_qkv(rng, B, L, Hq, Hkv, d)
    dt = rng.random((B, Hkv, L)).astype(np.float32)
    w = 5
    out = oracle.prefill(q, k, v, None, None, np.array([L]), w=w, scale=0.0, dt=dt)
    for g in range(Hkv):
        for i in range(L):
            kept = sorted(brute_kept(dt[0, g], L, L, L, w, i))
            wts = np.array([math.exp(float(dt[0, g, j])) for j in kept])
            want = (wts[:, None] * v[0, kept, g, :]).sum(0) / wts.sum()
            np.testing.assert_allclose(out[0, i, g], want, rtol=1e-13, atol=1e-14)


def test_prefill_first_row_is_first_value():
    rng = np.random.default_rng(11)
    q, k, v = _rand_qkv(rng, 2, 9, 4, 2, 6)
    W = rng.standard_normal((12, 2)) * 0.1
    out = oracle.prefill(q, k, v, W, np.array([-1.0, -3.0]), np.array([9, 9]), w=3, scale=0.4)
    for h in range(4):
        np.testing.assert_allclose(out[:, 0, h], v[:, 0, h // 2], rtol=0, atol=1e-15)


def test_decode_short_cache_equals_sdpa_full_attention_plus_bias():
    rng = np.random.default_rng(12)
    B, Lk, Hq, Hkv, d = 3, 40, 4, 2, 8
    q = rng.standard_normal((B, Hq, d))
    kc = rng.standard_normal((B, Lk, Hkv, d))
    vc = rng.standard_normal((B, Lk, Hkv, d))
    W = rng.standard_normal((Hkv * d, Hkv)) * 0.1
    A = np.array([-1.5, -0.2])
    lengths = np.array([40, 17, 1])
    out = oracle.decode_step(q, kc, vc, W, A, lengths, w=64, scale=d ** -0.5)
    dt = oracle.dt_scores(vc, W, A)
    add = np.full((B, Hq, 1, Lk), -np.inf)
    for b in range(B):
        for h in range(Hq):
            add[b, h, 0, :lengths[b]] = dt[b, h // 2, :lengths[b]]
    ref = _sdpa(q[:, None], kc, vc, add, d ** -0.5)[:, 0]
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_decode_ignores_cache_beyond_length_and_window_one():
    rng = np.random.default_rng(13)
    B, Lk, Hq, Hkv, d = 2, 50, 2, 1, 4
    q = rng.standard_normal((B, Hq, d))
    kc = rng.standard_normal((B, Lk, Hkv, d))
    vc = rng.standard_normal((B, Lk, Hkv, d))
    dt = rng.random((B, Hkv, Lk)).astype(np.float32)
    lengths = np.array([31, 50])
    out1 = oracle.decode_step(q, kc, vc, None, None, lengths, w=1, scale=0.5, dt=dt)
    for b in range(B):
        n = int(lengths[b])
        best = max(range(n), key=lambda j: (dt[b, 0, j], -j))
        np.testing.assert_allclose(out1[b, 0], vc[b, best, 0], atol=1e-15, rtol=0)
    kc2, vc2, dt2 = kc.copy(), vc.copy(), dt.copy()
    kc2[0, 31:] = 99.0
    vc2[0, 31:] = -99.0
    dt2[0, :, 31:] = 1e30
    a = oracle.decode_step(q, kc, vc, None, None, lengths, w=7, scale=0.5, dt=dt)
    b_ = oracle.decode_step(q, kc2, vc2, None, None, lengths, w=7, scale=0.5, dt=dt2)
    np.testing.assert_array_equal(a[0], b_[0])


def test_decode_equals_last_prefill_row():
    rng = np.random.default_rng(14)
    L, Hq, Hkv, d = 45, 4, 2, 8
    q, k, v = _rand_qkv(rng, 1, L, Hq, Hkv, d)
    dt = rng.random((1, Hkv, L)).astype(np.float32)
    w = 11
    pre = oracle.prefill(q, k, v, None, None, np.array([L]), w=w, scale=0.3, dt=dt)
    dec = oracle.decode_step(q[:, L - 1], k, v, None, None, np.array([L]), w=w, scale=0.3, dt=dt)
    np.testing.assert_allclose(dec, pre[:, L - 1], rtol=1e-13, atol=1e-14)


def check_prefill_rows_sdpa(prefill_rows, seed=15):
    """prefill_rows (the per-(batch, query head) row sampler the full-size
    parity tests and the CPU baseline call) against float64 SDPA with an
    additive mask built from first principles: brute-force rank counting for
    the kept set [Guide §DMA.3], dt on kept keys, -inf elsewhere, GQA group
    h // n_rep [Guide §Config].  Covers n_rep 1, 2 and 3, right padding, a
    window below the length with forced ties, and a non-contiguous row set
    that includes the first and last rows."""
    rng = np.random.default_rng(seed)
    for Hq, Hkv in ((2, 2), (4, 2), (6, 2)):
        B, L, d, w = 2, 23, 8, 5
        q, k, v = _rand_qkv(rng, B, L, Hq, Hkv, d)
        # few distinct dt values: many exact ties at the window boundary
        dt = rng.choice(np.array([0.25, 0.5, 0.75, 1.5], np.float32), size=(B, Hkv, L))
        lengths = np.array([L, 14])
        scale = 0.31
        add = np.full((B, Hq, L, L), -np.inf)
        n_rep = Hq // Hkv
        for b in range(B):
            for h in range(Hq):
                g = h // n_rep
                for i in range(L):
                    for j in brute_kept(dt[b, g], int(lengths[b]), L, L, w, i):
                        add[b, h, i, j] = float(dt[b, g, j])
        ref = _sdpa(q, k, v, add, scale)
        rows = [L - 1, 0, 3, 9, 14, 13, 17]
        for b in range(B):
            for h in range(Hq):
                got = prefill_rows(q, k, v, dt, lengths, w, scale, b, h, rows)
                np.testing.assert_allclose(got, ref[b, rows, h, :], rtol=1e-12, atol=1e-12)


def test_prefill_rows_equals_sdpa_with_brute_force_mask():
    check_prefill_rows_sdpa(oracle.prefill_rows)
