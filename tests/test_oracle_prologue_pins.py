"""Pins for the oracle's prologue (q_norm / k_norm RMSNorm over head_dim,
rotary position embedding, KV-cache append), each against something other
than the oracle itself: hand-worked values, the complex-number form of the
rotation, the relative-position property that defines it, and invariants.
Planted mistakes in copies of the oracle must fail them.

Cited page: "Transformers 中的 Doge 小语言模型完全指南" ([Guide]), section
"动态掩码注意力（DMA）" forward-chain steps 1-2 and section "DogeConfig 全参数详解"
(rms_norm_eps = 1e-6).
"""
import math

import numpy as np
import pytest

import oracle
import oracle.dma_oracle as om


# ---- reusable checks (take the functions under test as arguments) ----------

def check_rms_norm(rms_norm):
    # hand example: x = (3, 4), mean square 12.5
    y = rms_norm(np.array([[3.0, 4.0]]), np.array([1.0, 2.0]), 0.0)
    assert y[0, 0] == pytest.approx(3.0 / math.sqrt(12.5), rel=1e-15)
    assert y[0, 1] == pytest.approx(8.0 / math.sqrt(12.5), rel=1e-15)
    # eps enters under the root: x = (1, 1), eps = 3 -> 1 / sqrt(1 + 3) = 1/2
    assert rms_norm(np.array([[1.0, 1.0]]), np.ones(2), 3.0)[0, 0] == pytest.approx(0.5, rel=1e-15)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 3, 16))
    y = rms_norm(x, np.ones(16), 0.0)
    np.testing.assert_allclose((y * y).mean(-1), 1.0, rtol=1e-13)      # unit mean square
    np.testing.assert_allclose(rms_norm(7.5 * x, np.ones(16), 0.0), y, rtol=1e-13)   # scale invariance


def check_rope(rope):
    # d = 2: one pair rotated by pos * theta^0 = pos radians
    x = np.array([[[0.6, -1.3]]])
    for p in (0, 1, 5, 1000):
        y = rope(x, np.array([p]), 10000.0)
        c, s = math.cos(p), math.sin(p)
        assert y[0, 0, 0] == pytest.approx(0.6 * c + 1.3 * s, abs=1e-13)
        assert y[0, 0, 1] == pytest.approx(-1.3 * c + 0.6 * s, abs=1e-13)
    rng = np.random.default_rng(2)
    d, theta = 16, 500.0
    x = rng.standard_normal((7, 2, d))
    pos = np.array([0, 1, 2, 3, 100, 4095, 70000])
    y = rope(x, pos, theta)
    # complex form: z_i = x_i + j x_{i+d/2} multiplied by exp(j pos theta^(-2i/d))
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    rot = np.exp(1j * pos[:, None, None] * theta ** (-2.0 * np.arange(d // 2) / d)[None, None, :])
    want = z * rot
    np.testing.assert_allclose(y[..., : d // 2], want.real, atol=1e-12)
    np.testing.assert_allclose(y[..., d // 2:], want.imag, atol=1e-12)
    # position 0 is the identity
    np.testing.assert_array_equal(rope(x[:1], np.array([0]), theta), x[:1])
    # relative position: q.k after rotation depends only on the offset
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 1, d))
    for m, n in ((3, 1), (40, 38), (1002, 1000)):
        a = float((rope(q, np.array([m]), theta) * rope(k, np.array([n]), theta)).sum())
        b = float((rope(q, np.array([2]), theta) * rope(k, np.array([0]), theta)).sum())
        assert a == pytest.approx(b, rel=1e-10)
    # composition of rotations
    np.testing.assert_allclose(rope(rope(x, pos, theta), pos + 11, theta), rope(x, 2 * pos + 11, theta), atol=1e-11)


def check_prologue(prologue, rms_norm):
    rng = np.random.default_rng(3)
    B, L, Hq, Hkv, d, Lmax = 2, 5, 4, 2, 8, 20
    q = rng.standard_normal((B, L, Hq, d))
    k = rng.standard_normal((B, L, Hkv, d))
    v = rng.standard_normal((B, L, Hkv, d))
    qw = rng.uniform(0.5, 2.0, d)
    kw = rng.uniform(0.5, 2.0, d)
    kc0 = rng.standard_normal((B, Lmax, Hkv, d))
    vc0 = rng.standard_normal((B, Lmax, Hkv, d))
    positions = np.array([0, 9])
    qo, kc, vc = prologue(q, k, v, qw, kw, 1e-6, 10000.0, positions, kc0, vc0)
    for b in range(B):
        p = int(positions[b])
        rows = list(range(p, p + L))
        rest = [r for r in range(Lmax) if r not in rows]
        np.testing.assert_array_equal(kc[b, rest], kc0[b, rest])         # untouched cache rows
        np.testing.assert_array_equal(vc[b, rest], vc0[b, rest])
        np.testing.assert_array_equal(vc[b, rows], v[b])                  # V appended unchanged
        # norm first, then rotation: each (i, i + d/2) pair keeps the length the
        # normalised, weighted pair had (a rotation preserves it)
        for x, w, out in ((q[b], qw, qo[b]), (k[b], kw, kc[b, rows])):
            ms = (x * x).mean(-1, keepdims=True) + 1e-6
            n = w * x / np.sqrt(ms)
            pair = lambda t: t[..., : d // 2] ** 2 + t[..., d // 2:] ** 2
            np.testing.assert_allclose(pair(out), pair(n), rtol=1e-12)
    # position 0 of sequence 0: no rotation at all
    np.testing.assert_allclose(qo[0, 0], rms_norm(q[0, 0], qw, 1e-6), rtol=1e-14)
    # shifting a sequence's position leaves every q.k of its new tokens unchanged
    # (relative positions), but moves where K lands in the cache
    qo2, kc2, _ = prologue(q, k, v, qw, kw, 1e-6, 10000.0, positions + np.array([3, 0]), kc0, vc0)
    s1 = np.einsum("lhd,mgd->lhmg", qo[0], kc[0, 0:L])
    s2 = np.einsum("lhd,mgd->lhmg", qo2[0], kc2[0, 3:3 + L])
    np.testing.assert_allclose(s1, s2, rtol=1e-10, atol=1e-10)


# ---- the pins ---------------------------------------------------------------

def test_rms_norm_pins():
    check_rms_norm(oracle.rms_norm)


def test_rope_pins():
    check_rope(oracle.rope)


def test_prologue_pins():
    check_prologue(oracle.prologue, oracle.rms_norm)


# ---- planted mistakes -------------------------------------------------------

def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_mutant_rms_norm_without_mean_is_caught():
    _fails(check_rms_norm, lambda x, w, eps: np.asarray(w) * x / np.sqrt((np.asarray(x) ** 2).sum(-1, keepdims=True) + eps))


def test_mutant_rms_norm_eps_outside_root_is_caught():
    _fails(check_rms_norm, lambda x, w, eps: np.asarray(w) * x / (np.sqrt((np.asarray(x) ** 2).mean(-1, keepdims=True)) + eps))


def _rope_interleaved(x, pos, theta):
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    ang = om.rope_angles(pos, d, theta)
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = b * c + a * s
    return out


def _rope_sign(x, pos, theta):
    return om.rope(x, -np.asarray(pos), theta)


def _rope_freq_exponent(x, pos, theta):
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, np.float64)[:, None] * np.power(theta, -np.arange(d // 2) / d)[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def test_mutant_rope_interleaved_pairs_is_caught():
    _fails(check_rope, _rope_interleaved)


def test_mutant_rope_sign_is_caught():
    _fails(check_rope, _rope_sign)


def test_mutant_rope_frequency_is_caught():
    _fails(check_rope, _rope_freq_exponent)


def test_mutant_prologue_rotation_before_norm_is_caught():
    def bad(q, k, v, qw, kw, eps, theta, positions, k_cache, v_cache):
        q = np.asarray(q, np.float64)
        k = np.asarray(k, np.float64)
        B, L = q.shape[:2]
        kc = np.array(k_cache, np.float64, copy=True)
        vc = np.array(v_cache, np.float64, copy=True)
        qo = np.empty_like(q)
        for b in range(B):
            pos = int(positions[b]) + np.arange(L)
            qo[b] = om.rms_norm(om.rope(q[b], pos, theta), qw, eps)
            kc[b, pos] = om.rms_norm(om.rope(k[b], pos, theta), kw, eps)
            vc[b, pos] = v[b]
        return qo, kc, vc
    _fails(check_prologue, bad, oracle.rms_norm)


def test_mutant_prologue_position_offset_ignored_for_q_is_caught():
    def bad(q, k, v, qw, kw, eps, theta, positions, k_cache, v_cache):
        qo, kc, vc = om.prologue(q, k, v, qw, kw, eps, theta, positions, k_cache, v_cache)
        L = np.asarray(q).shape[1]
        for b in range(np.asarray(q).shape[0]):
            qo[b] = om.rope(om.rms_norm(np.asarray(q[b], np.float64), qw, eps), np.arange(L), theta)
        return qo, kc, vc
    _fails(check_prologue, bad, oracle.rms_norm)
