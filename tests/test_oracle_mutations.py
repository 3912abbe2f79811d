"""Planted mistakes in the oracle (CPU only) must fail at least one pin.

Each mutant swaps one oracle function for a plausibly-wrong variant (a dropped
term, a wrong sign, an off-by-one, a transposed operand, a reversed tie-break)
and runs the pins that should catch it.
"""
import numpy as np
import pytest

import oracle
import oracle.dma_oracle as om
import tests.test_oracle_pins as pins


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


# ---- S1 mutants -------------------------------------------------------------

def _dt_transposed_flatten(v, W, A):
    v = np.asarray(v, np.float64)
    B, L, Hkv, d = v.shape
    x = v.transpose(0, 1, 3, 2).reshape(B, L, Hkv * d) @ np.asarray(W, np.float64)
    return np.exp(np.asarray(A)[None, None] * om.softplus(x)).transpose(0, 2, 1)


def _dt_dropped_max_term(v, W, A):
    v = np.asarray(v, np.float64)
    B, L, Hkv, d = v.shape
    x = v.reshape(B, L, Hkv * d) @ np.asarray(W, np.float64)
    sp = np.log1p(np.exp(-np.abs(x)))           # forgot max(x, 0)
    return np.exp(np.asarray(A)[None, None] * sp).transpose(0, 2, 1)


def _dt_sign_flip(v, W, A):
    return om.dt_scores64(v, W, -np.asarray(A))


def test_mutant_transposed_flatten_is_caught():
    _fails(pins.check_dt_flatten_order, _dt_transposed_flatten)


def test_mutant_softplus_dropped_term_is_caught():
    _fails(pins.check_dt_sigmoid_closed_form, _dt_dropped_max_term)
    _fails(pins.check_dt_worked_example, _dt_dropped_max_term)


def test_mutant_A_sign_is_caught():
    _fails(pins.check_dt_worked_example, _dt_sign_flip)


# ---- S2 mutants -------------------------------------------------------------

def _mask_factory(tie_high_first=False, causal_shift=0, strict_window=False):
    def rows_fn(dt_row, len_b, Lq, Lk, w, rows):
        dt_row = np.asarray(dt_row, np.float32).astype(np.float64)
        out = np.full((len(list(rows)), Lk), om.MIN_DTYPE)
        for r, i in enumerate(rows):
            lim = min(i + (Lk - Lq) + 1 + causal_shift, len_b)
            m = np.full(Lk, om.MIN_DTYPE)
            m[:max(lim, 0)] = dt_row[:max(lim, 0)]
            if Lk > w or (strict_window and Lk >= w):
                if tie_high_first:
                    order = (Lk - 1) - np.argsort(-m[::-1], kind="stable")
                else:
                    order = np.argsort(-m, kind="stable")
                keep = np.zeros(Lk, bool)
                keep[order[:w - (1 if strict_window and Lk == w else 0)]] = True
                m[~keep] = om.MIN_DTYPE
            out[r] = m
        return out

    def kept(dt, lengths, Lq, Lk, w):
        dt = np.asarray(dt, np.float32)
        B, Hkv, _ = dt.shape
        res = np.zeros((B, Hkv, Lq, Lk), bool)
        for b in range(B):
            for g in range(Hkv):
                res[b, g] = rows_fn(dt[b, g], int(lengths[b]), Lq, Lk, w, list(range(Lq))) > om.MIN_DTYPE
        return res
    return rows_fn, kept


def test_mutant_tie_break_is_caught():
    _, kept = _mask_factory(tie_high_first=True)
    _fails(pins.check_mask_brute_force, kept)


def test_mutant_causal_off_by_one_is_caught():
    for shift in (-1, 1):
        _, kept = _mask_factory(causal_shift=shift)
        _fails(pins.check_mask_brute_force, kept)


def test_mutant_window_boundary_is_caught():
    _, kept = _mask_factory(strict_window=True)
    _fails(pins.check_mask_brute_force, kept)


# ---- S3 / S4 mutants --------------------------------------------------------

def _attn_bias_sign(q_rows, K, V, mask_rows, scale):
    m = np.where(mask_rows > om.MIN_DTYPE, -mask_rows, mask_rows)
    return _plain_attention(q_rows, K, V, m, scale)


def _plain_attention(q_rows, K, V, mask_rows, scale):
    s = scale * (np.asarray(q_rows, np.float64) @ np.asarray(K, np.float64).T) + mask_rows
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ np.asarray(V, np.float64)


def _attn_scale_on_bias(q_rows, K, V, mask_rows, scale):
    s = scale * ((np.asarray(q_rows, np.float64) @ np.asarray(K, np.float64).T) + mask_rows)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p / p.sum(axis=1, keepdims=True)) @ np.asarray(V, np.float64)


def _attn_transposed_v(q_rows, K, V, mask_rows, scale):
    s = scale * (np.asarray(q_rows, np.float64) @ np.asarray(K, np.float64).T) + mask_rows
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    Vt = np.asarray(V, np.float64)
    return p @ Vt[::-1]                     # wrong key <-> value-row pairing


def test_mutant_bias_sign_is_caught(monkeypatch):
    monkeypatch.setattr(om, "attention_rows", _attn_bias_sign)
    _fails(pins.test_prefill_zero_scale_is_dt_weighted_mean)
    _fails(pins.test_prefill_dense_bias_and_padding_equals_sdpa_additive_mask)


def test_mutant_scale_applied_to_bias_is_caught(monkeypatch):
    monkeypatch.setattr(om, "attention_rows", _attn_scale_on_bias)
    _fails(pins.test_prefill_dense_bias_and_padding_equals_sdpa_additive_mask)


def test_mutant_value_pairing_is_caught(monkeypatch):
    monkeypatch.setattr(om, "attention_rows", _attn_transposed_v)
    _fails(pins.test_prefill_dense_A_zero_equals_causal_gqa_sdpa)
    _fails(pins.test_decode_short_cache_equals_sdpa_full_attention_plus_bias)


def test_mutant_gqa_mapping_is_caught(monkeypatch):
    # query head h reading kv head h % H_kv instead of h // n_rep
    orig = om.prefill

    def bad_prefill(q, k, v, W, A, lengths, w, scale, dt=None, row_block=1024):
        q = np.asarray(q, np.float64)
        Hq, Hkv = q.shape[2], np.asarray(k).shape[2]
        perm = [(h % Hkv) * (Hq // Hkv) + h // Hkv for h in range(Hq)]
        return orig(q[:, :, perm], k, v, W, A, lengths, w, scale, dt=dt, row_block=row_block)[:, :, np.argsort(perm)]

    monkeypatch.setattr(oracle, "prefill", bad_prefill)
    _fails(pins.test_prefill_dense_bias_and_padding_equals_sdpa_additive_mask)


# ---- prefill_rows mutants (the row sampler of the full-size parity tests) ----

def _rows_factory(wrong_group=False, row_shift=0):
    def rows_fn(q, k, v, dt, lengths, w, scale, b, h, rows):
        Hq, Hkv = q.shape[2], k.shape[2]
        g = h % Hkv if wrong_group else h // (Hq // Hkv)
        rows = list(rows)
        M = om.dynamic_mask_rows(dt[b, g], int(lengths[b]), q.shape[1], q.shape[1], w,
                                 [min(max(r + row_shift, 0), q.shape[1] - 1) for r in rows])
        return om.attention_rows(np.asarray(q[b, rows, h, :], np.float64), k[b, :, g, :], v[b, :, g, :], M, scale)
    return rows_fn


def test_mutant_prefill_rows_group_is_caught():
    _fails(pins.check_prefill_rows_sdpa, _rows_factory(wrong_group=True))


def test_mutant_prefill_rows_offset_is_caught():
    for shift in (-1, 1):
        _fails(pins.check_prefill_rows_sdpa, _rows_factory(row_shift=shift))
