"""The benchmark's work accounting, on the CPU.

Prefill throughput counts 4*d FLOPs per kept (query row, key) pair per query
head, and decode bandwidth counts the algorithmic KV bytes of a step.  The
pair count is checked against the oracle's own kept masks (materialised on
small random cases, ties included) and, for the benchmark workloads, against
closed forms: a row i of a sequence of valid length n keeps min(w, i + 1, n)
keys when the top-k is active.
"""
import numpy as np
import pytest

import bench
from doge_dynamic_mask_b200.workloads import WORKLOADS
from oracle import dma_oracle as oracle


def test_kept_pairs_equal_the_oracle_mask_count():
    rng = np.random.default_rng(21)
    for trial in range(16):
        L = int(rng.integers(1, 70))
        w = int(rng.integers(1, 80))
        B, Hkv = 2, 2
        lengths = rng.integers(1, L + 1, size=B).astype(np.int32)
        if trial % 4 == 0:   # forced ties
            dt = rng.choice(np.array([0.25, 0.5, 1.0], np.float32), size=(B, Hkv, L))
        else:
            dt = rng.uniform(0.01, 1.0, size=(B, Hkv, L)).astype(np.float32)
        kept = oracle.kept_mask(dt, lengths, L, L, w)
        for g in range(Hkv):
            assert int(kept[:, g].sum()) == bench.kept_pairs(L, w, lengths), (trial, L, w, lengths)


def _sum_min(L, w):
    # sum over rows i < L of min(w, i + 1)
    m = min(L, w)
    return m * (m + 1) // 2 + (L - m) * w


@pytest.mark.parametrize("name", ["tiny", "dense_eq", "sparse_pad", "long"])
def test_prefill_flops_of_the_workloads(name):
    wl = WORKLOADS[name]
    if wl.len_lo is None:
        lengths = np.full(wl.B, wl.L, np.int32)
    else:
        lengths = np.array([wl.len_lo, wl.len_hi, (wl.len_lo + wl.len_hi) // 2, wl.len_lo + 1][: wl.B], np.int32)
    per_bh = _sum_min(wl.L, wl.w) if wl.L > wl.w else wl.L * (wl.L + 1) // 2
    # with every valid length above w, rows past the length still keep w keys
    assert bench.kept_pairs(wl.L, wl.w, lengths) == wl.B * per_bh
    assert bench.prefill_flops(wl, lengths) == 4 * wl.d * wl.Hq * wl.B * per_bh
    expected = {"tiny": 14_368, "dense_eq": 2_098_176, "sparse_pad": 14_681_088, "long": 65_012_736}[name]
    assert per_bh == expected


def test_dense_eq_flops_and_decode_bytes():
    wl = WORKLOADS["dense_eq"]
    assert bench.prefill_flops(wl, np.full(wl.B, wl.L)) == 34_376_515_584
    dec = WORKLOADS["decode"]
    lengths = np.full(dec.B, dec.L, np.int32)
    v_scan = dec.B * dec.L * dec.Hkv * dec.d * 2
    kept_rows = dec.B * dec.Hkv * 2 * dec.w * dec.d * 2
    q_and_o = 2 * dec.B * dec.Hq * dec.d * 2
    assert bench.decode_bytes(dec, lengths) == v_scan + kept_rows + q_and_o == 9_127_329_792
    # a sequence shorter than the window keeps all of its keys
    short = lengths.copy()
    short[0] = 100
    assert bench.decode_bytes(dec, short) == bench.decode_bytes(dec, lengths) - dec.Hkv * 2 * (dec.w - 100) * dec.d * 2


def test_valid_rows_pairs_equal_the_oracle_mask_count_over_valid_rows():
    rng = np.random.default_rng(22)
    for trial in range(12):
        L = int(rng.integers(1, 60))
        w = int(rng.integers(1, 70))
        lengths = rng.integers(1, L + 1, size=3).astype(np.int32)
        dt = rng.uniform(0.01, 1.0, size=(3, 1, L)).astype(np.float32)
        kept = oracle.kept_mask(dt, lengths, L, L, w)
        want = sum(int(kept[b, 0, :lengths[b]].sum()) for b in range(3))
        assert bench.kept_pairs_valid_rows(L, w, lengths) == want, (trial, L, w, lengths)
    # full-length sequences: the valid-rows count is the whole count
    assert bench.kept_pairs_valid_rows(2048, 2048, [2048] * 2) == bench.kept_pairs(2048, 2048, [2048] * 2)
