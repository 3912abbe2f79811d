"""The prefill selector's run-of-tiles derivation, checked on the CPU.

The prefill selection walks runs of consecutive row tiles.  Only a run's
first tile selects over its whole prefix.  Every later tile is derived from
the tile before it:
  - the threshold at the tile's first row is the w-th best of the previous
    tile's last-row kept set plus at most one new key (the new row's own key);
  - the tile's key union is the previous union filtered by that threshold,
    followed by the tile's new keys that pass it.
The per-row thresholds then come from the union's smallest keys, and every
key's row interval from those thresholds.

This test restates those steps in plain Python and checks them against the
oracle's thresholds and kept masks.  Exactness rests on two facts from the
page "Transformers 中的 Doge 小语言模型完全指南" (section
"动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", step 3): the per-key score
does not depend on the query row, and each row keeps its keep_window_size
best visible keys.  Cases cover random tile sizes and run lengths, valid
lengths that end inside, at the edge of, and before a run's tiles, and
forced ties.
"""
import numpy as np

from oracle import dma_oracle as oracle


def _index(key):
    return 0xFFFFFFFF - (key & 0xFFFFFFFF)


def _run_plans(dt, L, w, length, T, tpc):
    """Per-row thresholds and kept (key, lo, hi) intervals of every tile, the
    tiles taken in runs of tpc as the selector does."""
    keys = [oracle.composite_key(dt[j], j) for j in range(L)]
    n_tiles = (L + T - 1) // T
    taus = [None] * L
    lists = [None] * n_tiles
    for t_first in range(0, n_tiles, tpc):
        have = False
        U_prev, q_prev, tau_last = [], 0, 0
        for t in range(t_first, min(n_tiles, t_first + tpc)):
            r0 = t * T
            nrows = min(T, L - r0)
            p = min(r0, length - 1)
            q = min(r0 + nrows - 1, length - 1)
            if not (L > w) or q + 1 <= w:
                for r in range(nrows):
                    taus[r0 + r] = 0
                lists[t] = [(j, max(j - r0, 0), nrows) for j in range(q + 1)]
                have = False
                continue
            if have:
                tau0 = tau_last
                if p != q_prev:   # one new key competes with the previous last-row kept set
                    nk = keys[p]
                    above = [k for k in U_prev if k > tau_last]
                    a2 = min(above) if above else (1 << 64) - 1
                    tau0 = tau_last if nk < tau_last else min(nk, a2)
                U = [k for k in U_prev if k >= tau0] + [keys[j] for j in range(q_prev + 1, q + 1) if keys[j] >= tau0]
            else:
                tau0 = sorted(keys[: p + 1], reverse=True)[w - 1] if p + 1 > w else 0
                U = [keys[j] for j in range(q + 1) if keys[j] >= tau0]
            n_old = w if p + 1 > w else p + 1
            bot = sorted(U)[:T]
            row_tau = []
            for r in range(nrows):
                ip = min(r0 + r, length - 1)
                if ip + 1 <= w:
                    tau = 0
                else:
                    visible = n_old + sum(1 for k in U[n_old:] if _index(k) <= ip)
                    rank = visible - w + 1
                    cands = [k for k in bot if _index(k) <= ip]
                    tau = cands[rank - 1]
                row_tau.append(tau)
                taus[r0 + r] = tau
            lst = []
            for k in U:
                j = _index(k)
                lo = max(j - r0, 0)
                hi = next((r for r in range(nrows) if row_tau[r] > k), nrows)
                if hi > lo:
                    lst.append((j, lo, hi))
            lists[t] = lst
            U_prev, q_prev, tau_last, have = U, q, row_tau[nrows - 1], True
    return taus, lists


def test_runs_of_tiles_reproduce_the_oracle_selection():
    rng = np.random.default_rng(2024)
    for trial in range(120):
        T = int(rng.choice([4, 8, 16]))
        L = int(rng.integers(1, 12 * T))
        w = int(rng.integers(1, 5 * T))
        length = int(rng.integers(1, L + 1)) if trial % 2 else L
        tpc = int(rng.integers(1, 6))
        kind = trial % 4
        if kind == 0:
            dt = rng.uniform(0.05, 1.0, L).astype(np.float32)
        elif kind == 1:
            dt = rng.choice(np.array([0.25, 0.5, 0.75], np.float32), L)
        elif kind == 2:
            dt = np.ones(L, np.float32)   # A = 0: every key ties
        else:
            dt = np.sort(rng.uniform(0.05, 1.0, L)).astype(np.float32)[:: 1 if trial % 8 < 4 else -1].copy()
        lengths = np.array([length])
        want_tau = oracle.thresholds(dt[None, None], lengths, L, L, w)[0, 0]
        want_kept = oracle.kept_mask(dt[None, None], lengths, L, L, w)[0, 0]
        taus, lists = _run_plans(dt, L, w, length, T, tpc)
        assert [int(x) for x in want_tau] == taus, (trial, T, L, w, length, tpc)
        for t, lst in enumerate(lists):
            r0 = t * T
            nrows = min(T, L - r0)
            rebuilt = np.zeros((nrows, L), bool)
            for j, lo, hi in lst:
                rebuilt[lo:hi, j] = True
            assert np.array_equal(rebuilt, want_kept[r0:r0 + nrows]), (trial, t, T, L, w, length, tpc)
            if L > w:
                assert len(lst) <= w + T - 1
