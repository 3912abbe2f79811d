"""The procedure the backward kernel follows, restated in plain numpy on the
CPU and checked against the float64 oracle: each 128-row tile walks its
kept-key list (the union of its rows' kept keys, each key with the interval
of tile rows that keep it) twice, first for the rows' softmax statistics
(log2 units), then for P = 2^(x - lse), dS = P (dP - D), dQ accumulated over
the list, and the keys' dK, dV and d_dt contributions (d_dt as the column sum
of dS, the ones column of the [Q | 1] product).  It models the algorithm, not
the CUDA code; tiles of 8 rows and 8 keys stand in for 128 so that small
cases span several tiles and ragged ends."""
import math

import numpy as np
import pytest

import oracle

TILE = 8


def tile_lists(kept, r0, nrows):
    """Key list of rows r0 .. r0+nrows-1 of one (b, g): keys every row keeps
    first, then the others, index order within each class; each with the tile
    rows [lo, hi) that keep it."""
    rows = kept[r0:r0 + nrows]
    union = np.nonzero(rows.any(axis=0))[0]
    full = [int(j) for j in union if rows[:, j].all()]
    part = [int(j) for j in union if not rows[:, j].all()]
    out = []
    for j in full + part:
        rr = np.nonzero(rows[:, j])[0]
        assert (np.diff(rr) == 1).all()          # one contiguous interval of rows
        out.append((j, int(rr[0]), int(rr[-1]) + 1))
    return out


def backward_by_tiles(q, k, v, dt, lengths, w, scale, out, dout):
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    n_rep = Hq // Hkv
    log2e = 1.0 / math.log(2.0)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    d_dt = np.zeros((B, Hkv, L))
    for b in range(B):
        for g in range(Hkv):
            kept = oracle.kept_mask(dt[b:b + 1, g:g + 1], lengths[b:b + 1], L, L, w)[0, 0]
            for r0 in range(0, L, TILE):
                nrows = min(TILE, L - r0)
                lst = tile_lists(kept, r0, nrows)
                for h in range(g * n_rep, (g + 1) * n_rep):
                    Q = q[b, r0:r0 + nrows, h]
                    dO = dout[b, r0:r0 + nrows, h]
                    D = (dO * out[b, r0:r0 + nrows, h]).sum(1)
                    m = np.full(nrows, -np.inf)
                    l = np.zeros(nrows)
                    tiles = [lst[i:i + TILE] for i in range(0, len(lst), TILE)]
                    def xs(tl):
                        x = np.full((nrows, len(tl)), -np.inf)
                        for c, (j, lo, hi) in enumerate(tl):
                            x[lo:hi, c] = (scale * (Q[lo:hi] @ k[b, j, g]) + float(dt[b, g, j])) * log2e
                        return x
                    for tl in tiles:                         # pass 1
                        x = xs(tl)
                        m_new = np.maximum(m, x.max(1))
                        fin = np.isfinite(m_new)
                        l[fin] = l[fin] * np.exp2(m[fin] - m_new[fin]) + np.exp2(x[fin] - m_new[fin][:, None]).sum(1)
                        m[fin] = m_new[fin]
                    lse = m + np.log2(l)
                    for tl in tiles:                         # pass 2
                        x = xs(tl)
                        P = np.exp2(x - lse[:, None])
                        keys = [j for j, _, _ in tl]
                        Kt, Vt = k[b, keys, g], v[b, keys, g]
                        dS = P * (dO @ Vt.T - D[:, None])
                        dq[b, r0:r0 + nrows, h] += scale * dS @ Kt
                        QO = np.concatenate([Q, np.ones((nrows, 1))], axis=1)   # [Q | 1]
                        dk_t = dS.T @ QO
                        dk[b, keys, g] += scale * dk_t[:, :d]
                        d_dt[b, g, keys] += dk_t[:, d]
                        dv[b, keys, g] += P.T @ dO
    return dq, dk, dv, d_dt


@pytest.mark.parametrize("B,L,Hq,Hkv,w,lens", [
    (1, 29, 2, 1, 5, None),
    (2, 23, 6, 2, 7, (12, 23)),      # padding, n_rep 3
    (2, 17, 4, 2, 40, None),         # window above the length
    (1, 30, 4, 4, 1, None),          # one key per row
])
def test_tiled_backward_matches_oracle(B, L, Hq, Hkv, w, lens):
    rng = np.random.default_rng(B * 100 + L)
    d = 6
    q = rng.standard_normal((B, L, Hq, d))
    k = rng.standard_normal((B, L, Hkv, d))
    v = rng.standard_normal((B, L, Hkv, d))
    W = rng.standard_normal((Hkv * d, Hkv)) * 0.3
    A = -rng.uniform(0.2, 2.0, Hkv)
    lengths = np.full(B, L) if lens is None else rng.integers(lens[0], lens[1] + 1, B)
    dout = rng.standard_normal((B, L, Hq, d))
    scale = 0.4
    dt = oracle.dt_scores(v, W, A)
    out = oracle.prefill(q, k, v, W, A, lengths, w, scale, dt=dt)
    want = oracle.prefill_backward(q, k, v, W, A, lengths, w, scale, dout, dt_fixed=dt)
    got = backward_by_tiles(q, k, v, dt, lengths, w, scale, out, dout)
    # dv: the attention part only (the oracle's dv adds the dt path)
    x = v.reshape(B, L, Hkv * d) @ W
    dx = want[3].transpose(0, 2, 1) * np.exp(A * oracle.softplus(x)) * A / (1 + np.exp(-x))
    dv_attn = want[2] - (dx.reshape(B * L, Hkv) @ W.T).reshape(B, L, Hkv, d)
    for name, g_, w_ in (("dq", got[0], want[0]), ("dk", got[1], want[1]), ("dv", got[2], dv_attn),
                         ("d_dt", got[3], want[3])):
        np.testing.assert_allclose(g_, w_, rtol=1e-9, atol=1e-10, err_msg=name)
