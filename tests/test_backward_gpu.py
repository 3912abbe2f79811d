"""Parity of the backward (through the C ABI) with the float64 oracle, the
kept-key selection held fixed and built from the same float32 dt (the
oracle's, passed as dt_in).  The forward output the backward takes is the
oracle's, rounded to bf16.

The row normalisers the forward can hand over (dma_forward_prefill with
lse_out) are checked against float64 too, and the backward is run with them.

Bars (derived from the arithmetic): the kernels round P and dS to bf16 for
the tensor core (relative error 2^-9 each, accumulated in float32 over up to
a few thousand keys or rows with mixed signs) and round dq, dk, dv to bf16;
every gradient G must satisfy
  max |got - want| <= 2e-2 * max |want|   and   mean |got - want| <= 4e-3 * mean |want|,
except dA, a sum over every token of d_dt * dt * softplus(x) whose terms cancel
almost completely (d_dt sums to zero over the keys, since each softmax row's
dS does): its error is bounded by the same relative bar applied to the sum
of the terms' magnitudes, |got - want| <= 2e-2 * sum |d_dt dt softplus(x)|.
"""
import numpy as np
import pytest
import torch

import oracle
from doge_dynamic_mask_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_REL = 2e-2, 4e-3


@pytest.fixture(scope="module")
def dma():
    from doge_dynamic_mask_b200 import build
    build.build()
    from doge_dynamic_mask_b200 import dma as m
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_grad_close(got, want, what):
    g = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    assert np.isfinite(g).all(), what
    err = np.abs(g - want)
    scale_max, scale_mean = np.abs(want).max(), np.abs(want).mean()
    assert err.max() <= MAX_REL * scale_max and err.mean() <= MEAN_REL * scale_mean, (
        f"{what}: max {err.max():.3e} (bar {MAX_REL * scale_max:.3e}), mean {err.mean():.3e} "
        f"(bar {MEAN_REL * scale_mean:.3e})")


def check_lse(dma, x, d, dt, wl):
    """The forward's row normalisers (dma_forward_prefill with lse_out) against
    float64: lse = log2 of the sum over the row's kept keys of
    exp(scale q.k + dt).  The kernel forms q.k from bf16 inputs in float32 and
    carries dt / scale through the tensor core as three bf16 terms, so the bar
    is 2e-3 * (1 + max |z|) in log2 units."""
    lse = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.float32, device="cuda")
    dma.dma_forward_prefill(d["q"], d["k"], d["v"], d["W"], d["A"], d["lengths"], wl.w,
                            dt_in=torch.from_numpy(dt).cuda(), lse_out=lse)
    torch.cuda.synchronize()
    got = lse.cpu().numpy().astype(np.float64)
    q, k = f64(x["q"]), f64(x["k"])
    kept = oracle.kept_mask(dt, x["lengths"].numpy(), wl.L, wl.L, wl.w)
    n_rep = wl.Hq // wl.Hkv
    for b in range(wl.B):
        for h in range(wl.Hq):
            g = h // n_rep
            z = wl.scale * q[b, :, h] @ k[b, :, g].T + dt[b, g].astype(np.float64)[None, :]
            zk = np.where(kept[b, g], z, -np.inf)
            zmax = zk.max(axis=1, keepdims=True)
            want = (zmax[:, 0] + np.log(np.exp(zk - zmax).sum(axis=1))) / np.log(2.0)
            bar = 2e-3 * (1.0 + np.abs(np.where(kept[b, g], z, 0.0)).max())
            err = np.abs(got[b, h] - want)
            assert err.max() <= bar, (b, h, err.max(), bar)
    return lse


def run_case(dma, wl, dout_seed=1, via_lse=False):
    x = make_inputs(wl)
    q, k, v = f64(x["q"]), f64(x["k"]), f64(x["v"])
    W, A = x["W"].double().numpy(), x["A"].double().numpy()
    lengths = x["lengths"].numpy()
    dt = oracle.dt_scores(v, W, A)
    out = oracle.prefill(q, k, v, W, A, lengths, wl.w, wl.scale, dt=dt)
    g = torch.Generator().manual_seed(dout_seed)
    dout = torch.randn(x["q"].shape, generator=g).to(torch.bfloat16)
    want = oracle.prefill_backward(q, k, v, W, A, lengths, wl.w, wl.scale, f64(dout), dt_fixed=dt)
    d = {n: t.cuda() for n, t in x.items()}
    lse = check_lse(dma, x, d, dt, wl) if via_lse else None
    got = dma.dma_backward_prefill(d["q"], d["k"], d["v"], d["W"], d["A"], d["lengths"], wl.w,
                                   torch.from_numpy(out).to(torch.bfloat16).cuda(), dout.cuda(),
                                   dt_in=torch.from_numpy(dt).cuda(), want_d_dt=True, lse_in=lse)
    torch.cuda.synchronize()
    names = ("dq", "dk", "dv", "dW", "d_dt")
    order = (0, 1, 2, 4, 3)    # oracle returns dq, dk, dv, d_dt, dW, dA
    for name, gi, wi in zip(names, (0, 1, 2, 3, 5), order):
        assert_grad_close(got[gi], want[wi], name)
    # dA: bar on the magnitude of its terms
    B, L, Hkv, d = v.shape
    x64 = v.reshape(B, L, Hkv * d) @ W
    sp = oracle.softplus(x64)
    terms = np.abs(want[3].transpose(0, 2, 1) * np.exp(A * sp) * sp).sum(axis=(0, 1))
    err = np.abs(f64(got[4]) - want[5])
    assert (err <= MAX_REL * terms).all(), (err, terms)


def wl(B, L, Hq, Hkv, d, w, lens=None, seed=0):
    lo, hi = (None, None) if lens is None else lens
    return Workload("bwd", "prefill", B=B, L=L, Hq=Hq, Hkv=Hkv, d=d, w=w, a_lo=-2.0, a_hi=-0.1, seed=seed,
                    len_lo=lo, len_hi=hi)


@pytest.mark.parametrize("case", [
    wl(1, 200, 4, 2, 64, 64, seed=1),              # top-k active, ragged row tile
    wl(2, 130, 2, 2, 64, 1000, seed=2),            # window >= L: causal + bias
    wl(2, 300, 6, 2, 64, 96, lens=(150, 300), seed=3),   # padding, n_rep 3
    wl(1, 257, 4, 4, 128, 100, seed=4),            # d = 128
    wl(1, 400, 2, 1, 128, 400, seed=5),            # d = 128, dense
])
def test_backward_matches_oracle(dma, case):
    run_case(dma, case)


@pytest.mark.parametrize("case", [
    wl(1, 200, 4, 2, 64, 64, seed=1),              # top-k active, ragged row tile
    wl(2, 300, 6, 2, 64, 96, lens=(150, 300), seed=3),   # padding, n_rep 3
    wl(2, 130, 2, 2, 64, 1000, seed=2),            # window >= L: the forward builds its own lists
    wl(1, 257, 4, 4, 128, 100, seed=4),            # d = 128
])
def test_backward_with_forward_normalisers(dma, case):
    """The forward hands each row's log-sum-exp to the backward, which then
    skips recomputing the row statistics; both are checked against float64."""
    run_case(dma, case, via_lse=True)
