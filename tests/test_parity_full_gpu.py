"""Parity at the full benchmark sizes, in the launch configuration the benchmark
times (the same entry points on the same workloads): every output is computed
by the CUDA path; the oracle recomputes sampled rows one by one.

Bars as in test_parity_gpu: tau bit-exact on sampled rows (same float32 dt),
outputs max-abs <= 2e-2 and mean-abs <= 2e-3 on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from doge_dynamic_mask_b200.workloads import WORKLOADS, make_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

OUT_MAX, OUT_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module")
def dma():
    from doge_dynamic_mask_b200 import build
    build.build()
    from doge_dynamic_mask_b200 import dma as m
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def sample_rows(L, lengths_b, w, rng, n_rand=12):
    fixed = [0, 1, 127, 128, w - 1, w, w + 1, L // 2, L - 1, lengths_b - 1, min(L - 1, lengths_b)]
    rows = sorted({r for r in fixed if 0 <= r < L} | set(rng.integers(0, L, n_rand).tolist()))
    return rows


@pytest.mark.parametrize("name,heads", [("dense_eq", (0, 7)), ("sparse_pad", (0, 5)), ("long", (0, 9, 15))])
def test_prefill_full_size_sampled(dma, name, heads):
    wl = WORKLOADS[name]
    x = make_inputs(wl, device="cuda")
    ws = dma.new_workspace(dma.dma_workspace_size(wl.B, wl.L, wl.L, wl.Hq, wl.Hkv, wl.d, wl.w))
    out = dma.dma_forward_prefill(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w, workspace=ws)
    assert dma.dma_check(ws) == 0
    lengths = x["lengths"].cpu().numpy()
    W, A = x["W"].double().cpu().numpy(), x["A"].double().cpu().numpy()
    rng = np.random.default_rng(7)
    batches = sorted({0, wl.B - 1})
    errs = []
    for b in batches:
        q = f64(x["q"][b:b + 1])
        k = f64(x["k"][b:b + 1])
        v = f64(x["v"][b:b + 1])
        dt = oracle.dt_scores(v, W, A)                      # [1, Hkv, L] float32
        rows = sample_rows(wl.L, int(lengths[b]), wl.w, rng)
        # tau of the sampled rows, bit-exact, from the same float32 dt
        tau = torch.empty((1, wl.Hkv, wl.L), dtype=torch.int64, device="cuda")
        dma.dma_build_mask(torch.from_numpy(dt).cuda(), x["lengths"][b:b + 1].clone(), wl.L, wl.w, tau_out=tau)
        got_tau = tau.cpu().numpy().view(np.uint64)
        for g in sorted({h // (wl.Hq // wl.Hkv) for h in heads}):
            for i in rows:
                assert int(got_tau[0, g, i]) == oracle.threshold_row(dt[0, g], int(lengths[b]), wl.L, wl.L, wl.w, i)
        got = f64(out[b])
        for h in heads:
            want = oracle.prefill_rows(q, k, v, dt, lengths[b:b + 1], wl.w, wl.scale, 0, h, rows)
            errs.append(np.abs(got[rows, h, :] - want))
    err = np.concatenate([e.ravel() for e in errs])
    assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN, (err.max(), err.mean())


def test_decode_full_size_sampled(dma):
    wl = WORKLOADS["decode"]
    x = make_inputs(wl, device="cuda")
    ws = dma.new_workspace(dma.dma_workspace_size(wl.B, 1, wl.L, wl.Hq, wl.Hkv, wl.d, wl.w))
    out = dma.dma_decode_step(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w, workspace=ws)
    assert dma.dma_check(ws) == 0
    lengths = x["lengths"].cpu().numpy()
    W, A = x["W"].double().cpu().numpy(), x["A"].double().cpu().numpy()
    got = f64(out)
    errs = []
    for b in (0, 37, wl.B - 1):
        want = oracle.decode_step(f64(x["q"][b:b + 1]), f64(x["k"][b:b + 1]), f64(x["v"][b:b + 1]), W, A,
                                  lengths[b:b + 1], wl.w, wl.scale)
        errs.append(np.abs(got[b] - want[0]))
    err = np.concatenate([e.ravel() for e in errs])
    assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN, (err.max(), err.mean())
