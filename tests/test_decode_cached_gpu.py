"""Incremental decode with cached dt, through the C ABI, against the oracle.

A decode state is built over the first tokens of each sequence, then a series
of steps extends every sequence by one or more tokens (their K and V already
sit in the caches).  After every step:
  - the output matches the oracle's decode step over the same lengths within
    the output tolerance of every parity test;
  - the kept key set of every (batch, kv head) equals the oracle's selection
    computed from the state's own float32 dt, bit for bit;
  - the state's dt matches the oracle's dt within the dt tolerance.
At the end the output also matches the full-recompute dma_decode_step.
"""
import numpy as np
import pytest
import torch

from doge_dynamic_mask_b200.workloads import Workload, make_inputs
from oracle import dma_oracle as oracle

pytestmark = pytest.mark.gpu

OUT_MAX, OUT_MEAN = 2e-2, 2e-3
DT_RTOL = 1e-5


@pytest.fixture(scope="module")
def dma():
    from doge_dynamic_mask_b200 import build
    build.build()
    from doge_dynamic_mask_b200 import dma as m
    return m


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("Hq,Hkv,d,w,start,grow", [
    (8, 4, 128, 256, (100, 250, 1000), (1, 3, 1)),     # sequence 1 crosses w while growing
    (4, 2, 64, 100, (1, 99, 600), (2, 1, 5)),           # starts below, at and above w
])
def test_cached_steps_match_the_oracle(dma, Hq, Hkv, d, w, start, grow):
    B, Lk = 3, 1200
    wl = Workload("cached", "decode", B=B, L=Lk, Hq=Hq, Hkv=Hkv, d=d, w=w, a_lo=-2.0, a_hi=-0.1, seed=Lk + w)
    x = make_inputs(wl, device="cpu")
    dev = {k: v.cuda() for k, v in x.items()}
    kc, vc = f64(x["k"]), f64(x["v"])
    W, A = x["W"].double().numpy(), x["A"].double().numpy()
    dt_oracle = oracle.dt_scores(vc, W, A)
    lengths = np.array(start, dtype=np.int32)
    state = dma.dma_decode_state_init(dev["v"], dev["W"], dev["A"], torch.from_numpy(lengths).cuda(), w, Hq)
    assert dma.dma_check(state) == 0
    for step in range(6):
        lengths = np.minimum(lengths + np.array(grow, dtype=np.int32), Lk).astype(np.int32)
        lens_dev = torch.from_numpy(lengths).cuda()
        out = dma.dma_decode_step_cached(dev["q"], dev["k"], dev["v"], dev["W"], dev["A"], lens_dev, w, state)
        assert dma.dma_check(state, clear=False) == 0
        want = oracle.decode_step(f64(x["q"]), kc, vc, None, None, lengths, w, wl.scale, dt=dt_oracle)
        err = np.abs(f64(out) - want)
        assert np.isfinite(err).all()
        assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN, (step, err.max(), err.mean())
        dt_s, count, idx = dma.decode_state_views(state, B, Lk, Hq, Hkv, d, w)
        dt_s = dt_s.cpu().numpy()
        for b in range(B):
            n = int(lengths[b])
            rel = np.abs(dt_s[b, :, :n] - dt_oracle[b, :, :n]) / np.abs(dt_oracle[b, :, :n])
            assert rel.max() <= DT_RTOL, (step, b, rel.max())
        kept = oracle.kept_mask(dt_s, lengths, 1, Lk, w)[:, :, 0]
        cnt, ix = count.cpu().numpy(), idx.cpu().numpy()
        for b in range(B):
            for g in range(Hkv):
                got = np.sort(ix[b, g, :cnt[b, g]])
                assert np.array_equal(got, np.nonzero(kept[b, g])[0]), (step, b, g)
    full = dma.dma_decode_step(dev["q"], dev["k"], dev["v"], dev["W"], dev["A"], lens_dev, w)
    diff = np.abs(f64(full) - f64(out))
    assert diff.max() <= OUT_MAX and diff.mean() <= OUT_MEAN


def test_a_shrinking_length_is_reported_and_the_state_kept(dma):
    B, Lk, Hq, Hkv, d, w = 2, 300, 4, 2, 64, 32
    wl = Workload("cached", "decode", B=B, L=Lk, Hq=Hq, Hkv=Hkv, d=d, w=w, a_lo=-2.0, a_hi=-0.1, seed=3)
    dev = {k: v.cuda() for k, v in make_inputs(wl, device="cpu").items()}
    lengths = torch.tensor([200, 100], dtype=torch.int32, device="cuda")
    state = dma.dma_decode_state_init(dev["v"], dev["W"], dev["A"], lengths, w, Hq)
    assert dma.dma_check(state) == 0
    before = state.clone()
    shrunk = torch.tensor([150, 100], dtype=torch.int32, device="cuda")
    dma.dma_decode_step_cached(dev["q"], dev["k"], dev["v"], dev["W"], dev["A"], shrunk, w, state)
    assert dma.dma_check(state) == 6          # DMA_ERR_BAD_LENGTH
    # sequence 0's part of the state is untouched (sequence 1 took in no token)
    dt_a, cnt_a, idx_a = dma.decode_state_views(before, B, Lk, Hq, Hkv, d, w)
    dt_b, cnt_b, idx_b = dma.decode_state_views(state, B, Lk, Hq, Hkv, d, w)
    assert torch.equal(cnt_a, cnt_b) and torch.equal(idx_a, idx_b) and torch.equal(dt_a, dt_b)
