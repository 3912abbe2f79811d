"""Parity of the prologue kernel (through the C ABI) with the CPU oracle:
q/k RMSNorm over head_dim, rotary embedding, KV-cache append.

Bar (derived from the arithmetic): the kernel works in float32 and rounds
each output once to bf16, so it may differ from the float64 oracle by the
rounding (at most 2^-8 of the value) plus float32 error (~1e-7 of the
operands): |got - want| <= 2^-8 |want| + 1e-4.  V rows are copied, and cache
rows outside the written range must be untouched: both bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from doge_dynamic_mask_b200.workloads import make_prologue_inputs

pytestmark = pytest.mark.gpu

RTOL = 2.0 ** -8
ATOL = 1e-4


@pytest.fixture(scope="module")
def dma():
    from doge_dynamic_mask_b200 import build
    build.build()
    from doge_dynamic_mask_b200 import dma as m
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_bf16_close(got, want, what):
    g = f64(got)
    assert np.isfinite(g).all(), what
    bad = np.abs(g - want) > RTOL * np.abs(want) + ATOL
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside the bound, max err {np.abs(g - want).max():.3e}"


def run_case(dma, B, L, Lmax, Hq, Hkv, d, theta, seed, positions=None):
    xh = make_prologue_inputs(B, L, Lmax, Hq, Hkv, d, seed, positions=positions)
    x = {k: v.cuda() for k, v in xh.items()}
    kc, vc = x["k_cache"].clone(), x["v_cache"].clone()
    ws = dma.new_workspace(256)
    q_out = dma.dma_prologue(x["q"], x["k"], x["v"], x["q_w"], x["k_w"], x["positions"], kc, vc,
                             eps=1e-6, rope_theta=theta, workspace=ws)
    status = dma.dma_check(ws)
    return xh, q_out, kc, vc, status


@pytest.mark.parametrize("B,L,Lmax,Hq,Hkv,d,theta", [
    (3, 37, 100, 8, 4, 64, 10000.0),
    (2, 129, 300, 16, 8, 128, 10000.0),
    (1, 5, 70000, 4, 1, 128, 500000.0),        # positions near 2^16: angles need double precision
    (4, 1, 33, 12, 4, 64, 10000.0),            # one new token per sequence (a decode step)
    (2, 17, 17, 2, 2, 64, 1000.0),             # the whole cache written
    # several ring stages per CTA with a ragged last stage (the stage ring
    # wraps, the copy warp refills slots, cache rows cycle through their slots)
    (2, 3000, 3100, 8, 4, 64, 10000.0),        # 16-token stages, two per CTA
    (1, 20000, 20000, 2, 2, 64, 10000.0),      # 16-token stages, five per CTA
    (1, 12000, 12500, 4, 2, 128, 10000.0),     # 115 KB of shared memory: one CTA per SM
])
def test_prologue_matches_oracle(dma, B, L, Lmax, Hq, Hkv, d, theta):
    positions = None if Lmax != 70000 else [Lmax - L]
    xh, q_out, kc, vc, status = run_case(dma, B, L, Lmax, Hq, Hkv, d, theta, seed=B * 1000 + L, positions=positions)
    assert status == 0
    want_q, want_kc, want_vc = oracle.prologue(f64(xh["q"]), f64(xh["k"]), f64(xh["v"]), f64(xh["q_w"]),
                                               f64(xh["k_w"]), 1e-6, theta, xh["positions"].numpy(),
                                               f64(xh["k_cache"]), f64(xh["v_cache"]))
    assert_bf16_close(q_out, want_q, "q")
    for b in range(B):
        p = int(xh["positions"][b])
        rows = slice(p, p + L)
        assert_bf16_close(kc[b, rows], want_kc[b, rows], f"k rows of sequence {b}")
        assert torch.equal(vc[b, rows].cpu(), xh["v"][b])                    # V appended bit for bit
        rest = np.ones(Lmax, bool)
        rest[rows] = False
        assert torch.equal(kc[b].cpu()[rest], xh["k_cache"][b][rest])        # other rows untouched
        assert torch.equal(vc[b].cpu()[rest], xh["v_cache"][b][rest])


def test_prologue_reports_tokens_outside_the_cache(dma):
    B, L, Lmax, Hq, Hkv, d = 2, 8, 40, 4, 2, 64
    p0 = Lmax - L + 3                 # sequence 0: its last three tokens fall past the cache
    xh, q_out, kc, vc, status = run_case(dma, B, L, Lmax, Hq, Hkv, d, 10000.0, seed=5, positions=[p0, 4])
    assert dma.STATUS[status] == "DMA_ERR_BAD_POSITION"
    # the oracle on a cache three rows longer, where every token fits
    big = np.zeros((B, Lmax + 3, Hkv, d))
    want_q, want_kc, want_vc = oracle.prologue(f64(xh["q"]), f64(xh["k"]), f64(xh["v"]), f64(xh["q_w"]),
                                               f64(xh["k_w"]), 1e-6, 10000.0, np.array([p0, 4]), big, big)
    assert_bf16_close(q_out, want_q, "q (written for every token)")
    assert_bf16_close(kc[0, p0:], want_kc[0, p0:Lmax], "k rows of sequence 0 that fit")
    assert torch.equal(kc[0, :p0].cpu(), xh["k_cache"][0, :p0])          # nothing wrapped around
    assert torch.equal(vc[0, :p0].cpu(), xh["v_cache"][0, :p0])
    assert torch.equal(vc[0, p0:].cpu(), xh["v"][0, :Lmax - p0])
    assert_bf16_close(kc[1, 4:4 + L], want_kc[1, 4:4 + L], "k rows of sequence 1")


def test_prologue_long_workload_sampled(dma):
    """Long-context geometry (B=1, L=32768, Hq=16, Hkv=8, d=128) written at the
    start of a 32768-row cache; sampled tokens checked against the oracle."""
    B, L, Lmax, Hq, Hkv, d = 1, 32768, 32768, 16, 8, 128
    xh, q_out, kc, vc, status = run_case(dma, B, L, Lmax, Hq, Hkv, d, 10000.0, seed=77, positions=[0])
    assert status == 0
    rng = np.random.default_rng(0)
    toks = np.unique(np.concatenate([[0, 1, 127, 128, L - 1], rng.integers(0, L, 60)]))
    for t in toks:
        t = int(t)
        one = lambda a: f64(a[:, t:t + 1])
        wq, wk, _ = oracle.prologue(one(xh["q"]), one(xh["k"]), one(xh["v"]), f64(xh["q_w"]), f64(xh["k_w"]), 1e-6,
                                    10000.0, np.array([t]), np.zeros((1, t + 1, Hkv, d)), np.zeros((1, t + 1, Hkv, d)))
        assert_bf16_close(q_out[:, t:t + 1], wq, f"q token {t}")
        assert_bf16_close(kc[:, t:t + 1], wk[:, t:t + 1], f"k token {t}")
        assert torch.equal(vc[0, t].cpu(), xh["v"][0, t])
