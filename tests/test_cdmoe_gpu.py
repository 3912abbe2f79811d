"""Parity of the CDMoE routing kernels (through the C ABI) with the CPU oracle.

Bars:
  kept experts   bit-exact (indices, order and float32 scores), given the same
                 float32 router logits (the oracle's, passed as logits_in)
  router logits  relative error <= 1e-4 against float64 (bf16 products are
                 exact in float32; the tensor core accumulates in float32)
  routed output  |got - want| <= 2^-8 |want| + 2e-3 * max|want| (float32
                 arithmetic, one rounding to bf16; the absolute part covers the
                 cancellation of a sum of 64 signed contributions)
"""
import numpy as np
import pytest
import torch

import oracle
from doge_dynamic_mask_b200.workloads import make_cdmoe_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dma():
    from doge_dynamic_mask_b200 import build
    build.build()
    from doge_dynamic_mask_b200 import dma as m
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_routed_close(got, want, what):
    g = f64(got)
    assert np.isfinite(g).all(), what
    bound = 2.0 ** -8 * np.abs(want) + 2e-3 * np.abs(want).max()
    bad = np.abs(g - want) > bound
    assert not bad.any(), f"{what}: {bad.sum()} outside, max err {np.abs(g - want).max():.3e}"


@pytest.mark.parametrize("T,hidden,num_experts,k", [
    (37, 256, 1024, 8),
    (130, 512, 4096, 16),
    (64, 1024, 16384, 64),       # DogeConfig's num_experts and num_experts_per_tok
    (3, 64, 256, 16),            # top_k = K: every key of both domains kept
    (5, 128, 256, 1),
])
def test_route_bit_exact_and_output_given_oracle_logits(dma, T, hidden, num_experts, k):
    x = make_cdmoe_inputs(T, hidden, num_experts, seed=T + k)
    logits = oracle.cdmoe_logits(f64(x["h"]), f64(x["W_router"]).T).astype(np.float32)
    want_out, want_e, want_s = oracle.cdmoe(f64(x["h"]), None, f64(x["down_embed"]), f64(x["up_embed"]), k,
                                            logits=logits)
    d = {n: v.cuda() for n, v in x.items()}
    ex = torch.empty((T, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((T, k), dtype=torch.float32, device="cuda")
    out = dma.dma_cdmoe_forward(d["h"], d["W_router"], d["down_embed"], d["up_embed"], k,
                                logits_in=torch.from_numpy(logits).cuda(), experts_out=ex, scores_out=sc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ex.cpu().numpy(), want_e)
    np.testing.assert_array_equal(sc.cpu().numpy(), want_s)
    assert_routed_close(out, want_out, "routed output")


def test_route_ties_go_to_lower_indices(dma):
    """Constant logits: every key ties; the lower indices win in both domains and in the product."""
    T, hidden, num_experts, k = 4, 64, 1024, 8
    x = make_cdmoe_inputs(T, hidden, num_experts, seed=9)
    d = {n: v.cuda() for n, v in x.items()}
    logits = torch.full((T, 64), 0.25, dtype=torch.float32, device="cuda")
    ex = torch.empty((T, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((T, k), dtype=torch.float32, device="cuda")
    dma.dma_cdmoe_forward(d["h"], d["W_router"], d["down_embed"], d["up_embed"], k, logits_in=logits,
                          experts_out=ex, scores_out=sc)
    torch.cuda.synchronize()
    assert ex.cpu().tolist() == [list(range(k))] * T
    assert (sc.cpu() == 0.5).all()


def test_full_path_with_router_gemm(dma):
    """The tensor-core router GEMM: logits within 1e-4 of float64; then the
    whole path (logits, routing, experts) against the oracle routed on the
    GPU's own logits is checked through the outputs, with near-tie flips
    allowed only where the oracle's two candidate scores are within the
    logits' error."""
    T, hidden, num_experts, k = 256, 1024, 16384, 64
    x = make_cdmoe_inputs(T, hidden, num_experts, seed=21)
    d = {n: v.cuda() for n, v in x.items()}
    ws = dma.new_workspace(dma.dma_cdmoe_workspace_size(T, num_experts))
    ex = torch.empty((T, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((T, k), dtype=torch.float32, device="cuda")
    out = dma.dma_cdmoe_forward(d["h"], d["W_router"], d["down_embed"], d["up_embed"], k, experts_out=ex,
                                scores_out=sc, workspace=ws)
    assert dma.dma_check(ws) == 0
    got_logits = ws[256:256 + T * 256 * 4].view(torch.float32).view(T, 256).cpu().numpy().astype(np.float64)
    want_logits = oracle.cdmoe_logits(f64(x["h"]), f64(x["W_router"]).T)
    err = np.abs(got_logits - want_logits)
    assert (err <= 1e-4 * np.abs(want_logits) + 1e-6).all(), err.max()
    want_out, want_e, _ = oracle.cdmoe(f64(x["h"]), None, f64(x["down_embed"]), f64(x["up_embed"]), k,
                                       logits=want_logits.astype(np.float32))
    same = (ex.cpu().numpy() == want_e).all(axis=1)
    assert same.mean() >= 0.9, same.mean()          # expert sets differ only on rare near-ties
    assert_routed_close(out[torch.from_numpy(same)], want_out[same], "routed output (same experts)")
