"""Pins for the oracle's CDMoE routing (router logits, top-k per domain, the
k best of their Cartesian product, the embedding-table experts), each against
something other than the oracle: brute force over every expert, closed forms,
torch.topk, hand-worked values.  Planted mistakes must fail them.

Cited page: "Transformers 中的 Doge 小语言模型完全指南" ([Guide]), section
"跨域 MoE（CDMoE）" and section "DogeConfig 全参数详解" (num_experts,
num_experts_per_tok, hidden_act).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.dma_oracle as om


def check_logits(cdmoe_logits):
    rng = np.random.default_rng(0)
    h = rng.standard_normal((3, 5))
    W = rng.standard_normal((5, 8))
    got = cdmoe_logits(h, W)
    for t in range(3):
        for c in range(8):
            assert got[t, c] == pytest.approx(sum(h[t, i] * W[i, c] for i in range(5)), rel=1e-13)


def check_route(cdmoe_route):
    rng = np.random.default_rng(1)
    # tie-free logits: the k best of the per-domain product are the k best of all K*K experts
    for K, k in ((6, 3), (8, 8), (5, 1), (16, 4)):
        logits = rng.standard_normal((7, 2 * K)).astype(np.float32)
        experts, scores = cdmoe_route(logits, k)
        for t in range(7):
            allsum = (logits[t, :K][:, None] + logits[t, K:][None, :]).astype(np.float32).ravel()
            best = sorted(range(K * K), key=lambda e: (-float(allsum[e]), e))[:k]
            assert experts[t].tolist() == best
            np.testing.assert_array_equal(scores[t], allsum[best])
    # constant logits: every key ties, the lower indices win in both domains and in the product
    K, k = 8, 4
    experts, scores = cdmoe_route(np.full((2, 2 * K), 0.5, np.float32), k)
    assert experts.tolist() == [[0, 1, 2, 3]] * 2
    np.testing.assert_array_equal(scores, 1.0)
    # per-domain selection agrees with torch.topk on tie-free rows
    K, k = 12, 5
    logits = rng.standard_normal((4, 2 * K)).astype(np.float32)
    experts, _ = cdmoe_route(logits, k)
    tx = torch.topk(torch.from_numpy(logits[:, :K]), k).indices.numpy()
    ty = torch.topk(torch.from_numpy(logits[:, K:]), k).indices.numpy()
    for t in range(4):
        assert set((experts[t] // K).tolist()) <= set(tx[t].tolist())
        assert set((experts[t] % K).tolist()) <= set(ty[t].tolist())
        assert experts[t][0] == tx[t][0] * K + ty[t][0]        # the best pair is the two best keys


def check_experts(cdmoe_experts):
    rng = np.random.default_rng(2)
    hid, E = 6, 9
    h = rng.standard_normal((2, hid))
    D = rng.standard_normal((E, hid))
    U = rng.standard_normal((E, hid))
    # one expert: weight 1, silu(h . d) u
    out = cdmoe_experts(h, np.array([[4], [7]]), np.array([[0.3], [-2.0]], np.float32), D, U)
    for t, e in ((0, 4), (1, 7)):
        a = float(h[t] @ D[e])
        np.testing.assert_allclose(out[t], a / (1 + math.exp(-a)) * U[e], rtol=1e-13)
    # hand-worked two experts: scores (log 3, 0) -> weights (3/4, 1/4)
    h1 = np.array([[1.0, 0.0]])
    D1 = np.array([[2.0, 0.0], [0.0, 5.0]])             # h . d = 2 and 0
    U1 = np.array([[1.0, 0.0], [0.0, 1.0]])
    out = cdmoe_experts(h1, np.array([[0, 1]]), np.array([[math.log(3.0), 0.0]]), D1, U1)
    np.testing.assert_allclose(out[0], [0.75 * 2.0 / (1 + math.exp(-2.0)), 0.0], rtol=1e-13, atol=1e-15)
    # equal scores: the plain mean of the experts' contributions
    ex = np.array([[1, 2, 3], [0, 5, 8]])
    out = cdmoe_experts(h, ex, np.zeros((2, 3), np.float32), D, U)
    for t in range(2):
        a = D[ex[t]] @ h[t]
        np.testing.assert_allclose(out[t], ((a / (1 + np.exp(-a)))[:, None] * U[ex[t]]).mean(0), rtol=1e-12)
    # linear in the up-projection table
    sc = rng.standard_normal((2, 3)).astype(np.float32)
    o1 = cdmoe_experts(h, ex, sc, D, U)
    o2 = cdmoe_experts(h, ex, sc, D, 2.5 * U)
    np.testing.assert_allclose(o2, 2.5 * o1, rtol=1e-12)


def test_logits_pins():
    check_logits(oracle.cdmoe_logits)


def test_route_pins():
    check_route(oracle.cdmoe_route)


def test_experts_pins():
    check_experts(oracle.cdmoe_experts)


def test_cdmoe_composes_its_parts():
    rng = np.random.default_rng(3)
    K, k, hid = 8, 3, 10
    h = rng.standard_normal((4, hid))
    W = rng.standard_normal((hid, 2 * K)) * 0.3
    D = rng.standard_normal((K * K, hid))
    U = rng.standard_normal((K * K, hid))
    out, experts, scores = oracle.cdmoe(h, W, D, U, k)
    assert experts.shape == (4, k) and (experts >= 0).all() and (experts < K * K).all()
    assert all(len(set(r)) == k for r in experts.tolist())       # k distinct experts per token
    assert (np.diff(scores, axis=1) <= 0).all()                   # best first


# ---- planted mistakes -------------------------------------------------------

def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_mutant_logits_transposed_is_caught():
    _fails(check_logits, lambda h, W: np.asarray(h) @ np.asarray(W)[::-1])


def _route_factory(swap_domains=False, tie_high=False, index_xy=False):
    def route(logits, k):
        logits = np.asarray(logits, np.float32)
        T, twoK = logits.shape
        K = twoK // 2
        ex = np.empty((T, k), np.int64)
        sc = np.empty((T, k), np.float32)
        for t in range(T):
            lx, ly = logits[t, :K], logits[t, K:]
            if swap_domains:
                lx, ly = ly, lx
            ix = om._topk_stable(lx, k)
            iy = om._topk_stable(ly, k)
            s = (lx[ix][:, None] + ly[iy][None, :]).astype(np.float32).ravel()
            e = ((iy[None, :] * K + ix[:, None]) if index_xy else (ix[:, None] * K + iy[None, :])).ravel()
            key2 = -e if tie_high else e
            o = np.lexsort((key2, -s.astype(np.float64)))[:k]
            ex[t], sc[t] = e[o], s[o]
        return ex, sc
    return route


def test_mutant_route_swapped_domains_is_caught():
    _fails(check_route, _route_factory(swap_domains=True))


def test_mutant_route_tie_break_is_caught():
    _fails(check_route, _route_factory(tie_high=True))


def test_mutant_route_expert_index_order_is_caught():
    _fails(check_route, _route_factory(index_xy=True))


def test_mutant_experts_relu_instead_of_silu_is_caught():
    def bad(h, experts, scores, D, U):
        h = np.asarray(h, np.float64)
        out = np.empty_like(h)
        for t in range(h.shape[0]):
            s = np.asarray(scores[t], np.float64)
            w = np.exp(s - s.max()); w /= w.sum()
            a = np.asarray(D)[experts[t]] @ h[t]
            out[t] = (w * np.maximum(a, 0)) @ np.asarray(U)[experts[t]]
        return out
    _fails(check_experts, bad)


def test_mutant_experts_unnormalised_weights_is_caught():
    def bad(h, experts, scores, D, U):
        h = np.asarray(h, np.float64)
        out = np.empty_like(h)
        for t in range(h.shape[0]):
            w = np.exp(np.asarray(scores[t], np.float64))
            a = np.asarray(D)[experts[t]] @ h[t]
            out[t] = (w * a / (1 + np.exp(-a))) @ np.asarray(U)[experts[t]]
        return out
    _fails(check_experts, bad)
