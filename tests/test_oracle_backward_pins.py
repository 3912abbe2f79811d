"""Pins for the oracle's prefill backward (kept-key selection held fixed):
float64 torch.autograd through an independently written forward (explicit
torch ops, the kept sets by brute-force rank counting), central finite
differences, and planted mistakes that must fail them.

Cited page: "Transformers 中的 Doge 小语言模型完全指南" ([Guide]), section
"动态掩码注意力（DMA）", step 3 and its closing paragraph (dt learnt end to end).
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.dma_oracle as om
from tests.test_oracle_pins import brute_kept


def _case(seed, B=2, L=13, Hq=4, Hkv=2, d=6, w=4):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, L, Hq, d))
    k = rng.standard_normal((B, L, Hkv, d))
    v = rng.standard_normal((B, L, Hkv, d))
    W = rng.standard_normal((Hkv * d, Hkv)) * 0.4
    A = -rng.uniform(0.2, 2.0, Hkv)
    lengths = np.array([L, L - 4][:B])
    dout = rng.standard_normal((B, L, Hq, d))
    return q, k, v, W, A, lengths, w, 0.37, dout


def _autograd(q, k, v, W, A, lengths, w, scale, dout):
    """Forward in torch float64 ops, kept sets from the float32 dt by rank
    counting (then fixed), gradients by autograd."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    n_rep = Hq // Hkv
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    tW, tA = torch.tensor(W, requires_grad=True), torch.tensor(A, requires_grad=True)
    x = torch.einsum("blc,cg->blg", tv.reshape(B, L, Hkv * d), tW)
    dt = torch.exp(tA * torch.nn.functional.softplus(x)).permute(0, 2, 1)     # [B, Hkv, L]
    dt32 = dt.detach().numpy().astype(np.float32)
    # the mask holds dt rounded to float32; the rounding passes gradients unchanged
    dt = dt + (torch.from_numpy(dt32.astype(np.float64)) - dt).detach()
    outs = []
    for b in range(B):
        for h in range(Hq):
            g = h // n_rep
            kept = np.zeros((L, L), bool)
            for i in range(L):
                for j in brute_kept(dt32[b, g], int(lengths[b]), L, L, w, i):
                    kept[i, j] = True
            bias = torch.where(torch.from_numpy(kept), dt[b, g][None, :].expand(L, L),
                               torch.full((L, L), float("-inf"), dtype=torch.float64))
            s = scale * tq[b, :, h, :] @ tk[b, :, g, :].T + bias
            p = torch.softmax(s, dim=-1)
            outs.append(((p @ tv[b, :, g, :]) * torch.from_numpy(dout[b, :, h, :])).sum())
    torch.stack(outs).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy(), tW.grad.numpy(), tA.grad.numpy()


def check_backward_autograd(prefill_backward, seed=0):
    for Hq, Hkv in ((4, 2), (3, 3), (6, 2)):
        args = _case(seed + Hq, Hq=Hq, Hkv=Hkv)
        dq, dk, dv, d_dt, dW, dA = prefill_backward(*args)
        gq, gk, gv, gW, gA = _autograd(*args)
        for got, want in ((dq, gq), (dk, gk), (dv, gv), (dW, gW), (dA, gA)):
            np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-11)


def check_backward_finite_differences(prefill_backward):
    """Central differences of sum(out * dout) in a few coordinates.  The mask
    holds dt rounded to float32, a staircase in W and A with steps of one
    float32 ulp, so the step is 1e-3 (thousands of ulps of dt) and the bar
    2e-3 relative; the kept sets are checked to stay the same across each step."""
    q, k, v, W, A, lengths, w, scale, dout = _case(5, B=1, L=9, Hq=2, Hkv=1, d=4, w=3)
    dq, dk, dv, _, dW, dA = prefill_backward(q, k, v, W, A, lengths, w, scale, dout)
    kept0 = oracle.kept_mask(oracle.dt_scores(v, W, A), lengths, 9, 9, w)

    def loss(q_, k_, v_, W_, A_):
        assert np.array_equal(oracle.kept_mask(oracle.dt_scores(v_, W_, A_), lengths, 9, 9, w), kept0)
        return float((oracle.prefill(q_, k_, v_, W_, A_, lengths, w, scale) * dout).sum())

    eps = 1e-3
    for name, arr, grad, idx in (("q", q, dq, (0, 7, 1, 2)), ("k", k, dk, (0, 3, 0, 1)), ("v", v, dv, (0, 5, 0, 3)),
                                 ("W", W, dW, (2, 0)), ("A", A, dA, (0,))):
        plus, minus = arr.copy(), arr.copy()
        plus[idx] += eps
        minus[idx] -= eps
        argsp = {"q": q, "k": k, "v": v, "W": W, "A": A}
        argsm = dict(argsp)
        argsp[name], argsm[name] = plus, minus
        fd = (loss(*argsp.values()) - loss(*argsm.values())) / (2 * eps)
        assert grad[idx] == pytest.approx(fd, rel=2e-3, abs=1e-6), name


def test_backward_matches_autograd():
    check_backward_autograd(oracle.prefill_backward)


def test_backward_matches_finite_differences():
    check_backward_finite_differences(oracle.prefill_backward)


def test_backward_d_dt_is_the_bias_gradient():
    """d_dt is the gradient with respect to the float32 dt the mask holds: with
    the dt chain cut (A = 0 makes dt identically 1 and dx zero), d_dt still
    equals autograd's gradient with respect to a free bias on the kept keys."""
    q, k, v, W, A, lengths, w, scale, dout = _case(8)
    A = np.zeros_like(A)
    _, _, _, d_dt, dW, dA = oracle.prefill_backward(q, k, v, W, A, lengths, w, scale, dout)
    np.testing.assert_array_equal(dW, 0.0)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    bias = torch.ones((B, Hkv, L), dtype=torch.float64, requires_grad=True)
    tot = 0
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            kept = np.zeros((L, L), bool)
            for i in range(L):
                for j in brute_kept(np.ones(L, np.float32), int(lengths[b]), L, L, w, i):
                    kept[i, j] = True
            s = scale * torch.from_numpy(q[b, :, h, :] @ k[b, :, g, :].T) + torch.where(
                torch.from_numpy(kept), bias[b, g][None, :].expand(L, L), torch.tensor(float("-inf"), dtype=torch.float64))
            tot = tot + ((torch.softmax(s, -1) @ torch.from_numpy(v[b, :, g, :])) * torch.from_numpy(dout[b, :, h, :])).sum()
    tot.backward()
    np.testing.assert_allclose(d_dt, bias.grad.numpy(), rtol=1e-9, atol=1e-12)


# ---- planted mistakes -------------------------------------------------------

def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def _mutant(drop_delta=False, no_dt_path=False, no_A_in_dx=False):
    def bwd(q, k, v, W, A, lengths, w, scale, dout, dt_fixed=None):
        q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
        W = np.asarray(W, np.float64); A = np.asarray(A, np.float64); dout = np.asarray(dout, np.float64)
        B, L, Hq, d = q.shape
        Hkv = k.shape[2]
        n_rep = Hq // Hkv
        x = v.reshape(B, L, Hkv * d) @ W
        sp = om.softplus(x)
        dt64 = np.exp(A[None, None, :] * sp)
        dt32 = dt64.transpose(0, 2, 1).astype(np.float32)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        d_dt = np.zeros((B, Hkv, L))
        for b in range(B):
            for g in range(Hkv):
                M = om.dynamic_mask_rows(dt32[b, g], int(lengths[b]), L, L, w, range(L))
                for r in range(n_rep):
                    h = g * n_rep + r
                    s = scale * (q[b, :, h] @ k[b, :, g].T) + M
                    P = np.exp(s - s.max(1, keepdims=True)); P /= P.sum(1, keepdims=True)
                    dP = dout[b, :, h] @ v[b, :, g].T
                    Dr = 0.0 if drop_delta else (dout[b, :, h] * (P @ v[b, :, g])).sum(1, keepdims=True)
                    dS = P * (dP - Dr)
                    dq[b, :, h] = scale * dS @ k[b, :, g]
                    dk[b, :, g] += scale * dS.T @ q[b, :, h]
                    dv[b, :, g] += P.T @ dout[b, :, h]
                    d_dt[b, g] += dS.sum(0)
        ddt = d_dt.transpose(0, 2, 1)
        dA = (ddt * dt64 * sp).sum((0, 1))
        dx = ddt * dt64 * (1.0 if no_A_in_dx else A[None, None, :]) / (1 + np.exp(-x))
        dW = v.reshape(B * L, -1).T @ dx.reshape(B * L, Hkv)
        if not no_dt_path:
            dv += (dx.reshape(B * L, Hkv) @ W.T).reshape(B, L, Hkv, d)
        return dq, dk, dv, d_dt, dW, dA
    return bwd


def test_mutant_backward_without_delta_is_caught():
    _fails(check_backward_autograd, _mutant(drop_delta=True))


def test_mutant_backward_without_dt_path_in_dv_is_caught():
    _fails(check_backward_autograd, _mutant(no_dt_path=True))


def test_mutant_backward_dt_chain_missing_A_is_caught():
    _fails(check_backward_finite_differences, _mutant(no_A_in_dx=True))
