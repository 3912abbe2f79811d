"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars (written here, used everywhere below):
  dt                 relative error <= 1e-5 (float32 path vs float64 oracle)
  masks              bit-exact (tau and the kept-key bitmask), given the same float32 dt
  attention outputs  max-abs <= 2e-2 and mean-abs <= 2e-3 against the float64 oracle (bf16 out)
"""
import numpy as np
import pytest
import torch

import oracle
from doge_dynamic_mask_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

DT_RTOL = 1e-5
OUT_MAX, OUT_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module")
def dma():
    from doge_dynamic_mask_b200 import build
    build.build()
    from doge_dynamic_mask_b200 import dma as m
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_out_close(got, want, what=""):
    err = np.abs(f64(got) - want)
    assert np.isfinite(f64(got)).all(), what
    assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN, f"{what}: max {err.max():.3e} mean {err.mean():.3e}"


def pack_bits(mask):
    """bool [..., Lk] -> uint32 words [..., ceil(Lk/32)], bit j%32 of word j/32."""
    Lk = mask.shape[-1]
    words = (Lk + 31) // 32
    pad = np.zeros(mask.shape[:-1] + (words * 32,), dtype=np.uint64)
    pad[..., :Lk] = mask
    pad = pad.reshape(mask.shape[:-1] + (words, 32))
    return (pad << np.arange(32, dtype=np.uint64)).sum(-1).astype(np.uint32)


def wl(B, L, Hq, Hkv, d, w, a=(-2.0, -0.1), lens=None, seed=0, mode="prefill"):
    lo, hi = (None, None) if lens is None else lens
    return Workload("case", mode, B=B, L=L, Hq=Hq, Hkv=Hkv, d=d, w=w, a_lo=a[0], a_hi=a[1], seed=seed,
                    len_lo=lo, len_hi=hi)


def inputs(w_, device="cuda"):
    x = make_inputs(w_, device="cpu")
    return {k: v.to(device) for k, v in x.items()}, x


# ----------------------------------------------------------------------------
# S1 dt
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("B,L,Hkv,d,a", [
    (1, 256, 2, 64, (-2.0, -0.1)),
    (8, 300, 4, 64, (-2.0, -0.1)),
    (1, 1000, 8, 128, (-4.0, -0.1)),
    (3, 77, 1, 128, (-2.0, -0.1)),
    (2, 129, 16, 64, (-2.0, -0.1)),
    (1, 64, 16, 128, (-2.0, 2.0)),
])
def test_dt_scores(dma, B, L, Hkv, d, a):
    dev, cpu = inputs(wl(B, L, Hkv, Hkv, d, 8, a=a, seed=B * 1000 + L))
    got = f64(dma.dma_dt_scores(dev["v"], dev["W"], dev["A"]))
    want = oracle.dt_scores64(f64(cpu["v"]), cpu["W"].double().numpy(), cpu["A"].double().numpy())
    rel = np.abs(got - want) / np.abs(want)
    assert rel.max() <= DT_RTOL, rel.max()


# ----------------------------------------------------------------------------
# S2 masks (bit-exact, given the same float32 dt)
# ----------------------------------------------------------------------------

def make_dt(kind, B, Hkv, L, seed):
    rng = np.random.default_rng(seed)
    if kind == "random":
        return rng.uniform(0.05, 1.0, size=(B, Hkv, L)).astype(np.float32)
    if kind == "ties":
        return rng.choice(np.array([0.25, 0.5, 0.625, 0.75, 1.0], np.float32), size=(B, Hkv, L))
    if kind == "const":
        return np.ones((B, Hkv, L), np.float32)
    ramp = np.linspace(0.01, 1.0, L, dtype=np.float32)
    if kind == "inc":
        return np.broadcast_to(ramp, (B, Hkv, L)).copy()
    if kind == "dec":
        return np.broadcast_to(ramp[::-1], (B, Hkv, L)).copy()
    raise ValueError(kind)


MASK_CASES = [
    (1, 2, 256, 64, None, "random"),
    (2, 2, 300, 37, [300, 161], "ties"),
    (2, 1, 520, 128, [520, 260], "random"),
    (1, 2, 700, 129, None, "const"),
    (1, 1, 1000, 300, None, "inc"),
    (1, 1, 1000, 300, None, "dec"),
    (3, 2, 257, 1, [257, 1, 100], "random"),
    (2, 2, 200, 500, [200, 150], "random"),
    (1, 2, 130, 127, None, "ties"),
    (1, 4, 5000, 2048, None, "random"),
    (1, 1, 6000, 4500, None, "const"),
]


@pytest.mark.parametrize("B,Hkv,L,w,lens,kind", MASK_CASES)
def test_prefill_mask_bit_exact(dma, B, Hkv, L, w, lens, kind):
    dt = make_dt(kind, B, Hkv, L, seed=L + w)
    lengths = np.array(lens if lens else [L] * B, dtype=np.int32)
    words = (L + 31) // 32
    tau = torch.empty((B, Hkv, L), dtype=torch.int64, device="cuda")
    bm = torch.empty((B, Hkv, L, words), dtype=torch.int32, device="cuda")
    ws = dma.dma_build_mask(torch.from_numpy(dt).cuda(), torch.from_numpy(lengths).cuda(), L, w,
                            tau_out=tau, bitmask_out=bm)
    assert dma.dma_check(ws) == 0
    want_tau = oracle.thresholds(dt, lengths, L, L, w)
    got_tau = tau.cpu().numpy().view(np.uint64)
    assert np.array_equal(got_tau, want_tau), np.argwhere(got_tau != want_tau)[:5]
    want_bm = pack_bits(oracle.kept_mask(dt, lengths, L, L, w))
    got_bm = bm.cpu().numpy().view(np.uint32)
    assert np.array_equal(got_bm, want_bm), np.argwhere(got_bm != want_bm)[:5]


@pytest.mark.parametrize("B,Hkv,Lk,w,lens,kind", [
    (3, 2, 3000, 100, [3000, 50, 2000], "random"),
    (2, 1, 70000, 2048, [70000, 65536], "ties"),
    (2, 2, 5000, 4096, [5000, 4097], "const"),
    (1, 1, 300, 512, None, "random"),
])
def test_decode_mask_bit_exact(dma, B, Hkv, Lk, w, lens, kind):
    dt = make_dt(kind, B, Hkv, Lk, seed=Lk + w)
    lengths = np.array(lens if lens else [Lk] * B, dtype=np.int32)
    words = (Lk + 31) // 32
    tau = torch.empty((B, Hkv, 1), dtype=torch.int64, device="cuda")
    bm = torch.empty((B, Hkv, 1, words), dtype=torch.int32, device="cuda")
    ws = dma.dma_build_mask(torch.from_numpy(dt).cuda(), torch.from_numpy(lengths).cuda(), 1, w,
                            tau_out=tau, bitmask_out=bm)
    assert dma.dma_check(ws) == 0
    assert np.array_equal(tau.cpu().numpy().view(np.uint64), oracle.thresholds(dt, lengths, 1, Lk, w))
    assert np.array_equal(bm.cpu().numpy().view(np.uint32), pack_bits(oracle.kept_mask(dt, lengths, 1, Lk, w)))


# ----------------------------------------------------------------------------
# S3 prefill attention
# ----------------------------------------------------------------------------

PREFILL_CASES = [
    WORKLOADS["tiny"],
    wl(2, 300, 4, 2, 64, 100, lens=(150, 300), seed=11),
    wl(1, 520, 4, 2, 128, 128, seed=12),
    wl(1, 384, 2, 2, 64, 1000, seed=13),
    wl(2, 257, 8, 2, 128, 64, lens=(130, 257), seed=14),
    wl(1, 1100, 6, 2, 64, 256, seed=15),
    wl(1, 1, 2, 1, 64, 4, seed=16),
    wl(1, 200, 2, 1, 128, 1, a=(-4.0, -0.1), seed=17),
    # keep_window_size >= L: no top-k, the attention kernel builds each tile's list itself
    wl(2, 300, 4, 2, 64, 512, lens=(150, 300), seed=18),
    wl(3, 257, 6, 2, 128, 257, lens=(1, 129), seed=19),
]


@pytest.mark.parametrize("w_", PREFILL_CASES, ids=lambda w_: f"B{w_.B}L{w_.L}Hq{w_.Hq}Hkv{w_.Hkv}d{w_.d}w{w_.w}")
def test_prefill_parity(dma, w_):
    dev, cpu = inputs(w_)
    q, k, v = f64(cpu["q"]), f64(cpu["k"]), f64(cpu["v"])
    W, A = cpu["W"].double().numpy(), cpu["A"].double().numpy()
    lengths = cpu["lengths"].numpy()
    dt32 = oracle.dt_scores(v, W, A)
    want = oracle.prefill(q, k, v, None, None, lengths, w_.w, w_.scale, dt=dt32)
    # same float32 dt on both sides: identical masks
    got = dma.dma_forward_prefill(dev["q"], dev["k"], dev["v"], None, None, dev["lengths"], w_.w,
                                  dt_in=torch.from_numpy(dt32).cuda())
    assert_out_close(got, want, "dt_in")
    # whole path (the kernel computes dt itself)
    ws = dma.new_workspace(dma.dma_workspace_size(w_.B, w_.L, w_.L, w_.Hq, w_.Hkv, w_.d, w_.w))
    got2 = dma.dma_forward_prefill(dev["q"], dev["k"], dev["v"], dev["W"], dev["A"], dev["lengths"], w_.w,
                                   workspace=ws)
    assert dma.dma_check(ws) == 0
    assert_out_close(got2, want, "full path")


@pytest.mark.parametrize("w_", [wl(2, 1500, 8, 2, 128, 300, lens=(700, 1500), seed=31),
                                 wl(1, 640, 4, 4, 128, 700, seed=32)],
                         ids=["topk_d128", "dense_d128"])
def test_prefill_repeated_calls_share_a_workspace(dma, w_):
    """At d = 128 the attention CTAs draw their work items from a counter in
    the workspace header, which the last CTA resets: repeated calls on one
    workspace must each cover every item exactly once (each matches the
    oracle) and leave the counter words at zero.  Without a top-k the lists
    are built in key order, so the calls agree bit for bit; with one, the
    order inside a list class is free (warps reserve their segments), so the
    float32 sums may round differently from call to call."""
    dev, cpu = inputs(w_)
    q, k, v = f64(cpu["q"]), f64(cpu["k"]), f64(cpu["v"])
    W, A = cpu["W"].double().numpy(), cpu["A"].double().numpy()
    dt32 = oracle.dt_scores(v, W, A)
    want = oracle.prefill(q, k, v, None, None, cpu["lengths"].numpy(), w_.w, w_.scale, dt=dt32)
    ws = dma.new_workspace(dma.dma_workspace_size(w_.B, w_.L, w_.L, w_.Hq, w_.Hkv, w_.d, w_.w))
    outs = []
    for _ in range(3):
        outs.append(dma.dma_forward_prefill(dev["q"], dev["k"], dev["v"], dev["W"], dev["A"], dev["lengths"], w_.w,
                                            workspace=ws).clone())
        assert dma.dma_check(ws) == 0
        header = ws[:256].view(torch.int32).cpu()
        assert int(header[16]) == 0 and int(header[17]) == 0, "work-item counter (bytes 64-71) not reset"
    for i, o in enumerate(outs):
        assert_out_close(o, want, f"call {i}")
    if w_.w >= w_.L:
        for o in outs[1:]:
            assert torch.equal(o, outs[0]), "a repeated call differs"


# ----------------------------------------------------------------------------
# S4 decode
# ----------------------------------------------------------------------------

DECODE_CASES = [
    wl(2, 3000, 4, 2, 128, 256, lens=(1000, 3000), seed=21, mode="decode"),
    wl(3, 700, 8, 4, 64, 1000, lens=(1, 700), seed=22, mode="decode"),
    wl(1, 4096, 16, 8, 128, 2048, seed=23, mode="decode"),
    wl(2, 333, 2, 2, 64, 7, seed=24, mode="decode"),
]


@pytest.mark.parametrize("w_", DECODE_CASES, ids=lambda w_: f"B{w_.B}Lk{w_.L}Hq{w_.Hq}Hkv{w_.Hkv}d{w_.d}w{w_.w}")
def test_decode_parity(dma, w_):
    dev, cpu = inputs(w_)
    q, kc, vc = f64(cpu["q"]), f64(cpu["k"]), f64(cpu["v"])
    W, A = cpu["W"].double().numpy(), cpu["A"].double().numpy()
    lengths = cpu["lengths"].numpy()
    dt32 = oracle.dt_scores(vc, W, A)
    want = oracle.decode_step(q, kc, vc, None, None, lengths, w_.w, w_.scale, dt=dt32)
    got = dma.dma_decode_step(dev["q"], dev["k"], dev["v"], None, None, dev["lengths"], w_.w,
                              dt_in=torch.from_numpy(dt32).cuda())
    assert_out_close(got, want, "dt_in")
    ws = dma.new_workspace(dma.dma_workspace_size(w_.B, 1, w_.L, w_.Hq, w_.Hkv, w_.d, w_.w))
    got2 = dma.dma_decode_step(dev["q"], dev["k"], dev["v"], dev["W"], dev["A"], dev["lengths"], w_.w,
                               workspace=ws)
    assert dma.dma_check(ws) == 0
    assert_out_close(got2, want, "full path")


# ----------------------------------------------------------------------------
# errors reported through the status word
# ----------------------------------------------------------------------------

def test_bad_length_is_reported_and_clamped(dma):
    w_ = wl(2, 160, 2, 1, 64, 32, seed=31)
    dev, _ = inputs(w_)
    bad = torch.tensor([0, 999], dtype=torch.int32, device="cuda")
    ws = dma.new_workspace(dma.dma_workspace_size(2, 160, 160, 2, 1, 64, 32))
    out = dma.dma_forward_prefill(dev["q"], dev["k"], dev["v"], dev["W"], dev["A"], bad, 32, workspace=ws)
    assert dma.dma_check(ws) == 6            # DMA_ERR_BAD_LENGTH
    assert torch.isfinite(out.float()).all()
    assert dma.dma_check(ws) == 0            # cleared by the first check


def test_small_workspace_is_rejected(dma):
    w_ = wl(1, 128, 2, 1, 64, 32, seed=32)
    dev, _ = inputs(w_)
    ws = dma.new_workspace(64)
    with pytest.raises(dma.DMAError) as e:
        dma.dma_forward_prefill(dev["q"], dev["k"], dev["v"], dev["W"], dev["A"], None, 32, workspace=ws)
    assert e.value.status == 3
