"""Failure detection and write bounds on the GPU, without faulting it.

- A bounded wait that runs out: the diagnostic entry point waits on a barrier
  nothing completes; the wait gives up after about a second, the status word
  reports DMA_ERR_TIMEOUT, and the context stays usable for the next call.
- Canary words: every output buffer is the middle of a larger buffer filled
  with a pattern; after the call the pattern around it must be intact (the
  kernels write nowhere outside their outputs).
"""
import time

import numpy as np
import pytest
import torch

from doge_dynamic_mask_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

PAD = 4096   # bytes of canary on each side (a multiple of 16)


@pytest.fixture(scope="module")
def dma():
    from doge_dynamic_mask_b200 import build
    build.build()
    from doge_dynamic_mask_b200 import dma as m
    return m


def guarded(shape, dtype):
    """(view of the output, checker): the view sits between two canary zones."""
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((n + 2 * PAD,), 0xA5, dtype=torch.uint8, device="cuda")
    view = raw[PAD:PAD + n].view(dtype).view(*shape)

    def intact():
        torch.cuda.synchronize()
        return bool((raw[:PAD] == 0xA5).all()) and bool((raw[PAD + n:] == 0xA5).all())
    return view, intact


def test_a_bounded_wait_runs_out_and_is_reported(dma):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    dma.dma_selftest_wait(ws)
    assert dma.dma_check(ws) == 5            # DMA_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 0.1 < elapsed < 30.0, elapsed
    assert dma.dma_check(ws) == 0            # cleared
    # the context is still usable
    wl = Workload("after", "prefill", B=1, L=256, Hq=4, Hkv=2, d=64, w=64, a_lo=-2.0, a_hi=-0.1, seed=0)
    x = {k: v.cuda() for k, v in make_inputs(wl).items()}
    out = dma.dma_forward_prefill(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w)
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("L,w,d,lens", [(300, 100, 64, (150, 300)), (257, 64, 128, None), (384, 1000, 64, (200, 384))])
def test_prefill_and_dt_write_only_their_outputs(dma, L, w, d, lens):
    lo, hi = (None, None) if lens is None else lens
    wl = Workload("canary", "prefill", B=2, L=L, Hq=4, Hkv=2, d=d, w=w, a_lo=-2.0, a_hi=-0.1, seed=L,
                  len_lo=lo, len_hi=hi)
    x = {k: v.cuda() for k, v in make_inputs(wl).items()}
    out, ok_out = guarded(tuple(x["q"].shape), torch.bfloat16)
    dma.dma_forward_prefill(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], w, out=out)
    assert ok_out()
    dt, ok_dt = guarded((2, 2, L), torch.float32)
    dma.dma_dt_scores(x["v"], x["W"], x["A"], dt_out=dt)
    assert ok_dt()


def test_mask_outputs_write_only_their_buffers(dma):
    B, Hkv, L, w = 2, 2, 300, 37
    dt = torch.rand((B, Hkv, L), dtype=torch.float32, device="cuda") + 0.01
    lengths = torch.tensor([300, 161], dtype=torch.int32, device="cuda")
    tau, ok_tau = guarded((B, Hkv, L), torch.int64)
    words = (L + 31) // 32
    bm, ok_bm = guarded((B, Hkv, L, words), torch.int32)
    ws = dma.dma_build_mask(dt, lengths, L, w, tau_out=tau, bitmask_out=bm)
    assert dma.dma_check(ws) == 0
    assert ok_tau() and ok_bm()


@pytest.mark.parametrize("cached", [False, True])
def test_decode_writes_only_its_output(dma, cached):
    wl = Workload("canary", "decode", B=3, L=700, Hq=8, Hkv=4, d=64, w=100, a_lo=-2.0, a_hi=-0.1, seed=7,
                  len_lo=1, len_hi=700)
    x = {k: v.cuda() for k, v in make_inputs(wl).items()}
    out, ok_out = guarded(tuple(x["q"].shape), torch.bfloat16)
    if cached:
        state = dma.dma_decode_state_init(x["v"], x["W"], x["A"], x["lengths"], wl.w, wl.Hq)
        dma.dma_decode_step_cached(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w, state, out=out)
        assert dma.dma_check(state) == 0
    else:
        dma.dma_decode_step(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w, out=out)
    assert ok_out()
