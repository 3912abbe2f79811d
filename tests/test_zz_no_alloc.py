"""The allocation-free decode entry point, called through the C ABI.

dma_decode_step_noalloc serves callers that cannot allocate device memory
themselves (a host framework that owns all device memory through its own pool
and forbids raw cudaMalloc, or plain C callers without a device allocator): it
keeps its scratch in a fixed array inside the library.  Its output must match
the ordinary dma_decode_step (which takes a caller-provided workspace) within
the output tolerance used by every parity test here, on two calls in a row
(the second call reuses the array the first one left behind), and so must
the float64 oracle's; a second call must not change the device's free memory.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from doge_dynamic_mask_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

OUT_MAX, OUT_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module")
def dma():
    from doge_dynamic_mask_b200 import build
    build.build()
    from doge_dynamic_mask_b200 import dma as m
    return m


def _noalloc(lib, x, wl, out):
    vp = ctypes.c_void_p
    f = lib.dma_decode_step_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, vp, vp] + [ctypes.c_int] * 6 + [ctypes.c_float, vp, vp, vp]
    stream = vp(torch.cuda.current_stream().cuda_stream)
    p = lambda t: vp(t.data_ptr())
    return f(p(x["q"]), p(x["k"]), p(x["v"]), p(x["W"]), p(x["A"]), p(x["lengths"]), wl.B, wl.L, wl.Hq, wl.Hkv,
             wl.d, wl.w, wl.scale, None, p(out), stream)


def test_noalloc_decode_matches_workspace_decode_twice(dma):
    lib = dma.raw()
    for seed in (101, 202):
        wl = Workload("noalloc", "decode", B=4, L=8192, Hq=16, Hkv=8, d=128, w=2048, a_lo=-2.0, a_hi=-0.1,
                      seed=seed, len_lo=3000, len_hi=8192)
        x = {k: v.cuda() for k, v in make_inputs(wl).items()}
        want = dma.dma_decode_step(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w)
        got = torch.full_like(want, float("nan"))
        assert _noalloc(lib, x, wl, got) == 0
        torch.cuda.synchronize()
        err = (got.float() - want.float()).abs().cpu().numpy()
        assert np.isfinite(err).all()
        assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN, (seed, err.max(), err.mean())


def test_noalloc_decode_matches_oracle_and_allocates_nothing(dma):
    """Against the float64 oracle directly, on two calls in a row; the second
    call (after the first has loaded the kernels) leaves the device's free
    memory exactly as it was."""
    import oracle
    lib = dma.raw()
    wl = Workload("noalloc", "decode", B=2, L=5000, Hq=8, Hkv=4, d=128, w=1024, a_lo=-2.0, a_hi=-0.1,
                  seed=303, len_lo=900, len_hi=5000)
    xh = make_inputs(wl)
    x = {k: v.cuda() for k, v in xh.items()}
    f64 = lambda t: t.float().numpy().astype(np.float64)
    want = oracle.decode_step(f64(xh["q"]), f64(xh["k"]), f64(xh["v"]), xh["W"].double().numpy(),
                              xh["A"].double().numpy(), xh["lengths"].numpy(), wl.w, wl.scale)
    outs = [torch.full_like(x["q"], float("nan")) for _ in range(2)]
    assert _noalloc(lib, x, wl, outs[0]) == 0
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    assert _noalloc(lib, x, wl, outs[1]) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    for out in outs:
        err = np.abs(out.float().cpu().numpy() - want)
        assert np.isfinite(err).all()
        assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN, (err.max(), err.mean())


def test_noalloc_rejects_steps_beyond_its_scratch(dma):
    lib = dma.raw()
    # the full 64 x 65536-key cache needs about 134 MB of per-key scores: more than the 64 MiB array
    wl = Workload("big", "decode", B=64, L=65536, Hq=16, Hkv=8, d=128, w=2048, a_lo=-2.0, a_hi=-0.1, seed=1)
    small = Workload("small", "decode", B=1, L=128, Hq=16, Hkv=8, d=128, w=64, a_lo=-2.0, a_hi=-0.1, seed=1)
    x = {k: v.cuda() for k, v in make_inputs(small).items()}
    out = torch.empty_like(x["q"])
    assert _noalloc(lib, x, wl, out) == 3       # DMA_ERR_WORKSPACE, returned before any launch
