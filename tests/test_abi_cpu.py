"""CPU-only checks of the C ABI: the library builds, loads, exports every entry
point include/dma.h declares, and rejects bad arguments on the host before
touching a GPU."""
import ctypes
import os
import re

import pytest

from doge_dynamic_mask_b200 import build as dma_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dma.h")


@pytest.fixture(scope="module")
def lib():
    path = dma_build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"DMA_API\s+[\w\s\*]+?\b(dma_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("dma_dt_scores", "dma_build_mask", "dma_forward_prefill", "dma_decode_step",
              "dma_workspace_size", "dma_check", "dma_status_string", "dma_last_cuda_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings(lib):
    lib.dma_status_string.restype = ctypes.c_char_p
    assert lib.dma_status_string(0) == b"DMA_OK"
    assert lib.dma_status_string(6) == b"DMA_ERR_BAD_LENGTH"
    assert lib.dma_status_string(99) == b"DMA_ERR_UNKNOWN"


def test_workspace_size_host_logic(lib):
    f = lib.dma_workspace_size
    f.restype = ctypes.c_size_t
    # prefill vs decode geometry; unsupported shapes give 0
    assert f(1, 256, 256, 4, 2, 64, 64) > 0
    assert f(64, 1, 65536, 16, 8, 128, 2048) > 64 * 8 * 65536 * 4      # holds dt of the whole cache
    assert f(1, 3, 256, 4, 2, 64, 64) == 0                            # neither prefill nor decode
    assert f(1, 256, 256, 4, 2, 96, 64) == 0                          # d not supported
    assert f(1, 256, 256, 6, 4, 64, 64) == 0                          # Hq not a multiple of Hkv
    assert f(1, 65536, 65536, 4, 2, 64, 9000) == 0                    # window above the selector's limit
    assert f(1, 4096, 4096, 4, 2, 64, 9000) > 0                       # ... fine when Lk <= w (no top-k)
    # monotone in the sequence length
    assert f(2, 4096, 4096, 8, 4, 64, 2048) > f(2, 2048, 2048, 8, 4, 64, 2048)


def test_argument_errors_are_reported_before_any_device_work(lib):
    vp = ctypes.c_void_p
    p16 = vp(1 << 20)          # aligned dummy address, never dereferenced
    bad = vp((1 << 20) + 4)    # misaligned
    lib.dma_forward_prefill.restype = ctypes.c_int
    lib.dma_forward_prefill.argtypes = [vp, vp, vp, vp, vp, vp] + [ctypes.c_int] * 6 + [
        ctypes.c_float, vp, vp, vp, ctypes.c_size_t, vp]
    args = [p16, p16, p16, p16, p16, None, 1, 256, 4, 2, 64, 64, 0.125, None, p16, p16, 1 << 30, None]
    # (the unmodified args would pass validation and launch kernels on dummy
    # pointers, so only invalid variants are ever passed here)
    a = list(args); a[0] = None
    assert lib.dma_forward_prefill(*a) == 1                     # DMA_ERR_INVALID_ARG
    a = list(args); a[1] = bad
    assert lib.dma_forward_prefill(*a) == 1
    a = list(args); a[8] = 6; a[9] = 4
    assert lib.dma_forward_prefill(*a) == 1                     # Hq % Hkv != 0
    a = list(args); a[10] = 80
    assert lib.dma_forward_prefill(*a) == 2                     # DMA_ERR_UNSUPPORTED
    a = list(args); a[12] = float("nan")
    assert lib.dma_forward_prefill(*a) == 1
    a = list(args); a[12] = 0.0
    assert lib.dma_forward_prefill(*a) == 1                     # the prefill scale must be positive
    a = list(args); a[12] = -0.125
    assert lib.dma_forward_prefill(*a) == 1
    a = list(args); a[3] = None; a[4] = None
    assert lib.dma_forward_prefill(*a) == 1                     # neither W/A nor dt_in
    lib.dma_build_mask.restype = ctypes.c_int
    lib.dma_build_mask.argtypes = [vp, vp] + [ctypes.c_int] * 5 + [vp, vp, vp, ctypes.c_size_t, vp]
    assert lib.dma_build_mask(p16, None, 1, 2, 7, 256, 64, None, None, p16, 1 << 30, None) == 1   # Lq neither L nor 1
    assert lib.dma_build_mask(None, None, 1, 2, 256, 256, 64, None, None, p16, 1 << 30, None) == 1
    lib.dma_dt_scores.restype = ctypes.c_int
    lib.dma_dt_scores.argtypes = [vp, vp, vp] + [ctypes.c_int] * 4 + [vp, vp]
    assert lib.dma_dt_scores(p16, p16, p16, 1, 16, 3, 64, p16, None) == 2          # Hkv = 3
    assert lib.dma_dt_scores(p16, p16, p16, 0, 16, 2, 64, p16, None) == 1          # B = 0


def test_cached_decode_state_size_and_argument_errors(lib):
    vp = ctypes.c_void_p
    p16 = vp(1 << 20)          # aligned dummy address, never dereferenced
    bad = vp((1 << 20) + 4)    # misaligned
    size = lib.dma_decode_state_size
    size.restype = ctypes.c_size_t
    size.argtypes = [ctypes.c_int] * 6
    ws = lib.dma_workspace_size
    ws.restype = ctypes.c_size_t
    # a state holds a decode workspace's plan plus two ints per (batch, kv head)
    assert size(64, 65536, 16, 8, 128, 2048) >= ws(64, 1, 65536, 16, 8, 128, 2048) + 2 * 64 * 8 * 4
    assert size(1, 256, 6, 4, 64, 64) == 0          # Hq not a multiple of Hkv
    assert size(1, 256, 4, 2, 96, 64) == 0          # d not supported
    init = lib.dma_decode_state_init
    init.restype = ctypes.c_int
    init.argtypes = [vp, vp, vp, vp] + [ctypes.c_int] * 6 + [vp, ctypes.c_size_t, vp]
    args = [p16, p16, p16, None, 1, 256, 4, 2, 64, 64, p16, 1 << 30, None]
    a = list(args); a[0] = None
    assert init(*a) == 1
    a = list(args); a[10] = bad
    assert init(*a) == 1
    a = list(args); a[8] = 80
    assert init(*a) == 2                             # DMA_ERR_UNSUPPORTED
    step = lib.dma_decode_step_cached
    step.restype = ctypes.c_int
    step.argtypes = [vp, vp, vp, vp, vp, vp] + [ctypes.c_int] * 6 + [ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
    args = [p16, p16, p16, p16, p16, None, 1, 256, 4, 2, 64, 64, 0.125, p16, p16, 1 << 30, None]
    a = list(args); a[14] = None                     # no state
    assert step(*a) == 1
    a = list(args); a[3] = None                      # W is required: the step computes dt of new tokens
    assert step(*a) == 1
    a = list(args); a[12] = float("nan")
    assert step(*a) == 1
    a = list(args); a[8] = 6; a[9] = 4
    assert step(*a) == 1


def test_prologue_argument_errors(lib):
    vp = ctypes.c_void_p
    p16 = vp(1 << 20)          # aligned dummy address, never dereferenced
    bad = vp((1 << 20) + 4)    # misaligned
    f = lib.dma_prologue
    f.restype = ctypes.c_int
    f.argtypes = [vp] * 5 + [ctypes.c_float, ctypes.c_float, vp] + [ctypes.c_int] * 6 + [vp] * 4 + [
        ctypes.c_size_t, vp]
    args = [p16] * 5 + [1e-6, 10000.0, p16, 2, 16, 64, 8, 4, 64, p16, p16, p16, p16, 256, None]
    a = list(args); a[0] = None
    assert f(*a) == 1                            # DMA_ERR_INVALID_ARG
    a = list(args); a[3] = bad
    assert f(*a) == 1
    a = list(args); a[7] = None                  # positions are required
    assert f(*a) == 1
    a = list(args); a[18] = 255
    assert f(*a) == 3                            # DMA_ERR_WORKSPACE: no room for the status word
    a = list(args); a[9] = 65
    assert f(*a) == 1                            # L > Lmax
    a = list(args); a[6] = 1.0
    assert f(*a) == 1                            # rope_theta must exceed 1
    a = list(args); a[5] = float("nan")
    assert f(*a) == 1
    a = list(args); a[13] = 96
    assert f(*a) == 2                            # d not supported
    a = list(args); a[11] = 6
    assert f(*a) == 1                            # Hq % Hkv != 0
    lib.dma_status_string.restype = ctypes.c_char_p
    assert lib.dma_status_string(7) == b"DMA_ERR_BAD_POSITION"


def test_cdmoe_workspace_and_argument_errors(lib):
    vp = ctypes.c_void_p
    p16 = vp(1 << 20)          # aligned dummy address, never dereferenced
    size = lib.dma_cdmoe_workspace_size
    size.restype = ctypes.c_size_t
    size.argtypes = [ctypes.c_int, ctypes.c_int]
    assert size(100, 16384) == 256 + ((100 * 256 * 4 + 255) // 256) * 256      # header + float32 logits
    assert size(100, 1000) == 0                                                  # not a square of 16..128
    f = lib.dma_cdmoe_forward
    f.restype = ctypes.c_int
    f.argtypes = [vp] * 4 + [ctypes.c_int] * 4 + [vp] * 5 + [ctypes.c_size_t, vp]
    args = [p16] * 4 + [8, 1024, 16384, 64] + [None, p16, None, None, p16, 1 << 20, None]
    a = list(args); a[0] = None
    assert f(*a) == 1
    a = list(args); a[1] = None                       # no router weight and no logits
    assert f(*a) == 1
    a = list(args); a[10] = p16                       # experts_out without scores_out
    assert f(*a) == 1
    a = list(args); a[7] = 65
    assert f(*a) == 2                                 # top_k above 64
    a = list(args); a[6] = 1000
    assert f(*a) == 2                                 # num_experts not K * K
    a = list(args); a[5] = 1000
    assert f(*a) == 2                                 # hidden not a multiple of 64
    a = list(args); a[13] = 100
    assert f(*a) == 3                                 # workspace too small
