"""Thin Python binding of libdma (argument marshalling only).

Every function here forwards to the C entry point of the same name in
``libdma.so`` (declared in include/dma.h) with device pointers taken from torch
tensors and the current torch CUDA stream.  No step of the computation runs in
Python, and there is no fallback: importing this module fails loudly if the
library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdma.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"libdma.so is not built ({_LIB_PATH}); run `python -m doge_dynamic_mask_b200.build` (needs nvcc)")
_lib = ctypes.CDLL(_LIB_PATH)

DMA_OK = 0
STATUS = {0: "DMA_OK", 1: "DMA_ERR_INVALID_ARG", 2: "DMA_ERR_UNSUPPORTED", 3: "DMA_ERR_WORKSPACE",
          4: "DMA_ERR_CUDA", 5: "DMA_ERR_TIMEOUT", 6: "DMA_ERR_BAD_LENGTH", 7: "DMA_ERR_BAD_POSITION"}

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_lib.dma_workspace_size.restype = _sz
_lib.dma_workspace_size.argtypes = [_i] * 7
_lib.dma_dt_scores.restype = _i
_lib.dma_dt_scores.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp]
_lib.dma_build_mask.restype = _i
_lib.dma_build_mask.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]
_lib.dma_forward_prefill.restype = _i
_lib.dma_forward_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _sz,
                                     _vp]
_lib.dma_forward_prefill_lse.restype = _i
_lib.dma_forward_prefill_lse.argtypes = [_vp] * 6 + [_i] * 6 + [_f] + [_vp] * 4 + [_sz, _vp]
_lib.dma_decode_step.restype = _i
_lib.dma_decode_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _sz, _vp]
_lib.dma_decode_state_size.restype = _sz
_lib.dma_decode_state_size.argtypes = [_i] * 6
_lib.dma_decode_state_init.restype = _i
_lib.dma_decode_state_init.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
_lib.dma_decode_step_cached.restype = _i
_lib.dma_decode_step_cached.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _sz, _vp]
_lib.dma_prologue.restype = _i
_lib.dma_prologue.argtypes = [_vp] * 5 + [_f, _f, _vp] + [_i] * 6 + [_vp] * 4 + [_sz, _vp]
_lib.dma_cdmoe_workspace_size.restype = _sz
_lib.dma_cdmoe_workspace_size.argtypes = [_i, _i]
_lib.dma_cdmoe_forward.restype = _i
_lib.dma_cdmoe_forward.argtypes = [_vp] * 4 + [_i] * 4 + [_vp] * 5 + [_sz, _vp]
_lib.dma_backward_workspace_size.restype = _sz
_lib.dma_backward_workspace_size.argtypes = [_i] * 6
_lib.dma_backward_prefill.restype = _i
_lib.dma_backward_prefill.argtypes = [_vp] * 6 + [_i] * 6 + [_f] + [_vp] * 11 + [_sz, _vp]
_lib.dma_selftest_wait.restype = _i
_lib.dma_selftest_wait.argtypes = [_vp, _vp]
_lib.dma_check.restype = _i
_lib.dma_check.argtypes = [_vp, _i, _vp]
_lib.dma_status_string.restype = ctypes.c_char_p
_lib.dma_status_string.argtypes = [_i]
_lib.dma_last_cuda_error.restype = _i
_lib.dma_last_cuda_error.argtypes = []
_lib.dma_set_stage_events.restype = _i
_lib.dma_set_stage_events.argtypes = [_vp, _i]


class DMAError(RuntimeError):
    def __init__(self, status: int, where: str):
        name = _lib.dma_status_string(status).decode()
        extra = f" (cudaError {_lib.dma_last_cuda_error()})" if status == 4 else ""
        super().__init__(f"{where}: {name}{extra}")
        self.status = status


def _ok(status: int, where: str):
    if status != DMA_OK:
        raise DMAError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libdma must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def lib_path() -> str:
    return _LIB_PATH


def dma_workspace_size(B, Lq, Lk, Hq, Hkv, d, keep_window_size) -> int:
    return int(_lib.dma_workspace_size(B, Lq, Lk, Hq, Hkv, d, keep_window_size))


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zeroed device workspace (the status word must start at zero)."""
    return torch.zeros(int(nbytes), dtype=torch.uint8, device=device or "cuda")


def dma_dt_scores(v, W_dt, A, dt_out=None, stream=None):
    B, L, Hkv, d = v.shape
    if dt_out is None:
        dt_out = torch.empty((B, Hkv, L), dtype=torch.float32, device=v.device)
    _ok(_lib.dma_dt_scores(_ptr(v), _ptr(W_dt), _ptr(A), B, L, Hkv, d, _ptr(dt_out), _stream(stream)),
        "dma_dt_scores")
    return dt_out


def dma_build_mask(dt, lengths, Lq, keep_window_size, workspace=None, tau_out=None, bitmask_out=None,
                   stream=None):
    B, Hkv, Lk = dt.shape
    if workspace is None:
        workspace = new_workspace(dma_workspace_size(B, Lq, Lk, Hkv, Hkv, 64, keep_window_size), dt.device)
    _ok(_lib.dma_build_mask(_ptr(dt), _ptr(lengths), B, Hkv, Lq, Lk, keep_window_size, _ptr(tau_out),
                            _ptr(bitmask_out), _ptr(workspace), workspace.numel(), _stream(stream)),
        "dma_build_mask")
    return workspace


def dma_forward_prefill(q, k, v, W_dt, A, lengths, keep_window_size, scale=None, dt_in=None, out=None,
                        workspace=None, stream=None, lse_out=None):
    """With lse_out ([B, Hq, L] float32) the rows' normalisers are written too
    (dma_forward_prefill_lse), for dma_backward_prefill(lse_in=...)."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = new_workspace(dma_workspace_size(B, L, L, Hq, Hkv, d, keep_window_size), q.device)
    if lse_out is None:
        _ok(_lib.dma_forward_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(W_dt), _ptr(A), _ptr(lengths), B, L, Hq, Hkv,
                                     d, keep_window_size, float(scale), _ptr(dt_in), _ptr(out), _ptr(workspace),
                                     workspace.numel(), _stream(stream)),
            "dma_forward_prefill")
    else:
        _ok(_lib.dma_forward_prefill_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(W_dt), _ptr(A), _ptr(lengths), B, L, Hq,
                                         Hkv, d, keep_window_size, float(scale), _ptr(dt_in), _ptr(out),
                                         _ptr(lse_out), _ptr(workspace), workspace.numel(), _stream(stream)),
            "dma_forward_prefill_lse")
    return out


def dma_decode_step(q, k_cache, v_cache, W_dt, A, lengths, keep_window_size, scale=None, dt_in=None, out=None,
                    workspace=None, stream=None):
    B, Hq, d = q.shape
    Lk, Hkv = k_cache.shape[1], k_cache.shape[2]
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = new_workspace(dma_workspace_size(B, 1, Lk, Hq, Hkv, d, keep_window_size), q.device)
    _ok(_lib.dma_decode_step(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(W_dt), _ptr(A), _ptr(lengths), B, Lk, Hq,
                             Hkv, d, keep_window_size, float(scale), _ptr(dt_in), _ptr(out), _ptr(workspace),
                             workspace.numel(), _stream(stream)),
        "dma_decode_step")
    return out


def dma_prologue(q, k, v, q_norm_w, k_norm_w, positions, k_cache, v_cache, eps=1e-6, rope_theta=10000.0,
                 q_out=None, workspace=None, stream=None):
    """q/k RMSNorm over head_dim, rotary embedding, and the KV-cache append of
    L new tokens per sequence (token t of sequence b at cache row positions[b] + t).
    Returns q_out; k_cache and v_cache are written in place."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    Lmax = k_cache.shape[1]
    if q_out is None:
        q_out = torch.empty_like(q)
    if workspace is None:
        workspace = new_workspace(256, q.device)
    _ok(_lib.dma_prologue(_ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), float(eps), float(rope_theta),
                          _ptr(positions), B, L, Lmax, Hq, Hkv, d, _ptr(q_out), _ptr(k_cache), _ptr(v_cache),
                          _ptr(workspace), workspace.numel(), _stream(stream)),
        "dma_prologue")
    return q_out


def dma_backward_workspace_size(B, L, Hq, Hkv, d, keep_window_size) -> int:
    return int(_lib.dma_backward_workspace_size(B, L, Hq, Hkv, d, keep_window_size))


def dma_backward_prefill(q, k, v, W_dt, A, lengths, keep_window_size, out, dout, scale=None, dt_in=None,
                         workspace=None, want_d_dt=False, stream=None, lse_in=None):
    """Gradients of sum(out * dout) with the selection held fixed: returns
    (dq, dk, dv) bf16, dW_dt and dA float32, and d_dt [B, Hkv, L] float32 when
    want_d_dt.  lse_in: the forward's row normalisers (dma_forward_prefill with
    lse_out), else they are recomputed."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = d ** -0.5
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dW = torch.empty_like(W_dt)
    dA = torch.empty_like(A)
    d_dt = torch.empty((B, Hkv, L), dtype=torch.float32, device=q.device) if want_d_dt else None
    if workspace is None:
        workspace = new_workspace(dma_backward_workspace_size(B, L, Hq, Hkv, d, keep_window_size), q.device)
    _ok(_lib.dma_backward_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(W_dt), _ptr(A), _ptr(lengths), B, L, Hq, Hkv, d,
                                  keep_window_size, float(scale), _ptr(dt_in), _ptr(out), _ptr(dout),
                                  _ptr(lse_in), _ptr(dq),
                                  _ptr(dk), _ptr(dv), _ptr(d_dt), _ptr(dW), _ptr(dA), _ptr(workspace),
                                  workspace.numel(), _stream(stream)),
        "dma_backward_prefill")
    return (dq, dk, dv, dW, dA, d_dt) if want_d_dt else (dq, dk, dv, dW, dA)


def dma_cdmoe_workspace_size(T, num_experts) -> int:
    return int(_lib.dma_cdmoe_workspace_size(T, num_experts))


def dma_cdmoe_forward(h, W_router, down_embed, up_embed, top_k, logits_in=None, out=None, experts_out=None,
                      scores_out=None, workspace=None, stream=None):
    """Routed CDMoE output [T, hidden] (bf16).  With experts_out / scores_out
    ([T, top_k] int32 / float32) the kept experts are written too, best first."""
    T, hidden = h.shape
    num_experts = down_embed.shape[0]
    if out is None:
        out = torch.empty_like(h)
    if workspace is None:
        size = dma_cdmoe_workspace_size(T, num_experts)
        if size == 0:
            raise ValueError("unsupported CDMoE geometry")
        workspace = new_workspace(size, h.device)
    _ok(_lib.dma_cdmoe_forward(_ptr(h), _ptr(W_router), _ptr(down_embed), _ptr(up_embed), T, hidden, num_experts,
                               top_k, _ptr(logits_in), _ptr(out), _ptr(experts_out), _ptr(scores_out),
                               _ptr(workspace), workspace.numel(), _stream(stream)),
        "dma_cdmoe_forward")
    return out


def dma_decode_state_size(B, Lk, Hq, Hkv, d, keep_window_size) -> int:
    return int(_lib.dma_decode_state_size(B, Lk, Hq, Hkv, d, keep_window_size))


def dma_decode_state_init(v_cache, W_dt, A, lengths, keep_window_size, Hq, state=None, stream=None):
    """Decode state for incremental steps: dt of every cached token and each
    (batch, kv head)'s kept set.  Returns the state (a uint8 device tensor)."""
    B, Lk, Hkv, d = v_cache.shape
    size = dma_decode_state_size(B, Lk, Hq, Hkv, d, keep_window_size)
    if size == 0:
        raise ValueError("unsupported decode geometry")
    if state is None:
        state = torch.empty(size, dtype=torch.uint8, device=v_cache.device)
    _ok(_lib.dma_decode_state_init(_ptr(v_cache), _ptr(W_dt), _ptr(A), _ptr(lengths), B, Lk, Hq, Hkv, d,
                                   keep_window_size, _ptr(state), state.numel(), _stream(stream)),
        "dma_decode_state_init")
    return state


def dma_decode_step_cached(q, k_cache, v_cache, W_dt, A, lengths, keep_window_size, state, scale=None, out=None,
                           stream=None):
    """One decode step that takes in only the tokens cached since the previous step."""
    B, Hq, d = q.shape
    Lk, Hkv = k_cache.shape[1], k_cache.shape[2]
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    _ok(_lib.dma_decode_step_cached(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(W_dt), _ptr(A), _ptr(lengths), B,
                                    Lk, Hq, Hkv, d, keep_window_size, float(scale), _ptr(out), _ptr(state),
                                    state.numel(), _stream(stream)),
        "dma_decode_step_cached")
    return out


# keys per split of the decode attention: the kept lists are padded to a
# multiple of it (the library's layout of a decode workspace)
DECODE_CHUNK = 128


def decode_state_views(state, B, Lk, Hq, Hkv, d, keep_window_size):
    """(dt [B, Hkv, Lk] float32, kept count [B, Hkv] int32, kept key lists [B, Hkv, cap] int32) views of a
    decode state, for tests: the layout is that of a decode workspace."""
    bg = B * Hkv
    cap = -(-min(Lk, keep_window_size) // DECODE_CHUNK) * DECODE_CHUNK
    def up(x):
        return -(-x // 256) * 256
    off = 256
    dt = state[off:off + bg * Lk * 4].view(torch.float32).view(B, Hkv, Lk)
    off = up(off + bg * Lk * 4)
    off = up(off + bg * 8)                   # tau
    idx = state[off:off + bg * cap * 4].view(torch.int32).view(B, Hkv, cap)
    off = up(off + bg * cap * 4)
    off = up(off + bg * cap * 4)             # bias
    count = state[off:off + bg * 4].view(torch.int32).view(B, Hkv)
    return dt, count, idx


def dma_selftest_wait(workspace, stream=None):
    """Launch the bounded-wait diagnostic: its wait runs out (about one second)
    and records a timeout that dma_check then reports."""
    _ok(_lib.dma_selftest_wait(_ptr(workspace), _stream(stream)), "dma_selftest_wait")


def dma_check(workspace, clear=True, stream=None) -> int:
    """Synchronises the stream and returns the device-recorded status (0 = DMA_OK)."""
    return int(_lib.dma_check(_ptr(workspace), 1 if clear else 0, _stream(stream)))


class StageEvents:
    """Context manager: while active, prefill/decode calls on this thread record
    4 torch CUDA events (before S1, after S1, after S2, after the attention)."""

    def __init__(self):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        for e in self.events:          # materialise the underlying cudaEvent_t
            e.record()
        self._arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in self.events])

    def __enter__(self):
        _ok(_lib.dma_set_stage_events(self._arr, 4), "dma_set_stage_events")
        return self

    def __exit__(self, *exc):
        _lib.dma_set_stage_events(None, 0)

    def stage_ms(self):
        """(S1, S2, attention) milliseconds of the last recorded call."""
        e = self.events
        return (e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3]))


def dma_status_string(status: int) -> str:
    return _lib.dma_status_string(status).decode()


def raw():
    """The ctypes handle (for tests that call the C ABI with raw pointers)."""
    return _lib
