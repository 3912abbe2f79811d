"""Seeded synthetic inputs for the DMA hot path.

This module only draws random tensors with the shapes and value distributions
of the five workloads below; it holds none of the method's arithmetic, so both
the CUDA path and the CPU oracle can be fed from it.

Value recipe (every workload): Q/K/V drawn N(0, 1) in float32 and rounded to
bf16; dt_proj weight W [H_kv*d, H_kv] float32 ~ N(0, 0.02) (std 0.02, the
models' initializer_range); A [H_kv] float32 ~ U[a_lo, a_hi]; valid lengths
U[len_lo, len_hi] (inclusive, right padding) or all full.  The draw order is
fixed: q, k, v, W, A, lengths.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str            # "prefill" or "decode"
    B: int
    L: int               # prefill: Lq = Lk = L; decode: cache length Lk
    Hq: int
    Hkv: int
    d: int
    w: int               # keep_window_size
    a_lo: float
    a_hi: float
    seed: int
    len_lo: Optional[int] = None   # None: every sequence is full length
    len_hi: Optional[int] = None

    @property
    def scale(self) -> float:
        return self.d ** -0.5

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # Tiny prefill: one sequence, causal, no padding.
    "tiny": Workload("tiny", "prefill", B=1, L=256, Hq=4, Hkv=2, d=64, w=64,
                     a_lo=-2.0, a_hi=-0.1, seed=0),
    # Dense-equivalent: keep_window_size >= L, reduces to causal attention + dt bias.
    "dense_eq": Workload("dense_eq", "prefill", B=8, L=2048, Hq=8, Hkv=4, d=64, w=2048,
                         a_lo=-2.0, a_hi=-0.1, seed=1),
    # Sparse prefill with right padding, lengths U[4096, 8192].
    "sparse_pad": Workload("sparse_pad", "prefill", B=4, L=8192, Hq=8, Hkv=4, d=64, w=2048,
                           a_lo=-2.0, a_hi=-0.1, seed=2, len_lo=4096, len_hi=8192),
    # Long-context prefill, sharper dt spread.
    "long": Workload("long", "prefill", B=1, L=32768, Hq=16, Hkv=8, d=128, w=2048,
                     a_lo=-4.0, a_hi=-0.1, seed=3),
    # Decode: one new query per sequence against a 65536-long cache.
    "decode": Workload("decode", "decode", B=64, L=65536, Hq=16, Hkv=8, d=128, w=2048,
                       a_lo=-2.0, a_hi=-0.1, seed=4),
}


def _randn_bf16(shape, gen, device, chunk_rows=None):
    """N(0,1) float32 draws rounded to bf16; drawn in chunks along dim 0 so a
    multi-GB tensor never needs a float32 copy of itself."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if chunk_rows is None or shape[0] <= chunk_rows:
        out.copy_(torch.randn(shape, generator=gen, device=device, dtype=torch.float32))
        return out
    for s in range(0, shape[0], chunk_rows):
        e = min(shape[0], s + chunk_rows)
        out[s:e].copy_(torch.randn((e - s,) + tuple(shape[1:]), generator=gen, device=device,
                                   dtype=torch.float32))
    return out


def make_inputs(wl: Workload, device="cpu", seed: Optional[int] = None):
    """Draw one batch of inputs for workload `wl` on `device`.

    Returns a dict of torch tensors:
      prefill: q [B,L,Hq,d], k/v [B,L,Hkv,d] (bf16)
      decode : q [B,Hq,d], k/v [B,L,Hkv,d] (bf16; L is the cache length)
      W [Hkv*d, Hkv] f32, A [Hkv] f32, lengths [B] int32.
    The same (workload, seed, device type) always gives the same tensors.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed if seed is None else seed)
    B, L, Hq, Hkv, d = wl.B, wl.L, wl.Hq, wl.Hkv, wl.d
    if wl.mode == "prefill":
        q = _randn_bf16((B, L, Hq, d), gen, device, chunk_rows=1)
    else:
        q = _randn_bf16((B, Hq, d), gen, device)
    k = _randn_bf16((B, L, Hkv, d), gen, device, chunk_rows=1)
    v = _randn_bf16((B, L, Hkv, d), gen, device, chunk_rows=1)
    W = (torch.randn((Hkv * d, Hkv), generator=gen, device=device, dtype=torch.float32) * 0.02)
    A = torch.rand((Hkv,), generator=gen, device=device, dtype=torch.float32) * (wl.a_hi - wl.a_lo) + wl.a_lo
    if wl.len_lo is None:
        lengths = torch.full((B,), L, dtype=torch.int32, device=device)
    else:
        lengths = torch.randint(wl.len_lo, wl.len_hi + 1, (B,), generator=gen, device=device,
                                dtype=torch.int64).to(torch.int32)
    return {"q": q, "k": k, "v": v, "W": W, "A": A, "lengths": lengths}


def shrink(wl: Workload, **kw) -> Workload:
    """A smaller variant of a workload (same value recipe) for tests."""
    return wl.replace(name=wl.name + "_small", **kw)


def make_prologue_inputs(B, L, Lmax, Hq, Hkv, d, seed, device="cpu", positions=None):
    """Inputs of the prologue (q/k RMSNorm, rotary embedding, KV-cache append):
    projected q [B,L,Hq,d], k/v [B,L,Hkv,d] and caches [B,Lmax,Hkv,d] ~ N(0,1)
    rounded to bf16; RMSNorm weights [d] ~ U[0.5, 1.5] float32 (a learned
    scale around its initial value 1); positions [B] int32 ~ U[0, Lmax - L]
    unless given.  Draw order: q, k, v, q_norm_w, k_norm_w, positions,
    k_cache, v_cache."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _randn_bf16((B, L, Hq, d), gen, device, chunk_rows=1)
    k = _randn_bf16((B, L, Hkv, d), gen, device, chunk_rows=1)
    v = _randn_bf16((B, L, Hkv, d), gen, device, chunk_rows=1)
    q_w = torch.rand((d,), generator=gen, device=device, dtype=torch.float32) + 0.5
    k_w = torch.rand((d,), generator=gen, device=device, dtype=torch.float32) + 0.5
    pos = torch.randint(0, Lmax - L + 1, (B,), generator=gen, device=device, dtype=torch.int64).to(torch.int32)
    if positions is not None:
        pos = torch.as_tensor(positions, dtype=torch.int32, device=device)
    k_cache = _randn_bf16((B, Lmax, Hkv, d), gen, device, chunk_rows=1)
    v_cache = _randn_bf16((B, Lmax, Hkv, d), gen, device, chunk_rows=1)
    return {"q": q, "k": k, "v": v, "q_w": q_w, "k_w": k_w, "positions": pos, "k_cache": k_cache,
            "v_cache": v_cache}


def make_cdmoe_inputs(T, hidden, num_experts, seed, device="cpu"):
    """Inputs of the CDMoE routing: hidden states h [T, hidden] ~ N(0, 1) and
    the router weight W_router [2K, hidden] (K = sqrt(num_experts)) ~ N(0, 0.02)
    plus the expert tables down_embed / up_embed [num_experts, hidden]
    ~ N(0, 0.02) (the models' initializer_range), all rounded to bf16.
    Draw order: h, W_router, down_embed, up_embed."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    K = int(round(num_experts ** 0.5))
    h = _randn_bf16((T, hidden), gen, device)
    w = (torch.randn((2 * K, hidden), generator=gen, device=device, dtype=torch.float32) * 0.02).to(torch.bfloat16)
    down = (torch.randn((num_experts, hidden), generator=gen, device=device, dtype=torch.float32) * 0.02).to(
        torch.bfloat16)
    up = (torch.randn((num_experts, hidden), generator=gen, device=device, dtype=torch.float32) * 0.02).to(
        torch.bfloat16)
    return {"h": h, "W_router": w, "down_embed": down, "up_embed": up}
