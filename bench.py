"""Benchmark of the DMA hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]

Headline (`value`): prefill TFLOP/s on the dense-equivalent workload
(B=8, L=2048, Hq=8, Hkv=4, d=64, keep_window_size=2048), counting 4*d FLOPs
per kept (query, key) pair per query head; a step is one dma_forward_prefill
call (dt scores, dynamic-mask selection, attention).  The same line reports
decode GB/s (B=64, cache 65536, Hq=16, Hkv=8, d=128, w=2048; algorithmic KV
bytes) and TFLOP/s of the sparse-padded and long-context prefill workloads.

Timing: a CUDA event pair per step on the launching stream, L2 flushed
(256 MiB write) between timed steps, the K timed steps enqueued ahead of the
device so that no host gap is timed, W untimed warm-up steps, a barrier and a
device synchronize on both sides of the timed region, max over ranks.  The
stage split (and the attention kernel's time for the roofline) comes from K
more steps after the timed region, each with the library's stage events.  Multi-GPU:
one process per GPU (torchrun), every rank runs its own copy of the workload
(weak scaling, no data-path collective).

--impl reference times the CPU oracle (the only reference implementation of
this method) on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from doge_dynamic_mask_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "DMA prefill TFLOP/s (kept keys) & decode KV GB/s, % of B200 peak"
HEADLINE = "dense_eq"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------
# work accounting (from the workload definition and the valid lengths)
# ----------------------------------------------------------------------------

def kept_pairs(L, w, lengths):
    """Kept (query row, key) pairs per query head, summed over the batch: row i
    of a sequence of valid length n keeps min(w, min(i+1, n)) keys when L > w,
    else min(i+1, n)."""
    total = 0
    i = np.arange(L, dtype=np.int64)
    for n in np.asarray(lengths, dtype=np.int64):
        vis = np.minimum(i + 1, n)
        total += int(np.minimum(vis, w).sum()) if L > w else int(vis.sum())
    return total


def prefill_flops(wl, lengths):
    return 4 * wl.d * wl.Hq * kept_pairs(wl.L, wl.w, lengths)


def kept_pairs_valid_rows(L, w, lengths):
    """kept_pairs restricted to the valid query rows i < n of each sequence
    (the padded rows, which the kernels also compute, left out)."""
    total = 0
    for n in np.asarray(lengths, dtype=np.int64):
        vis = np.arange(1, int(n) + 1, dtype=np.int64)
        total += int(np.minimum(vis, w).sum()) if L > w else int(vis.sum())
    return total


def prefill_flops_valid_rows(wl, lengths):
    return 4 * wl.d * wl.Hq * kept_pairs_valid_rows(wl.L, wl.w, lengths)


def decode_bytes(wl, lengths):
    """V read for dt over the whole cache + the kept K and V rows + q and out."""
    B, Lk, Hkv, d, Hq = wl.B, wl.L, wl.Hkv, wl.d, wl.Hq
    v_scan = B * Lk * Hkv * d * 2
    kept = sum(min(wl.w, int(n)) if Lk > wl.w else int(n) for n in lengths)
    kv_rows = kept * Hkv * 2 * d * 2
    return v_scan + kv_rows + 2 * B * Hq * d * 2


# ----------------------------------------------------------------------------
# multi-rank aggregation (weak scaling: every rank runs its own copy)
# ----------------------------------------------------------------------------

def max_over_ranks(v, dist=None, device=None):
    """Largest value over all ranks (timings are reported as the slowest rank)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank, ms_max, world):
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


def _free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_entry(rank, world, port, target, args):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    target(args)


def spawn_ranks(world, target, args, timeout_s=1800):
    """Runs target(args) in `world` fresh processes (spawn), one per GPU, with
    RANK, LOCAL_RANK, WORLD_SIZE and MASTER_ADDR/PORT set as torchrun sets
    them; returns the first non-zero exit code, or 0."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_entry, args=(r, world, port, target, args)) for r in range(world)]
    for p in procs:
        p.start()
    rc = 0
    t0 = time.time()
    for p in procs:
        p.join(timeout=max(1.0, timeout_s - (time.time() - t0)))
        if p.exitcode is None:
            p.kill()
            p.join()
            rc = rc or 1
        else:
            rc = rc or p.exitcode
    return rc


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def kernel_traffic(kernel):
    """DRAM bytes per launch of `kernel` from profiles/traffic.json, or None
    when that record is missing or was taken on a different kernel source."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[kernel]
        src = open(os.path.join(ROOT, rec["source_file"]), "rb").read()
        if hashlib.sha256(src).hexdigest()[:16] != rec["source_sha256_prefix"]:
            return None
        return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples during the timed region."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 7 and parts[0].isdigit():
                    rows.append(parts)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [int(r[0]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[3 + k].lower() == "active"})
        return {"sm_mhz": int(statistics.median(sm)), "sm_max_mhz": int(rows[0][1]), "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def run_steps(dma, step, first, steps, flush, stages=False):
    """Device time of `steps` calls step(first), step(first + 1), ...: the L2
    flush runs between calls, and all of it is enqueued before one
    synchronize, with a few flushes queued ahead of the first call so that
    the host enqueues ahead of the device: the events time device work only,
    never a host gap.  Without `stages` one event pair brackets each call and
    the per-call milliseconds are returned.  With `stages` every call records
    the library's four stage events (before S1, after S1, after S2, after the
    attention) and the per-call (S1, S2, attention) milliseconds are
    returned; an event waits for the work before it, so the two events
    inside the call add a little device time (about 2.5 us each) and this
    pass gives the split, not the step time."""
    torch.cuda.synchronize()
    if stages:
        evs = [dma.StageEvents() for _ in range(steps)]
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for _ in range(4):
        flush.zero_()
    for i, ev in enumerate(evs):
        if stages:
            with ev:
                step(first + i)
        else:
            ev[0].record()
            step(first + i)
            ev[1].record()
        flush.zero_()
    torch.cuda.synchronize()
    if stages:
        return [ev.stage_ms() for ev in evs]
    return [a.elapsed_time(b) for a, b in evs]


def timed(dma, step, first, steps, flush, ranks_sync):
    """The timed region (barrier + synchronize on both sides) and, after it,
    the stage-split pass: (ms per step, [S1, S2, attention] ms per step)."""
    ranks_sync()
    ms = run_steps(dma, step, first, steps, flush)
    ranks_sync()
    split = run_steps(dma, step, first + steps, steps, flush, stages=True)
    n = len(split)
    return sum(ms) / len(ms), [sum(x[k] for x in split) / n for k in range(3)]


def time_prefill(dma, wl, steps, warmup, flush, dev, ranks_sync):
    x = make_inputs(wl, device=dev)
    lengths = x["lengths"].cpu().numpy()
    ws = dma.new_workspace(dma.dma_workspace_size(wl.B, wl.L, wl.L, wl.Hq, wl.Hkv, wl.d, wl.w), dev)
    out = torch.empty_like(x["q"])

    def step():
        dma.dma_forward_prefill(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w, out=out, workspace=ws)

    for _ in range(warmup):
        step()
        flush.zero_()
    assert dma.dma_check(ws) == 0
    ms, stage = timed(dma, lambda i: step(), 0, steps, flush, ranks_sync)
    assert dma.dma_check(ws) == 0
    flops = prefill_flops(wl, lengths)
    flops_valid = prefill_flops_valid_rows(wl, lengths)
    # dt, selector (skipped when keep_window_size >= L: no top-k) and attention
    per_step = 2 if wl.L <= wl.w else 3
    return {"flops": flops, "flops_valid": flops_valid, "ms": ms, "stage_ms": stage, "launches": per_step * steps,
            "x": x, "ws": ws, "out": out}


def time_decode(dma, wl, steps, warmup, flush, dev, ranks_sync):
    x = make_inputs(wl, device=dev)
    lengths = x["lengths"].cpu().numpy()
    ws = dma.new_workspace(dma.dma_workspace_size(wl.B, 1, wl.L, wl.Hq, wl.Hkv, wl.d, wl.w), dev)
    out = torch.empty_like(x["q"])

    def step():
        dma.dma_decode_step(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w, out=out, workspace=ws)

    for _ in range(warmup):
        step()
        flush.zero_()
    assert dma.dma_check(ws) == 0
    ms, stage = timed(dma, lambda i: step(), 0, steps, flush, ranks_sync)
    assert dma.dma_check(ws) == 0
    nbytes = decode_bytes(wl, lengths)
    del x
    return {"bytes": nbytes, "ms": ms, "stage_ms": stage, "launches": 4 * steps}


def time_decode_cached(dma, wl, steps, warmup, flush, dev, ranks_sync):
    """The decode workload as incremental steps: the state is built over the
    caches minus the last warmup + 2 * steps tokens (untimed), then every step
    takes in one more token per sequence (dt of that token, kept-set update)
    and attends over the kept keys."""
    x = make_inputs(wl, device=dev)
    n_calls = warmup + 2 * steps   # warm-up, timed steps, stage-split steps
    start = wl.L - n_calls
    lens = [torch.full((wl.B,), start + 1 + i, dtype=torch.int32, device=dev) for i in range(n_calls)]
    state = dma.dma_decode_state_init(x["v"], x["W"], x["A"], torch.full((wl.B,), start, dtype=torch.int32,
                                                                        device=dev), wl.w, wl.Hq)
    assert dma.dma_check(state) == 0
    out = torch.empty_like(x["q"])

    def step(i):
        dma.dma_decode_step_cached(x["q"], x["k"], x["v"], x["W"], x["A"], lens[i], wl.w, state, out=out)

    for i in range(warmup):
        step(i)
        flush.zero_()
    assert dma.dma_check(state, clear=False) == 0
    ms, stage = timed(dma, step, warmup, steps, flush, ranks_sync)
    assert dma.dma_check(state) == 0
    # bytes a step must move: the new token's value row, the kept K and V rows, q and o
    kept = min(wl.w, wl.L)
    nbytes = wl.B * (wl.Hkv * wl.d * 2 + wl.Hkv * 2 * kept * wl.d * 2 + 2 * wl.Hq * wl.d * 2)
    del x, state
    return {"bytes": nbytes, "ms": ms, "stage_ms": stage, "launches": 3 * steps}


def time_prologue(dma, wl, steps, warmup, flush, dev, ranks_sync):
    """The prologue (q/k RMSNorm, rotary embedding, KV-cache append) over the
    workload's L tokens per sequence, written at the start of an L-row cache."""
    from doge_dynamic_mask_b200.workloads import make_prologue_inputs
    x = make_prologue_inputs(wl.B, wl.L, wl.L, wl.Hq, wl.Hkv, wl.d, wl.seed, device=dev,
                             positions=[0] * wl.B)
    ws = dma.new_workspace(256, dev)
    q_out = torch.empty_like(x["q"])

    def step(i):
        dma.dma_prologue(x["q"], x["k"], x["v"], x["q_w"], x["k_w"], x["positions"], x["k_cache"], x["v_cache"],
                         q_out=q_out, workspace=ws)

    for i in range(warmup):
        step(i)
        flush.zero_()
    assert dma.dma_check(ws) == 0
    ranks_sync()
    ms = run_steps(dma, step, 0, steps, flush)
    ranks_sync()
    assert dma.dma_check(ws) == 0
    # every projected row read once and written once (q to q_out, k and v to the cache)
    nbytes = 2 * wl.B * wl.L * (wl.Hq + 2 * wl.Hkv) * wl.d * 2
    del x
    return {"bytes": nbytes, "ms": sum(ms) / len(ms), "launches": steps}


def time_backward(dma, wl, steps, warmup, flush, dev, ranks_sync):
    """The backward of the prefill step (selection held fixed) on the
    workload: dt, the kept-key lists, the attention backward and the dt chain.
    The forward (run once, untimed) hands over out and each row's normaliser,
    as a training step's forward does."""
    x = make_inputs(wl, device=dev)
    lengths = x["lengths"].cpu().numpy()
    out = torch.empty_like(x["q"])
    lse = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.float32, device=dev)
    dma.dma_forward_prefill(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w, out=out, lse_out=lse)
    g = torch.Generator(device=dev).manual_seed(wl.seed + 100)
    dout = torch.randn(x["q"].shape, generator=g, device=dev).to(torch.bfloat16)
    ws = dma.new_workspace(dma.dma_backward_workspace_size(wl.B, wl.L, wl.Hq, wl.Hkv, wl.d, wl.w), dev)

    def step(i):
        dma.dma_backward_prefill(x["q"], x["k"], x["v"], x["W"], x["A"], x["lengths"], wl.w, out, dout,
                                 workspace=ws, lse_in=lse)

    for i in range(warmup):
        step(i)
        flush.zero_()
    assert dma.dma_check(ws) == 0
    ranks_sync()
    ms = run_steps(dma, step, 0, steps, flush)
    ranks_sync()
    split = run_steps(dma, step, steps, steps, flush, stages=True)
    assert dma.dma_check(ws) == 0
    # the five products of an attention backward (S, dP, dQ, dK, dV): 10 d FLOPs per kept pair per query head
    flops = 10 * wl.d * wl.Hq * kept_pairs(wl.L, wl.w, lengths)
    n = len(split)
    del x
    return {"flops": flops, "ms": sum(ms) / len(ms), "stage_ms": [sum(v[k] for v in split) / n for k in range(3)],
            "launches": 5 * steps}


CDMOE = {"T": 8192, "hidden": 1024, "num_experts": 16384, "top_k": 64, "seed": 11}


def time_cdmoe(dma, steps, warmup, flush, dev, ranks_sync):
    """CDMoE routing at DogeConfig's defaults (hidden 1024, 16384 experts, 64
    per token) for 8192 tokens: router GEMM, routing, embedding-table experts."""
    from doge_dynamic_mask_b200.workloads import make_cdmoe_inputs
    c = CDMOE
    x = make_cdmoe_inputs(c["T"], c["hidden"], c["num_experts"], c["seed"], device=dev)
    ws = dma.new_workspace(dma.dma_cdmoe_workspace_size(c["T"], c["num_experts"]), dev)
    out = torch.empty_like(x["h"])

    def step(i):
        dma.dma_cdmoe_forward(x["h"], x["W_router"], x["down_embed"], x["up_embed"], c["top_k"], out=out,
                              workspace=ws)

    for i in range(warmup):
        step(i)
        flush.zero_()
    assert dma.dma_check(ws) == 0
    ranks_sync()
    ms = run_steps(dma, step, 0, steps, flush)
    ranks_sync()
    split = run_steps(dma, step, steps, steps, flush, stages=True)
    assert dma.dma_check(ws) == 0
    n = len(split)
    # bytes a token must move: its down and up expert rows, h in, the output out
    row_bytes = c["T"] * (2 * c["top_k"] * c["hidden"] * 2 + 2 * c["hidden"] * 2)
    router_flops = 2 * c["T"] * c["hidden"] * 2 * int(round(c["num_experts"] ** 0.5))
    del x
    return {"ms": sum(ms) / len(ms), "stage_ms": [sum(v[k] for v in split) / n for k in range(3)],
            "bytes": row_bytes, "router_flops": router_flops, "launches": 2 * steps}


def time_e2e(dma, wl, steps, warmup, dev):
    """Same metric through the public call with host (pinned) buffers: the H2D
    copy of every input and the D2H read of the output are inside each step.
    A step's inputs (q, k, v, W_dt, A, lengths) sit in one pinned staging
    buffer, each at a 256-byte aligned offset, as a serving loop would fill
    it, and travel in one copy into one of two device buffers that hold the
    same layout (the call reads views of it).  Steps are pipelined as a
    serving loop would run them: step i+1's inputs travel host-to-device (one
    stream) while step i computes (a second) and step i-1's output travels
    device-to-host (a third); every step still copies its own inputs in and
    its own result out."""
    x0 = make_inputs(wl, device="cpu")
    names = list(x0.keys())
    offs, total = {}, 0
    for n in names:
        offs[n] = total
        total += (x0[n].numel() * x0[n].element_size() + 255) // 256 * 256

    def views(buf):
        return {n: buf[offs[n]:offs[n] + x0[n].numel() * x0[n].element_size()].view(x0[n].dtype).view(x0[n].shape)
                for n in names}

    h_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    for n, v in views(h_in).items():
        v.copy_(x0[n])
    lengths = x0["lengths"].numpy()
    d_in = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]
    xd = [views(b) for b in d_in]
    ws = [dma.new_workspace(dma.dma_workspace_size(wl.B, wl.L, wl.L, wl.Hq, wl.Hkv, wl.d, wl.w), dev)
          for _ in range(2)]
    out_d = [torch.empty_like(xd[0]["q"]) for _ in range(2)]
    out_h = [torch.empty(x0["q"].shape, dtype=x0["q"].dtype).pin_memory() for _ in range(2)]
    h2d = total
    d2h = out_h[0].numel() * out_h[0].element_size()
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def step(i):
        k = i & 1
        with torch.cuda.stream(s_in):
            if started[k]:
                s_in.wait_event(ev_comp[k])          # step i-2 has read these inputs
            d_in[k].copy_(h_in, non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[k])
            if started[k]:
                s_comp.wait_event(ev_out[k])         # step i-2's output has left
            dma.dma_forward_prefill(xd[k]["q"], xd[k]["k"], xd[k]["v"], xd[k]["W"], xd[k]["A"], xd[k]["lengths"],
                                    wl.w, out=out_d[k], workspace=ws[k])
            ev_comp[k].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[k])
            out_h[k].copy_(out_d[k], non_blocking=True)
            ev_out[k].record(s_out)
        started[k] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(warmup, warmup + steps):
        step(i)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return {"tflops": prefill_flops(wl, lengths) / (ms * 1e-3) / 1e12, "ms": ms, "h2d": h2d, "d2h": d2h}


def _oracle_worker_init():
    from threadpoolctl import threadpool_limits
    threadpool_limits(1)     # one BLAS thread per worker process


def _oracle_slice(job):
    """One (batch, query head) slice of the prefill through the oracle: dt of
    the whole sequence, then every row of the head."""
    import oracle
    q, k, v, W, A, lengths, w, scale, h = job
    dt = oracle.dt_scores(v, W, A)
    oracle.prefill_rows(q, k, v, dt, lengths, w, scale, 0, h, range(q.shape[1]))
    return h


class OraclePool:
    """Worker processes for the CPU baseline: one per host core this process
    may run on, each with one BLAS thread.  Started with spawn, so it is safe
    to create after CUDA has been initialised."""

    def __init__(self):
        import multiprocessing as mproc
        self.cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
        self.pool = mproc.get_context("spawn").Pool(self.cores, initializer=_oracle_worker_init)

    def close(self):
        self.pool.terminate()
        self.pool.join()


def cpu_baseline_prefill(wl, x, pool, budget_s=12.0):
    """The oracle as it stands on the host cores, on a bounded sample of the
    same workload: whole (batch, query head) slices, each with its own dt of
    the whole sequence, spread over the pool's processes, until every slice
    is done or about budget_s seconds have passed."""
    W = x["W"].double().cpu().numpy()
    A = x["A"].double().cpu().numpy()
    jobs = []
    for b in range(wl.B):
        q = x["q"][b:b + 1].float().cpu().numpy().astype(np.float64)
        k = x["k"][b:b + 1].float().cpu().numpy().astype(np.float64)
        v = x["v"][b:b + 1].float().cpu().numpy().astype(np.float64)
        lengths = x["lengths"][b:b + 1].cpu().numpy()
        for h in range(wl.Hq):
            jobs.append(((q, k, v, W, A, lengths, wl.w, wl.scale, h), lengths))
    t0 = time.perf_counter()
    flops, done = 0, 0
    for i, _ in enumerate(pool.pool.imap(_oracle_slice, [j for j, _ in jobs])):
        flops += prefill_flops(wl.replace(B=1, Hq=1), jobs[i][1])
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt_s = time.perf_counter() - t0
    return {"value": flops / dt_s / 1e12, "unit": "TFLOP/s", "cores": pool.cores, "kind": "oracle",
            "sample": f"{wl.name}: {done} of {wl.B * wl.Hq} (batch, query head) slices, all {wl.L} rows "
                      f"each, dt included, {dt_s:.1f} s over {pool.cores} worker processes (one BLAS thread each)"}


def run_only(args):
    """One workload, timed with the same rules, for profiler command lines."""
    from doge_dynamic_mask_b200 import dma
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wl = WORKLOADS[args.only]
    if args.batch:
        wl = wl.replace(B=args.batch)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    if args.backward:
        r = time_backward(dma, wl, args.steps, args.warmup, flush, dev, torch.cuda.synchronize)
        print(json.dumps({"workload": wl.name + " (backward)", "B": wl.B, "value": r["flops"] / (r["ms"] * 1e-3) / 1e12,
                          "unit": "TFLOP/s", "ms_per_step": r["ms"], "stage_ms": r["stage_ms"],
                          "gpu_launches": r["launches"]}), flush=True)
        return
    if args.cdmoe:
        r = time_cdmoe(dma, args.steps, args.warmup, flush, dev, torch.cuda.synchronize)
        print(json.dumps({"workload": "cdmoe", "value": CDMOE["T"] / (r["ms"] * 1e-3), "unit": "tokens/s",
                          "ms_per_step": r["ms"], "stage_ms": r["stage_ms"],
                          "expert_rows_gbs": r["bytes"] / (r["ms"] * 1e-3) / 1e9}), flush=True)
        return
    if args.prologue:
        r = time_prologue(dma, wl, args.steps, args.warmup, flush, dev, torch.cuda.synchronize)
        print(json.dumps({"workload": wl.name + " (prologue)", "B": wl.B, "value": r["bytes"] / (r["ms"] * 1e-3) / 1e9,
                          "unit": "GB/s", "ms_per_step": r["ms"], "gpu_launches": r["launches"]}), flush=True)
        return
    if args.cached:
        r = time_decode_cached(dma, wl, args.steps, args.warmup, flush, dev, torch.cuda.synchronize)
        line = {"workload": wl.name + " (cached dt)", "B": wl.B, "value": r["bytes"] / (r["ms"] * 1e-3) / 1e9,
                "unit": "GB/s"}
        line.update({"ms_per_step": r["ms"], "stage_ms": r["stage_ms"], "gpu_launches": r["launches"]})
        print(json.dumps(line), flush=True)
        return
    if wl.mode == "prefill":
        r = time_prefill(dma, wl, args.steps, args.warmup, flush, dev, torch.cuda.synchronize)
        line = {"workload": wl.name, "B": wl.B, "value": r["flops"] / (r["ms"] * 1e-3) / 1e12, "unit": "TFLOP/s"}
    else:
        r = time_decode(dma, wl, args.steps, args.warmup, flush, dev, torch.cuda.synchronize)
        line = {"workload": wl.name, "B": wl.B, "value": r["bytes"] / (r["ms"] * 1e-3) / 1e9, "unit": "GB/s"}
    line.update({"ms_per_step": r["ms"], "stage_ms": r["stage_ms"], "gpu_launches": r["launches"]})
    print(json.dumps(line), flush=True)


def run_ours(args):
    from doge_dynamic_mask_b200 import dma
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist

    def ranks_sync():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    def rank_max(v):
        return max_over_ranks(v, pg, dev)

    peaks = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    wl = WORKLOADS[HEADLINE]
    with ClockSampler(local) as clk:
        head = time_prefill(dma, wl, args.steps, args.warmup, flush, dev, ranks_sync)
    clocks = clk.summary()
    ms = rank_max(head["ms"])
    att_ms = rank_max(head["stage_ms"][2])
    value = aggregate_throughput(head["flops"], ms, world) / 1e12
    att_tflops = head["flops"] / (att_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "attn_prefill_kernel<64>", "achieved": round(att_tflops, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(att_tflops / peaks["bf16_tflops"], 4),
                "peak_source": f"{peaks['source']} bf16 burst",
                "traffic": kernel_traffic("attn_prefill_kernel<64>"), "traffic_unit": "bytes per launch",
                "per_launch": {"flops": head["flops"], "ms": round(att_ms, 5)}}

    result = {"metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
              "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
              "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
              "data": "synthetic",
              "config": {"workload": wl.name, "B": wl.B, "L": wl.L, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d,
                         "keep_window_size": wl.w, "l2": "flushed between timed steps (256 MiB write)",
                         "parallelism": f"replicas{world}"},
              "stage_ms": {"dt": round(head["stage_ms"][0], 5), "select": round(head["stage_ms"][1], 5),
                           "attention": round(head["stage_ms"][2], 5)},
              "roofline": roofline, "gpu_launches": head["launches"], "clocks": clocks}
    del head

    # the other workloads of the same method (same timing rules)
    others = {}
    if not args.quick:
        for name in ("sparse_pad", "long"):
            o = time_prefill(dma, WORKLOADS[name], args.steps, args.warmup, flush, dev, ranks_sync)
            oms = rank_max(o["ms"])
            a_ms = rank_max(o["stage_ms"][2])
            others[name] = {"value": round(aggregate_throughput(o["flops"], oms, world) / 1e12, 3), "unit": "TFLOP/s",
                            "valid_rows_value": round(aggregate_throughput(o["flops_valid"], oms, world) / 1e12, 3),
                            "ms_per_step": round(oms, 5),
                            "attention_tflops": round(o["flops"] / (a_ms * 1e-3) / 1e12, 2),
                            "attention_frac": round(o["flops"] / (a_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                            "stage_ms": [round(s, 5) for s in o["stage_ms"]]}
            result["gpu_launches"] += o["launches"]
            del o
            torch.cuda.empty_cache()
        d = time_decode(dma, WORKLOADS["decode"], args.steps, args.warmup, flush, dev, ranks_sync)
        dms = rank_max(d["ms"])
        dt_ms = rank_max(d["stage_ms"][0])
        gbs = d["bytes"] / (dms * 1e-3) / 1e9
        v_scan = WORKLOADS["decode"].B * WORKLOADS["decode"].L * WORKLOADS["decode"].Hkv * WORKLOADS["decode"].d * 2
        others["decode"] = {"value": round(world * gbs, 1), "unit": "GB/s", "ms_per_step": round(dms, 5),
                            "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
                            "bytes_per_step": d["bytes"], "stage_ms": [round(s, 5) for s in d["stage_ms"]],
                            "dt_kernel_gbs": round(v_scan / (dt_ms * 1e-3) / 1e9, 1)}
        result["gpu_launches"] += d["launches"]
        del d
        torch.cuda.empty_cache()
        bw = time_backward(dma, WORKLOADS[HEADLINE], args.steps, args.warmup, flush, dev, ranks_sync)
        bms = rank_max(bw["ms"])
        others["backward_dense_eq"] = {
            "value": round(aggregate_throughput(bw["flops"], bms, world) / 1e12, 3), "unit": "TFLOP/s",
            "ms_per_step": round(bms, 5), "frac_of_bf16_peak": round(bw["flops"] / (bms * 1e-3) / 1e12 /
                                                                      peaks["bf16_tflops"], 4),
            "stage_ms": [round(x_, 5) for x_ in bw["stage_ms"]],
            "note": "backward of the headline workload (selection held fixed, row normalisers from the forward): dt, kept-key lists, attention "
                    "backward and dt chain; 10 d FLOPs per kept pair per query head"}
        result["gpu_launches"] += bw["launches"]
        del bw
        torch.cuda.empty_cache()
        cm = time_cdmoe(dma, args.steps, args.warmup, flush, dev, ranks_sync)
        cms_ = rank_max(cm["ms"])
        others["cdmoe"] = {"value": round(world * CDMOE["T"] / (cms_ * 1e-3), 1), "unit": "tokens/s",
                           "ms_per_step": round(cms_, 5),
                           "expert_rows_gbs": round(cm["bytes"] / (cms_ * 1e-3) / 1e9, 1),
                           "frac_of_hbm": round(cm["bytes"] / (cms_ * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                           "router_tflops": round(cm["router_flops"] / (cm["stage_ms"][0] * 1e-3) / 1e12, 2)
                           if cm["stage_ms"][0] > 0 else None,
                           "stage_ms": [round(x_, 5) for x_ in cm["stage_ms"]],
                           "config": dict(CDMOE)}
        result["gpu_launches"] += cm["launches"]
        del cm
        torch.cuda.empty_cache()
        pr = time_prologue(dma, WORKLOADS["long"], args.steps, args.warmup, flush, dev, ranks_sync)
        pms = rank_max(pr["ms"])
        others["prologue_long"] = {"value": round(world * pr["bytes"] / (pms * 1e-3) / 1e9, 1), "unit": "GB/s",
                                   "ms_per_step": round(pms, 5),
                                   "frac_of_hbm": round(pr["bytes"] / (pms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                   "bytes_per_step": pr["bytes"],
                                   "note": "q/k RMSNorm + rotary embedding + KV-cache append of the long "
                                           "workload's 32768 tokens"}
        result["gpu_launches"] += pr["launches"]
        del pr
        torch.cuda.empty_cache()
        c = time_decode_cached(dma, WORKLOADS["decode"], args.steps, args.warmup, flush, dev, ranks_sync)
        cms = rank_max(c["ms"])
        others["decode_cached"] = {"value": round(world * c["bytes"] / (cms * 1e-3) / 1e9, 1), "unit": "GB/s",
                                   "ms_per_step": round(cms, 5),
                                   "frac_of_hbm": round(c["bytes"] / (cms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                   "bytes_per_step": c["bytes"], "stage_ms": [round(x, 5) for x in c["stage_ms"]],
                                   "note": "incremental steps with cached dt (one new token per sequence per step)"}
        result["gpu_launches"] += c["launches"]
        del c
        torch.cuda.empty_cache()
    result["workloads"] = others

    e2e = time_e2e(dma, wl, max(3, args.steps), args.warmup, dev)
    result["e2e"] = {"value": round(world * e2e["tflops"], 3), "unit": "TFLOP/s", "h2d_bytes_per_step": e2e["h2d"],
                     "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": round(e2e["ms"], 4)}
    if rank == 0:
        x = make_inputs(wl, device="cpu")
        pool = OraclePool()
        try:
            result["cpu_baseline"] = cpu_baseline_prefill(wl, x, pool)
        finally:
            pool.close()
        print(json.dumps(result), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[HEADLINE]
    x = make_inputs(wl, device="cpu")
    lengths = x["lengths"].numpy()
    per_step = []
    pool = OraclePool()
    try:
        for i in range(args.warmup + args.steps):
            r = cpu_baseline_prefill(wl, x, pool, budget_s=8.0)
            if i >= args.warmup:
                per_step.append(r)
    finally:
        pool.close()
    value = statistics.mean(r["value"] for r in per_step)
    total_flops = prefill_flops(wl, lengths)
    line = {"metric": METRIC, "impl": "reference", "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_flops / (value * 1e12) * 1e3 if value > 0 else None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "L": wl.L, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d,
                       "keep_window_size": wl.w},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": per_step[0]["cores"], "kind": "oracle",
                             "sample": per_step[0]["sample"] + " per step; ms_per_step extrapolated to the whole workload"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="headline workload only")
    ap.add_argument("--only", choices=sorted(WORKLOADS), help="time one workload only (profiling)")
    ap.add_argument("--batch", type=int, default=0, help="with --only: override the batch size")
    ap.add_argument("--cached", action="store_true", help="with --only decode: incremental steps with cached dt")
    ap.add_argument("--prologue", action="store_true", help="with --only: time the prologue on that geometry")
    ap.add_argument("--backward", action="store_true", help="with --only: time the backward on that workload")
    ap.add_argument("--cdmoe", action="store_true", help="with --only (any): time the CDMoE routing workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.only:
        run_only(args)
    elif args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # not launched by torchrun: start one process per GPU here
        if torch.cuda.device_count() < args.gpus:
            sys.exit(f"bench.py --gpus {args.gpus}: only {torch.cuda.device_count()} GPU(s) visible")
        sys.exit(spawn_ranks(args.gpus, run_ours, args))
    else:
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if world != args.gpus and args.gpus != 1:
            sys.exit(f"bench.py --gpus {args.gpus} under a launcher with WORLD_SIZE={world}")
        run_ours(args)


if __name__ == "__main__":
    main()
