#!/usr/bin/env python
"""Benchmark of the QSA layer (libqsa) on B200.

One step = one pass of the whole layer over one batch of seeded synthetic input:
  prefill (headline, 1,048,576-token context, last 16,384-token chunk, batch 1):
      compress the chunk's indexer keys -> score + select (top-512 + tail) -> sparse attention
  decode (reported beside it, 1,048,576-token context, 4 sequences x 4 positions):
      compress the new block -> score + select -> split-K sparse attention (last split merges)
The settings are those of the article "Qwen's million-token window has a 2,048-token keyhole",
section "Three speed claims, three different experiments".  The dense paged-GQA kernel of the
same library runs on the same pools for the sparse/dense ratio, and the fp64 oracle is timed on
the host cores as a baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs an independent replica of the
workload (the layer shards by sequence with no data-path collective); the timed region is
bracketed by a barrier and synchronisation and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QSA prefill tok/s and decode µs/step at 1M ctx; % of HBM/tensor roofline"
PREFILL = "C4"
DECODE = "C5"
DISTILL = "DISTILL"


# ------------------------------------------------------------------------------------ helpers

def log(msg: str):
    print(f"[bench] {msg}", file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), tf=float(d["bf16_tflops"]),
                    tf_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, tf=1590.0, tf_sus=1400.0, src="fallback")


def DISTILL_CONFIG():
    """The distillation-signal workload: a 1,024-token chunk at 65,536 tokens of context with the
    layer's heads (32q/4kv x 128, indexer 4 x 128)."""
    from qsa_synth import Config

    return Config("distill_chunk1024_ctx65536", "prefill", 1, 65536, 1024, 32, 4, 128, 4, 128,
                  needles=64, shuffle_pages=True, seed=0x05A6)


# The library's kernels per decode step (three calls): compress, the indexer's score and merge
# launches (the merge runs the exact selection itself for a row it cannot settle), the split-K
# arrival-counter reset, and the sparse attention.
DECODE_LAUNCHES_PER_STEP = 5


def prefill_launches_per_step(c) -> int:
    """The library's kernels per prefill step at idx_dim 128 (automatic score path): compress, the
    tensor-core indexer -- in its stream-K form a sample launch, a scan, the stream launch and a
    select launch, else one launch -- then the exact-fallback check, and the sparse attention.
    The form follows the library's geometry rule: stream-K when spreading the row tiles' key tiles
    over 148 CTAs saves more than its own cost of about 100 tile times."""
    R = (c.num_q + 127) // 128                   # 128-row tiles
    T = ((c.ctx - 1) // 4 + 127) // 128 + 1      # 128-block key tiles up to the largest position
    waves = (R + 147) // 148
    stream = R * T // 148 + 100 < waves * T
    return 1 + (4 if stream else 1) + 1 + 1


def positions_of(t: int, topk: int = 512) -> int:
    """Token positions attended by query position t: selected blocks plus the clipped tail."""
    n = min(topk, t // 4)
    return 4 * n + (t % 4) + 1


def algorithmic(c, q_pos):
    """Useful work per step (bytes or flops) of each stage, as defined for the roofline."""
    import numpy as np

    t = np.asarray(q_pos, dtype=np.int64)
    kv_row = c.Hkv * c.D * 2  # bytes of one K (or V) position row, all kv heads
    pos = np.array([positions_of(int(x), c.topk) for x in t], dtype=np.int64)
    per_seq_max = t.reshape(c.batch, -1).max(axis=1)
    return {
        "compress_bytes": c.num_q * c.Di * 2 + (c.num_q // 4) * c.Di * 2,
        "score_flops": int(2 * c.Hi * c.Di * (t // 4).sum()),
        "score_bytes_decode": int(((per_seq_max // 4) * c.Di * 2).sum()),
        "attn_bytes": int(pos.sum() * kv_row * 2),
        "attn_flops": int(pos.sum() * 4 * c.Hq * c.D),
        "dense_flops": int((4 * c.Hq * c.D * (t + 1)).sum()),
        "dense_bytes_decode": int(((per_seq_max + 1) * kv_row * 2).sum()),
    }


class Clocks:
    """nvidia-smi samples (200 ms) during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="qsa_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}", "--format=csv,noheader",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if not self.path or not os.path.exists(self.path):
            return out
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1].split()[0]))
                smax.append(float(f[2].split()[0]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if sm:
            out.update(sm_mhz=statistics.median(sm), sm_max_mhz=max(smax), samples=len(sm))
        out["reasons"] = sorted(reasons)
        return out


def traffic_for(kernel_file: str, key: str):
    """dram bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(key)
    except (OSError, ValueError):
        return None
    if not d:
        return None
    files = kernel_file if isinstance(kernel_file, (list, tuple)) else [kernel_file]
    srcs = [os.path.join(ROOT, "learned_block_sparse_qsa_b200", "csrc", f) for f in files]
    return d["bytes_per_launch"] if d.get("source_sha") == code_sha(*srcs) else None


def code_sha(*paths: str) -> str:
    """Hash of CUDA sources with comments and blank space removed: counters stay attached to
    the code they were taken on, and an edit of a comment does not orphan them."""
    text = "\n".join(open(p, encoding="utf-8").read() for p in paths)
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = " ".join(text.split())
    return hashlib.sha256(text.encode()).hexdigest()[:16]


# ------------------------------------------------------------------------------------ workload

class Workload:
    """Device inputs + runner for one config (the prefix of the context already compressed)."""

    def __init__(self, name: str, device, chunk: int = 0):
        import torch

        from learned_block_sparse_qsa_b200 import QsaConfig, QsaRunner
        from qsa_synth import CONFIGS
        from qsa_synth.device import DeviceInputs

        self.torch = torch
        base = CONFIGS[name] if name in CONFIGS else DISTILL_CONFIG()
        self.c = c = base if not chunk else base.replace(n_new=chunk)
        self.di = d = DeviceInputs(c, integer=False, device=device)
        self.cfg = QsaConfig.make(c.Hq, c.Hkv, c.D, c.Di, topk=c.topk)
        self.runner = QsaRunner(self.cfg, device)
        self.b = self.runner.batch(batch=c.batch, num_q=c.num_q, max_pages=c.max_pages,
                                   num_pages=c.num_pages, max_pos=c.ctx - 1, q_seq=d.q_seq,
                                   q_pos=d.q_pos, page_table=d.page_table)
        self.sel = torch.empty(c.num_q, c.topk + 1, dtype=torch.int32, device=device)
        self.n_sel = torch.empty(c.num_q, dtype=torch.int32, device=device)
        self.out = torch.empty_like(d.q)
        for s in range(c.batch):
            rows, seq, pos = d.prefix_rows(s)
            if rows.shape[0]:
                self.runner.compress(self.b, rows, seq, pos, d.kcomp_pool)
        torch.cuda.synchronize()
        self.q_pos_host = d.host.rows()[1]

    def stage_calls(self, decode: bool):
        """The step as a list of (stage name, callable) on the current stream."""
        from learned_block_sparse_qsa_b200 import (QSA_OP_SPARSE_ATTN_DECODE, qsa_sparse_attn_decode,
                                                   qsa_sparse_attn_prefill)

        d, r, b, cfg = self.di, self.runner, self.b, self.cfg
        calls = [("compress", lambda: r.compress(b, d.idx_k_new, d.new_seq, d.new_pos, d.kcomp_pool)),
                 ("score_topk", lambda: r.select(b, d.idx_q, d.idx_w, d.kcomp_pool, self.sel, self.n_sel))]
        if decode:
            ws, n = r.workspace(b, QSA_OP_SPARSE_ATTN_DECODE, 0)
            calls.append(("sparse_attn", lambda: qsa_sparse_attn_decode(
                cfg, b, d.q, d.k_pool, d.v_pool, self.sel, self.n_sel, self.out, None, 0, ws, n)))
        else:
            calls.append(("sparse_attn", lambda: qsa_sparse_attn_prefill(
                cfg, b, d.q, d.k_pool, d.v_pool, self.sel, self.n_sel, self.out)))
        return calls

    def step(self, decode: bool):
        for _, f in self.stage_calls(decode):
            f()


def time_steps(w: Workload, decode: bool, steps: int, warmup: int, dist, flush=None):
    """Per-stage and whole-step device times (ms) over `steps` timed steps."""
    torch = w.torch
    calls = w.stage_calls(decode)
    for _ in range(warmup):
        for _, f in calls:
            f()
    torch.cuda.synchronize()
    names = [n for n, _ in calls]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        if flush is not None:
            flush()
        ev[i][0].record()
        for j, (_, f) in enumerate(calls):
            f()
            ev[i][j + 1].record()
    t1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    stage_ms = {n: 0.0 for n in names}
    step_ms = []
    for i in range(steps):
        for j, n in enumerate(names):
            stage_ms[n] += ev[i][j].elapsed_time(ev[i][j + 1])
        step_ms.append(ev[i][0].elapsed_time(ev[i][-1]))
    return {n: v / steps for n, v in stage_ms.items()}, step_ms, t0.elapsed_time(t1)


def max_over_ranks(x: float, dist) -> float:
    """The largest of every rank's x (all ranks call it in the same order)."""
    if not dist:
        return x
    import torch

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank_step: int, steps: int, max_total_ms: float) -> float:
    """Whole-job units/s: every rank processes its own replica's units each step, and the job
    takes as long as the slowest rank."""
    return world * units_per_rank_step * steps / (max_total_ms / 1000.0)


def graph_decode_us(w: Workload, steps: int, warmup: int, flush):
    """Decode step captured in one CUDA graph; mean replay time (us), L2 flushed in between."""
    torch = w.torch
    for _ in range(max(warmup, 1)):
        w.step(True)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        w.step(True)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        w.step(True)
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        ts.append((a, b))
    torch.cuda.synchronize()
    us = [a.elapsed_time(b) * 1000 for a, b in ts]
    del g
    return statistics.mean(us), us


def fused_decode_us(w: Workload, steps: int, warmup: int, flush):
    """The fused one-launch decode step (qsa_decode_step), replayed as a one-node CUDA graph with
    L2 flushed before each replay (eager launches when the graph cannot be captured).  Checks its
    output against the three-call step's before timing."""
    torch = w.torch
    from learned_block_sparse_qsa_b200 import QSA_OP_DECODE_STEP, qsa_decode_step, qsa_workspace_size

    c, d, b = w.c, w.di, w.b
    n = qsa_workspace_size(w.cfg, b, QSA_OP_DECODE_STEP, 0)
    ws = torch.zeros(n, dtype=torch.uint8, device=d.q.device)
    out = torch.empty_like(w.out)

    def one():
        qsa_decode_step(w.cfg, b, d.idx_k_new, d.new_seq, d.new_pos, d.new_seq.numel(), d.kcomp_pool,
                        d.idx_q, d.idx_w, d.q, d.k_pool, d.v_pool, w.sel, w.n_sel, None, out, None, 0,
                        ws, n)

    one()
    w.step(True)
    torch.cuda.synchronize()
    if not torch.equal(out.view(torch.int16), w.out.view(torch.int16)):
        raise RuntimeError("fused decode step output differs from the three-call step")
    mode = "cuda_graph"
    g = None
    try:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            one()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            one()
    except Exception as e:  # pragma: no cover - capture support depends on the driver
        log(f"fused step not capturable ({e}); timing eager launches")
        g, mode = None, "eager"
        torch.cuda.synchronize()
    run = g.replay if g is not None else one
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        a.record()
        run()
        e.record()
        ts.append((a, e))
    torch.cuda.synchronize()
    del g
    return statistics.mean(x.elapsed_time(y) * 1000 for x, y in ts), mode


class Staging:
    """One pinned host buffer holding every per-step input of a workload, and device buffers it is
    copied into with a single host-to-device copy; tensors are 256-byte aligned views."""

    def __init__(self, torch, host_tensors: dict, copies: int, device):
        self.torch = torch
        self.layout, off = {}, 0
        for name, t in host_tensors.items():
            n = t.numel() * t.element_size()
            self.layout[name] = (off, t.dtype, tuple(t.shape), n)
            off += (n + 255) // 256 * 256
        self.nbytes = off
        self.host = torch.empty(off, dtype=torch.uint8).pin_memory()
        for name, t in host_tensors.items():
            o, _, _, n = self.layout[name]
            self.host[o:o + n].copy_(t.contiguous().view(-1).view(torch.uint8))
        self.dev = [torch.empty(off, dtype=torch.uint8, device=device) for _ in range(copies)]

    def view(self, i: int, name: str):
        o, dt, shape, n = self.layout[name]
        return self.dev[i][o:o + n].view(dt).view(shape)

    def h2d(self, i: int):
        self.dev[i].copy_(self.host, non_blocking=True)


def e2e_prefill(w: Workload, steps: int, warmup: int):
    """Whole step through the public API with host inputs: one host-to-device copy of the chunk's
    inputs (queries, indexer queries/weights/keys, the new K/V pages), the new pages scattered into
    the cache, the layer, one device-to-host copy of the output.  Successive steps are pipelined:
    step k+1's inputs travel (own stream, double buffer) while step k computes, and step k's
    output travels back (own stream) while step k+1 computes."""
    torch = w.torch
    c, d, r, b = w.c, w.di, w.runner, w.b
    lp0, lp1 = c.ctx_start // 64, (c.ctx - 1) // 64 + 1
    pages = d.page_table[0, lp0:lp1].long()
    st = Staging(torch, {"q": d.q.cpu(), "idx_q": d.idx_q.cpu(), "idx_w": d.idx_w.cpu(),
                         "idx_k": d.idx_k_new.cpu(), "k": d.k_pool[pages].cpu(),
                         "v": d.v_pool[pages].cpu()}, 2, d.q.device)
    outs = [torch.empty_like(d.q) for _ in range(2)]
    hout = torch.empty(d.q.shape, dtype=d.q.dtype).pin_memory()
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for k in range(n):
            i = k % 2
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(ev_done[i])  # step k-2 is done with staging buffer i
                st.h2d(i)
                ev_in[i].record(s_in)
            comp.wait_event(ev_in[i])
            if k >= 2:
                comp.wait_event(ev_out[i])       # step k-2's output has left outs[i]
            d.k_pool.index_copy_(0, pages, st.view(i, "k"))
            d.v_pool.index_copy_(0, pages, st.view(i, "v"))
            r.prefill(b, q=st.view(i, "q"), idx_q=st.view(i, "idx_q"), idx_w=st.view(i, "idx_w"),
                      kcomp_pool=d.kcomp_pool, k_pool=d.k_pool, v_pool=d.v_pool, out=outs[i],
                      sel=w.sel, n_sel=w.n_sel, idx_k_new=st.view(i, "idx_k"), new_seq=d.new_seq,
                      new_pos=d.new_pos)
            ev_done[i].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                hout.copy_(outs[i], non_blocking=True)
                ev_out[i].record(s_out)

    run(warmup)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    run(steps)
    e.record(s_out)
    torch.cuda.synchronize()
    ms = a.elapsed_time(e) / steps
    # the pipelined result must be the layer's: compare with one plain device step
    w.step(False)
    torch.cuda.synchronize()
    if not torch.equal(hout.view(torch.int16), w.out.cpu().view(torch.int16)):
        raise RuntimeError("end-to-end prefill output differs from the device step's output")
    d2h = hout.numel() * hout.element_size()
    return ms, st.nbytes, d2h


def e2e_decode(w: Workload, steps: int, warmup: int):
    """Whole decode step through the public API with host inputs: one host-to-device copy of the
    step's inputs (queries, indexer tensors, the new tokens' K/V rows), the rows scattered into the
    cache, the layer, one device-to-host copy of the output every step; the step is captured once
    as a CUDA graph and replayed."""
    torch = w.torch
    c, d = w.c, w.di
    q_pos = d.q_pos.long()
    q_seq = d.q_seq.long()
    pages = d.page_table[q_seq, q_pos // 64].long()
    slots = (q_pos % 64).long()
    st = Staging(torch, {"q": d.q.cpu(), "idx_q": d.idx_q.cpu(), "idx_w": d.idx_w.cpu(),
                         "idx_k": d.idx_k_new.cpu(), "k": d.k_pool[pages, slots].cpu(),
                         "v": d.v_pool[pages, slots].cpu()}, 1, d.q.device)
    hout = torch.empty(d.q.shape, dtype=d.q.dtype).pin_memory()
    from learned_block_sparse_qsa_b200 import QSA_OP_SPARSE_ATTN_DECODE, qsa_sparse_attn_decode

    r, b, cfg = w.runner, w.b, w.cfg
    ws, nws = r.workspace(b, QSA_OP_SPARSE_ATTN_DECODE, 0)

    def one():
        st.h2d(0)
        d.k_pool[pages, slots] = st.view(0, "k")
        d.v_pool[pages, slots] = st.view(0, "v")
        r.compress(b, st.view(0, "idx_k"), d.new_seq, d.new_pos, d.kcomp_pool)
        r.select(b, st.view(0, "idx_q"), st.view(0, "idx_w"), d.kcomp_pool, w.sel, w.n_sel)
        qsa_sparse_attn_decode(cfg, b, st.view(0, "q"), d.k_pool, d.v_pool, w.sel, w.n_sel, w.out,
                               None, 0, ws, nws)
        hout.copy_(w.out, non_blocking=True)

    # the whole step -- copy in, scatter, the layer's calls, copy out -- as one CUDA graph, the
    # way a serving loop replays it
    for _ in range(max(warmup, 1)):
        one()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        one()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        one()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        g.replay()
    e.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(e) * 1000 / steps
    del g
    w.step(True)
    torch.cuda.synchronize()
    if not torch.equal(hout.view(torch.int16), w.out.cpu().view(torch.int16)):
        raise RuntimeError("end-to-end decode output differs from the device step's output")
    return us, st.nbytes, hout.numel() * hout.element_size()


def dense_time_ms(w: Workload, decode: bool, reps: int, flush=None):
    torch = w.torch
    d = w.di
    out = torch.empty_like(w.out)
    w.runner.dense(w.b, q=d.q, k_pool=d.k_pool, v_pool=d.v_pool, out=out, decode=decode)
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        if flush:
            flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        w.runner.dense(w.b, q=d.q, k_pool=d.k_pool, v_pool=d.v_pool, out=out, decode=decode)
        b.record()
        ts.append((a, b))
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in ts)


# ------------------------------------------------------------------------------------ oracle

def _oracle_rows(h, kc, rows, workers: int):
    """Wall seconds of the oracle's selection and attention for the given query rows, run on
    `workers` host threads (BLAS limited to one thread each).  Inputs are generated outside the
    timed parts: the rows' queries first, then the K/V rows the selections name."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np
    from threadpoolctl import threadpool_limits

    from oracle import qsa_oracle as orc

    _, q_pos = h.rows()
    rows = list(rows)
    iq, iw, qq = h.idx_q(rows), h.idx_w(rows), h.q(rows)
    q_seq = h.rows()[0]
    with threadpool_limits(limits=1), ThreadPoolExecutor(max_workers=workers) as ex:
        def sel(i):
            t = int(q_pos[rows[i]])
            s, _ = orc.qsa_select(kc[int(q_seq[rows[i]])], iq[i], iw[i], t)
            return orc.expand(s, t)

        t0 = time.perf_counter()
        pos = list(ex.map(sel, range(len(rows))))
        t_sel = time.perf_counter() - t0
        kv = [h.kv(int(q_seq[r]), p) for r, p in zip(rows, pos)]   # input regeneration, untimed
        t0 = time.perf_counter()
        list(ex.map(lambda i: orc.attend(qq[i], *kv[i]), range(len(rows))))
        t_att = time.perf_counter() - t0
    return t_sel + t_att


def oracle_workers() -> int:
    return max(1, os.cpu_count() or 1)


def oracle_prefill_baseline(rows_per_step: int, steps: int):
    """The fp64 oracle on the host cores, on a bounded sample of the prefill workload: the
    chunk's compression, then selection + attention of evenly spaced query rows on one host
    thread per core."""
    import numpy as np

    from oracle import qsa_oracle as orc
    from qsa_synth import CONFIGS, HostInputs

    c = CONFIGS[PREFILL]
    h = HostInputs(c)
    kc_prefix = orc.compress(h.idx_k(0, 0, c.ctx_start))       # setup, not timed
    chunk_keys = h.idx_k(0, c.ctx_start, c.ctx)
    t0 = time.perf_counter()
    kc_chunk = orc.compress(chunk_keys)
    t_compress = time.perf_counter() - t0
    kc = {0: np.concatenate([kc_prefix, kc_chunk])}
    n = rows_per_step * steps
    rows = np.linspace(0, c.num_q - 1, n).round().astype(int)
    workers = oracle_workers()
    t_rows = _oracle_rows(h, kc, rows, workers)
    per_token = t_compress / c.num_q + t_rows / n
    return dict(value=1.0 / per_token, unit="tok/s", cores=workers, kind="oracle",
                sample=f"{n} evenly spaced query rows of the {c.num_q}-token chunk at "
                       f"{c.ctx}-token context (selection + attention each, {workers} threads, "
                       f"BLAS one thread each) plus the chunk's compression; tok/s extrapolated "
                       f"from seconds per token",
                seconds=t_compress + t_rows)


def oracle_decode_baseline():
    """The fp64 oracle on one sequence of the decode step: its new block's compression and the
    selection + attention of its 4 query positions on 4 host threads; the step (4 sequences, one
    after the other) is extrapolated as 4 times that."""
    import numpy as np

    from oracle import qsa_oracle as orc
    from qsa_synth import CONFIGS, HostInputs

    c = CONFIGS[DECODE]
    h = HostInputs(c)
    kc_prefix = orc.compress(h.idx_k(0, 0, c.ctx_start))       # setup, not timed
    new_keys = h.idx_k(0, c.ctx_start, c.ctx)
    t0 = time.perf_counter()
    kc_new = orc.compress(new_keys)
    t_compress = time.perf_counter() - t0
    kc = {0: np.concatenate([kc_prefix, kc_new])}
    t_rows = _oracle_rows(h, kc, range(c.n_new), c.n_new)
    us = (t_compress + t_rows) * c.batch * 1e6
    return dict(value=us, unit="us/step", cores=c.n_new, kind="oracle",
                sample=f"sequence 0 of {c.batch}: its new block's compression and its {c.n_new} "
                       f"query positions (selection + attention, {c.n_new} threads) at "
                       f"{c.ctx}-token context; the step is extrapolated as {c.batch} x that")


# ------------------------------------------------------------------------------------ training

def _time_ms(torch, fn, reps: int) -> float:
    fn()
    torch.cuda.synchronize()
    ev = []
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        ev.append((a, b))
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def _distill_workspace(cfg, b, device):
    """Workspace of the distillation call (None and 0 where its form needs none)."""
    import torch

    from learned_block_sparse_qsa_b200 import QSA_OP_DISTILL_KL, qsa_workspace_size

    n = qsa_workspace_size(cfg, b, QSA_OP_DISTILL_KL)
    return (torch.empty(n, dtype=torch.uint8, device=device) if n else None), n


def training_kernels(w: Workload, peaks, reps: int = 3):
    """The training-side kernels on the prefill workload's device inputs: the sparse attention
    backward (16,384 rows at 1M context, gradients accumulated into fp32 cache-shaped pools), and
    the indexer-distillation signal on a 1,024-row chunk at 65,536 tokens of context (dense work:
    two q.k passes over each row's whole context)."""
    import numpy as np

    torch = w.torch
    from learned_block_sparse_qsa_b200 import qsa_index_distill_kl, qsa_sparse_attn_backward

    c, d, r, b = w.c, w.di, w.runner, w.b
    lse = torch.empty(c.num_q, c.Hq, dtype=torch.float32, device=d.q.device)
    w.step(False)
    from learned_block_sparse_qsa_b200 import qsa_sparse_attn_prefill

    qsa_sparse_attn_prefill(w.cfg, b, d.q, d.k_pool, d.v_pool, w.sel, w.n_sel, w.out, lse)
    dout = torch.randn(d.q.shape, device=d.q.device, generator=torch.Generator(device=d.q.device).manual_seed(1)).to(torch.bfloat16)
    dq = torch.empty(d.q.shape, dtype=torch.float32, device=d.q.device)
    dk = torch.zeros(d.k_pool.shape, dtype=torch.float32, device=d.q.device)
    dv = torch.zeros_like(dk)
    bwd_ms = _time_ms(torch, lambda: qsa_sparse_attn_backward(
        w.cfg, b, d.q, d.k_pool, d.v_pool, w.sel, w.n_sel, w.out, lse, dout, dq, dk, dv), reps)
    work = algorithmic(c, w.q_pos_host)
    bwd_flops = work["attn_flops"] * 2.5  # S, dA, dQ, dK, dV products: 5 of the forward's 2
    del dk, dv, dq, dout
    torch.cuda.empty_cache()

    wd = Workload(DISTILL, d.q.device)
    cd = wd.c
    kl = torch.empty(cd.num_q, dtype=torch.float32, device=d.q.device)
    dd = wd.di
    wd.step(False)  # compresses the chunk's keys
    dws, dn = _distill_workspace(wd.cfg, wd.b, d.q.device)
    dist_ms = _time_ms(torch, lambda: qsa_index_distill_kl(
        wd.cfg, wd.b, dd.q, dd.k_pool, dd.idx_q, dd.idx_w, dd.kcomp_pool, kl, workspace=dws,
        ws_bytes=dn), reps)
    t = np.asarray(wd.q_pos_host, dtype=np.int64)
    dist_flops = int((2 * cd.Hq * cd.D * (t + 1 + 4 * (t // 4))).sum() + (2 * 4 * cd.Di * (t // 4)).sum())
    del wd
    torch.cuda.empty_cache()
    return {
        "sparse_attn_backward": {"workload": c.name, "ms": bwd_ms, "tokens_per_s": c.num_q / (bwd_ms * 1e-3),
                                 "gathered_gbs": work["attn_bytes"] / (bwd_ms * 1e-3) / 1e9,
                                 "tflops": bwd_flops / (bwd_ms * 1e-3) / 1e12,
                                 "note": "dk/dv added to fp32 pools by vector atomics"},
        "distill_kl": {"workload": cd.name, "ms": dist_ms, "tflops": dist_flops / (dist_ms * 1e-3) / 1e12,
                       "peak_tflops": peaks["tf"], "frac": dist_flops / (dist_ms * 1e-3) / 1e12 / peaks["tf"],
                       "kernel": "tcgen05" if dn else "mma.sync"},
    }


def training_kernels_case(w: Workload, reps: int):
    """The attention backward and the distillation signal on one --case workload (ncu target)."""
    torch = w.torch
    from learned_block_sparse_qsa_b200 import (qsa_index_distill_kl, qsa_sparse_attn_backward,
                                               qsa_sparse_attn_prefill)

    c, d, b = w.c, w.di, w.b
    lse = torch.empty(c.num_q, c.Hq, dtype=torch.float32, device=d.q.device)
    qsa_sparse_attn_prefill(w.cfg, b, d.q, d.k_pool, d.v_pool, w.sel, w.n_sel, w.out, lse)
    dout = torch.ones(d.q.shape, dtype=torch.bfloat16, device=d.q.device)
    dq = torch.empty(d.q.shape, dtype=torch.float32, device=d.q.device)
    dk = torch.zeros(d.k_pool.shape, dtype=torch.float32, device=d.q.device)
    dv = torch.zeros_like(dk)
    kl = torch.empty(c.num_q, dtype=torch.float32, device=d.q.device)
    bwd = _time_ms(torch, lambda: qsa_sparse_attn_backward(w.cfg, b, d.q, d.k_pool, d.v_pool, w.sel, w.n_sel,
                                                           w.out, lse, dout, dq, dk, dv), reps)
    dws, dn = _distill_workspace(w.cfg, b, d.q.device)
    dst = _time_ms(torch, lambda: qsa_index_distill_kl(w.cfg, b, d.q, d.k_pool, d.idx_q, d.idx_w,
                                                       d.kcomp_pool, kl, workspace=dws,
                                                       ws_bytes=dn), reps)
    return {"sparse_attn_backward_ms": bwd, "distill_kl_ms": dst}


# ------------------------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--case", default="", help="time one workload (C1..C5) only, per stage")
    ap.add_argument("--chunk", type=int, default=0, help="with --case: new tokens per sequence")
    ap.add_argument("--fused", action="store_true", help="with a decode --case: the one-launch step too")
    ap.add_argument("--train", action="store_true",
                    help="with a prefill --case: the attention backward and the distillation signal")
    ap.add_argument("--dense", action="store_true",
                    help="with a --case: the dense paged-GQA baseline on the same inputs too")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    peaks = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            return
        steps = max(1, args.steps)
        base = oracle_prefill_baseline(rows_per_step=4, steps=steps)
        from qsa_synth import CONFIGS

        c = CONFIGS[PREFILL]
        line = {"metric": METRIC, "value": base["value"], "unit": "tok/s", "impl": "reference",
                "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
                "ms_per_step": 1000.0 * base["seconds"] / steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": c.name, "batch": c.batch, "ctx": c.ctx, "chunk": c.n_new},
                "cpu_baseline": {k: base[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": base["value"], "unit": "tok/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch

    if args.case:  # one workload (e.g. a smaller chunk of the 1M-context prefill for ncu)
        torch.cuda.set_device(local)
        w = Workload(args.case, torch.device("cuda", local), args.chunk)
        decode = w.c.mode == "decode"
        stage_ms, step_ms, total_ms = time_steps(w, decode, args.steps, args.warmup, None)
        res = {"case": w.c.name, "num_q": w.c.num_q, "ms_per_step": total_ms / args.steps,
               "stages_ms": stage_ms}
        if decode and args.fused:
            flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=w.di.q.device)
            res["fused_step_us"], res["fused_timing"] = fused_decode_us(
                w, max(args.steps, 1), max(args.warmup, 1), lambda: flush_buf.zero_())
        if not decode and args.train:
            res["training_kernels"] = training_kernels_case(w, max(args.steps, 1))
        if args.dense:
            d = w.di
            out = torch.empty_like(w.out)
            run = lambda: w.runner.dense(w.b, q=d.q, k_pool=d.k_pool, v_pool=d.v_pool, out=out,
                                         decode=decode)
            res["dense_ms"] = _time_ms(torch, run, max(args.steps, 1))
        print(json.dumps(res))
        return

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_index = int(vis.split(",")[local]) if vis and vis.split(",")[local].isdigit() else local
    l2_flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    l2_flush_sum = torch.empty((), dtype=torch.int64, device=dev)

    def flush():
        # write a buffer twice the L2 size, then read it back: the timed step starts with an L2
        # that holds none of its data and no dirty lines to write back
        l2_flush_buf.zero_()
        torch.sum(l2_flush_buf.view(torch.int64), dim=0, out=l2_flush_sum)

    # ---------------------------------------------------------------- prefill (headline)
    w = Workload(PREFILL, dev)
    c = w.c
    work = algorithmic(c, w.q_pos_host)
    with Clocks(gpu_index) as clk:
        stage_ms, step_ms, total_ms = time_steps(w, False, args.steps, args.warmup, dist)
    clocks = clk.summary()
    total_ms = max_over_ranks(total_ms, dist)
    ms_step = total_ms / args.steps
    value = job_throughput(world, c.num_q, args.steps, total_ms)
    launches_per_step = prefill_launches_per_step(c)
    stages = {
        "compress": dict(ms=stage_ms["compress"], bound="hbm", unit="GB/s",
                         achieved=work["compress_bytes"] / (stage_ms["compress"] * 1e-3) / 1e9,
                         peak=peaks["hbm"], kernel_file="compress.cu"),
        "score_topk": dict(ms=stage_ms["score_topk"], bound="tensor", unit="TFLOP/s",
                           achieved=work["score_flops"] / (stage_ms["score_topk"] * 1e-3) / 1e12,
                           peak=peaks["tf"], kernel_file="score_tc.cu"),
        "sparse_attn": dict(ms=stage_ms["sparse_attn"], bound="hbm", unit="GB/s",
                            achieved=work["attn_bytes"] / (stage_ms["sparse_attn"] * 1e-3) / 1e9,
                            peak=peaks["hbm"], kernel_file=("attn.cu", "attn_sw.cuh")),
    }
    for s in stages.values():
        s["frac"] = s["achieved"] / s["peak"]
    dom = max(stages, key=lambda k: stages[k]["ms"])
    ds = stages[dom]
    per_launch = {"compress": work["compress_bytes"], "score_topk": work["score_flops"],
                  "sparse_attn": work["attn_bytes"]}[dom]
    roofline = {"bound": ds["bound"], "achieved": ds["achieved"], "peak": ds["peak"], "unit": ds["unit"],
                "frac": ds["frac"], "kernel": dom, "work_per_launch": per_launch,
                "peak_source": peaks["src"] + (" burst" if ds["bound"] == "tensor" else ""),
                "traffic": traffic_for(ds["kernel_file"], f"{dom}@{PREFILL}")}
    path_roof_ms = (work["compress_bytes"] / (peaks["hbm"] * 1e9) + work["score_flops"] / (peaks["tf"] * 1e12)
                    + work["attn_bytes"] / (peaks["hbm"] * 1e9)) * 1e3
    log(f"prefill {c.name}: {ms_step:.3f} ms/step, {value / 1e6:.3f} M tok/s, stages "
        + ", ".join(f"{k} {v['ms']:.3f} ms ({100 * v['frac']:.1f}% {v['bound']})" for k, v in stages.items()))
    e2e_ms, h2d, d2h = e2e_prefill(w, max(3, args.steps), 2)
    e2e_ms = max_over_ranks(e2e_ms, dist)
    log(f"prefill e2e {e2e_ms:.3f} ms/step")
    dense_ms = dense_time_ms(w, False, 3)
    log(f"dense prefill {dense_ms:.1f} ms ({work['dense_flops'] / (dense_ms * 1e-3) / 1e12:.1f} TFLOP/s)")
    train = training_kernels(w, peaks)
    log("training kernels: " + json.dumps(train))
    del w
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- decode
    wd = Workload(DECODE, dev)
    cd = wd.c
    workd = algorithmic(cd, wd.q_pos_host)
    dsteps = max(50, 5 * args.steps)
    dstage_ms, dstep_ms, _ = time_steps(wd, True, dsteps, args.warmup, dist, flush=flush)
    log("decode eager stages " + ", ".join(f"{k} {v * 1000:.1f} us" for k, v in dstage_ms.items()))
    graph_us, _ = graph_decode_us(wd, dsteps, args.warmup, flush)
    log(f"decode graph {graph_us:.1f} us/step")
    fused_us, fused_mode = fused_decode_us(wd, dsteps, args.warmup, flush)
    log(f"decode fused step {fused_us:.1f} us/step ({fused_mode})")
    graph_us = max_over_ranks(graph_us, dist)
    d_e2e_us, dh2d, dd2h = e2e_decode(wd, dsteps, args.warmup)
    d_e2e_us = max_over_ranks(d_e2e_us, dist)
    dense_dec_ms = dense_time_ms(wd, True, 5, flush)
    log(f"decode e2e {d_e2e_us:.1f} us/step; dense decode {dense_dec_ms * 1000:.1f} us")
    dstages = {
        "score_topk": dict(ms=dstage_ms["score_topk"], bound="hbm", unit="GB/s",
                           achieved=workd["score_bytes_decode"] / (dstage_ms["score_topk"] * 1e-3) / 1e9,
                           peak=peaks["hbm"]),
        "sparse_attn": dict(ms=dstage_ms["sparse_attn"], bound="hbm", unit="GB/s",
                            achieved=workd["attn_bytes"] / (dstage_ms["sparse_attn"] * 1e-3) / 1e9,
                            peak=peaks["hbm"]),
        "compress": dict(ms=dstage_ms["compress"]),
    }
    for s in dstages.values():
        if "achieved" in s:
            s["frac"] = s["achieved"] / s["peak"]
    dpath_roof_us = (workd["score_bytes_decode"] + workd["attn_bytes"]) / (peaks["hbm"] * 1e9) * 1e6
    del wd
    torch.cuda.empty_cache()

    cpu = dcpu = None
    if rank == 0 and world == 1:
        base = oracle_prefill_baseline(rows_per_step=16, steps=4)
        cpu = {k: base[k] for k in ("value", "unit", "cores", "kind", "sample")}
        dcpu = oracle_decode_baseline()
        log(f"oracle: prefill {cpu['value']:.2f} tok/s on {cpu['cores']} threads; decode "
            f"{dcpu['value'] / 1e3:.1f} ms/step")

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded counter-based N(0,1) stand-in + 64 planted needle blocks",
            "config": {"workload": c.name, "batch": c.batch, "ctx": c.ctx, "chunk": c.n_new,
                       "q_heads": c.Hq, "kv_heads": c.Hkv, "head_dim": c.D, "idx_heads": c.Hi,
                       "idx_dim": c.Di, "topk_blocks": c.topk, "page_tokens": c.page,
                       "l2": "inputs larger than L2 (2 GiB paged KV gathered per step); decode "
                             "steps flush L2 (256 MiB write + read back) between timed steps",
                       "parallelism": f"replicas x{world}"},
            "roofline": roofline,
            "stages_ms": {k: v["ms"] for k, v in stages.items()},
            "stages": {k: {kk: vv for kk, vv in v.items() if kk != "kernel_file"} for k, v in stages.items()},
            "path_roofline_ms": path_roof_ms, "path_roofline_frac": path_roof_ms / ms_step,
            "cpu_baseline": cpu,
            "e2e": {"value": job_throughput(world, c.num_q, 1, e2e_ms), "unit": "tok/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
            "training_kernels": train,
            "dense_baseline": {"prefill_ms": dense_ms, "sparse_over_dense_speedup": dense_ms / ms_step,
                               "dense_prefill_tflops": work["dense_flops"] / (dense_ms * 1e-3) / 1e12,
                               "decode_us": dense_dec_ms * 1000,
                               "decode_speedup": dense_dec_ms * 1000 / graph_us,
                               "dense_decode_gbs": workd["dense_bytes_decode"] / (dense_dec_ms * 1e-3) / 1e9,
                               "article_ratios_context": {"prefill": 7.6, "decode": 4.9}},
            "decode": {"workload": cd.name, "us_per_step": graph_us, "cuda_graph": True,
                       "fused_step_us": fused_us, "fused_step_timing": fused_mode,
                       "us_per_step_eager": statistics.mean(dstep_ms) * 1000,
                       "stages_us": {k: v["ms"] * 1000 for k, v in dstages.items()},
                       "stages": dstages, "path_roofline_us": dpath_roof_us,
                       "path_roofline_frac": dpath_roof_us / graph_us,
                       "cpu_baseline": dcpu,
                       "e2e": {"value": d_e2e_us, "unit": "us/step", "h2d_bytes_per_step": dh2d,
                               "d2h_bytes_per_step": dd2h},
                       "gpu_launches_per_step": DECODE_LAUNCHES_PER_STEP},
        }
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
