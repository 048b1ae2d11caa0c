"""Benchmark of the DSA hot path on B200: tokens/s at 128K context.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dsa|reference]

One JSON line on rank 0.  The headline `value` is prefill tokens/s of the
128K-token causal prefill (B=1, L=131072, k=2048, indexer 64x128 FP8, 128
heads over a 576/512 MLA row, score tiles of 4096 query rows).  One step is
one pass of that prefill through the three steps (indexer -> top-k per query
block, then sparse attention).  The `decode` object reports the 128K decode
(B=8 sequences, one query each), which adds the split-k combine; its step is
a few microsecond launches, so it is captured once as a CUDA graph and timed
by replay (per-kernel times from one graph per launch group), falling back
to eager steps if the capture fails or its selection differs.

Kernel timing: each step calls the C-ABI step entry points in the order
dsa_forward uses with a full workspace, with CUDA events between launches on
the launching stream, so every kernel's share of the step is measured live;
`e2e` runs dsa_forward itself on host (pinned) buffers with the copies inside
the timed region: for a long single-sequence prefill, one call per 4096-row
query block (a chunked prefill, seqlens = the block's end) with the copies of
the next block's queries and of the finished blocks' outputs overlapping the
compute on two copy streams; otherwise one call between the copies.  `alternatives.select_fused` times dsa_select over the same
query blocks on its own (the fused indexer + top-k that dsa_forward takes when
its workspace has no room for the score tile); it is not part of the step.
`extras` (one GPU only; --no-extras skips it) times the path's other forms
the same way: the decode over page pools against the contiguous one, the
dense attention beside the sparse one on the 8K prefill plus a short prefill
that dsa_forward runs wholly in the dense form, and one indexer training step
(scores, KL target, KL loss, backward) in its sparse and warm-up stages.

Inputs are synthetic (long_context_05_b200.inputs), larger than L2 for the
prefill; L2 is flushed between timed steps anyway (a 256 MiB write outside
the timed events).  Multi-GPU: one process per GPU, each rank runs its own
independent sequence(s) (weak scaling, no collective on the data path); the
step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_05_b200.inputs import WORKLOADS, make_inputs, to_paged  # noqa: E402
from long_context_05_b200.parallel import barrier as _barrier, max_over_ranks as _max_over_ranks  # noqa: E402
from long_context_05_b200.parallel import rank_seed  # noqa: E402

METRIC = "DSA tokens/s (prefill, decode) at 128K ctx; % of HBM / tensor-core roofline"
PREFILL = "prefill_128k"
DECODE = "decode_128k_b8"

# DRAM bytes (read + write) of one sparse-attention launch on prefill_128k,
# scaled from an ncu capture of the same kernel on prefill_chunk_128k (the
# command is kept with the capture summaries under profiles/).  It holds only
# for the kernel source it was taken from, so the bench reports it only while
# that source's hash matches.
ATTN_TRAFFIC = {"workload": "prefill_128k", "kernel": "sparse_attn",
                # DRAM read + write of one prefill_chunk_128k launch (92.39 MB +
                # 30.67 MB, ncu) times 256, the ratio of query rows
                "bytes": 92.39e6 * 256 + 30.67e6 * 256,
                "source": "long_context_05_b200/csrc/sparse_attn.cu",
                "sha256": "7606374af7813d86460dc014ed6b075e2dd843c8d1b6348b974638678cc1c406"}


def measured_traffic(workload: str, kernel: str):
    """Captured DRAM bytes per launch for (workload, kernel), or None if the
    kernel source changed since the capture (or none was taken)."""
    import hashlib
    t = ATTN_TRAFFIC
    if workload != t["workload"] or kernel != t["kernel"]:
        return None
    try:
        with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), t["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != t["sha256"]:
                return None
    except OSError:
        return None
    return t["bytes"]
FP8_PER_BF16 = 2.0  # nominal dense fp8 : bf16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_setup(n_gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        _barrier(torch.device("cuda", torch.cuda.current_device()))


def max_over_ranks(x, ws):
    return _max_over_ranks(x, device="cuda") if ws > 1 else x


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


class Flusher:
    """Writes a buffer larger than the 126 MB L2 between timed steps."""

    def __init__(self):
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def __call__(self):
        self.buf.fill_(1)


# ------------------------------------------------------------------ work model

def causal_pairs(wl):
    """(indexer pairs, attention pairs) of one batch: sum over queries of
    pos + 1 and min(pos + 1, k)."""
    ip = ap = 0
    for t in range(wl.T):
        v = wl.S - wl.T + t + 1
        ip += v
        ap += min(v, wl.k)
    return ip * wl.B, ap * wl.B


def dense_rows(wl):
    """Query rows whose visible keys all fit in k: the path keeps every one of
    them, so it scores and selects nothing for them (dsa_forward's rule)."""
    return max(0, min(wl.T, wl.k - (wl.S - wl.T)))


def scored_pairs(wl):
    """Indexer pairs the path scores: causal pairs of the rows past dense_rows."""
    d = dense_rows(wl)
    return wl.B * sum(wl.S - wl.T + t + 1 for t in range(d, wl.T))


# ------------------------------------------------------------------ GPU arm

class DsaRunner:
    """Runs one workload through the C ABI, step by step, with events."""

    def __init__(self, wl, seed_offset=0, page_size=0):
        from long_context_05_b200 import dsa
        self.dsa = dsa
        self.wl = wl = wl.with_(seed=rank_seed(wl.seed, seed_offset))
        self.inp = make_inputs(wl, "cuda")
        self.inp.pop("needle_pos", None)
        if page_size:
            # key-side caches in page pools, pages in a random order
            self.inp, self.table, num_pages = to_paged(self.inp, wl, page_size, wl.seed)
            self.shape = dsa.make_shape(wl, block_table=self.table, page_size=page_size, num_pages=num_pages)
        else:
            self.shape = dsa.make_shape(wl)
        self.ws = dsa.alloc_workspace(self.shape)
        self.outs = dsa.alloc_outputs(wl)
        self.ld = (wl.S + 63) // 64 * 64
        # each query block scores its rows into the workspace's score tile;
        # the top-k's scratch (histograms of the split path for few long rows,
        # as in decode) follows it, 256-byte aligned, as in dsa_forward
        nscore = wl.B * self.rows_per_block() * self.ld * 4
        self.scores = self.ws[:nscore].view(torch.float32).view(-1, self.ld)
        self.topk_ws = self.ws[(nscore + 255) // 256 * 256:] if wl.decode else None
        # the fused selection (dsa_select) where it applies: its own, smaller
        # workspace; timed beside the step as the alternative to indexer + topk
        self.ws_fused = None
        if not wl.decode and dsa.select_workspace_size(self.shape) < dsa.workspace_size(self.shape):
            self.ws_fused = dsa.alloc_workspace(self.shape, fused=True)
        self.stream = torch.cuda.current_stream()

    def rows_per_block(self):
        wl = self.wl
        return wl.T if wl.decode else min(wl.q_block, wl.T)

    def step(self, ev=None):
        """One pass of the path via the step entry points; if ev is a list,
        append (name, start_event, end_event) per launch group."""
        d, wl, i, o = self.dsa, self.wl, self.inp, self.outs
        qb = self.rows_per_block()

        def mark():
            if ev is None:
                return None
            e = torch.cuda.Event(enable_timing=True)
            e.record(self.stream)
            return e

        dr = dense_rows(wl)
        if dr:
            # rows that keep all their visible keys: the index fill only
            e0 = mark()
            d.topk(self.shape, self.scores, 0, dr, o.idx, self.topk_ws)
            e1 = mark()
            if ev is not None:
                ev.append(("topk", e0, e1))
        for q0 in range(dr, wl.T, qb):
            cnt = min(qb, wl.T - q0)
            e0 = mark()
            d.indexer_scores(self.shape, i["q_I"], i["q_scale"], i["w"], i["k_I"], i["k_scale"], q0, cnt, self.scores)
            e1 = mark()
            d.topk(self.shape, self.scores, q0, cnt, o.idx, self.topk_ws)
            e2 = mark()
            if ev is not None:
                ev.append(("indexer", e0, e1))
                ev.append(("topk", e1, e2))
        e3 = mark()
        d.sparse_attn(self.shape, i["q"], i["kv"], o.idx, o.out, o.lse, self.ws)
        e4 = mark()
        if ev is not None:
            ev.append(("sparse_attn", e3, e4))

    def step_part(self, name):
        """One of the step's launch groups alone (indexer, topk or sparse_attn),
        or "select": steps A and B of every block through the fused selection."""
        d, wl, i, o = self.dsa, self.wl, self.inp, self.outs
        qb = self.rows_per_block()
        if name == "sparse_attn":
            d.sparse_attn(self.shape, i["q"], i["kv"], o.idx, o.out, o.lse, self.ws)
            return
        dr = dense_rows(wl)
        if dr and name in ("topk", "select"):
            d.topk(self.shape, self.scores, 0, dr, o.idx, self.topk_ws)
        for q0 in range(dr, wl.T, qb):
            cnt = min(qb, wl.T - q0)
            if name == "select":
                d.select(self.shape, i["q_I"], i["q_scale"], i["w"], i["k_I"], i["k_scale"], q0, cnt, o.idx,
                         self.ws_fused)
            elif name == "indexer":
                d.indexer_scores(self.shape, i["q_I"], i["q_scale"], i["w"], i["k_I"], i["k_scale"], q0, cnt,
                                 self.scores)
            else:
                d.topk(self.shape, self.scores, q0, cnt, o.idx, self.topk_ws)

    def forward(self):
        self.dsa.forward(self.shape, self.inp, self.outs.out, self.outs.lse, self.outs.idx, self.ws)


def time_steps(runner, steps, warmup, ws):
    flush = Flusher()
    for _ in range(warmup):
        runner.step()
    torch.cuda.synchronize()
    st, det = runner.dsa.device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} detail {det:#x}")
    per_kernel = {}
    total_ms = 0.0
    launches0 = runner.dsa.launch_count()
    barrier(ws)
    torch.cuda.synchronize()
    for _ in range(steps):
        flush()
        ev = []
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record()
        runner.step(ev)
        s1.record()
        s1.synchronize()
        total_ms += s0.elapsed_time(s1)
        for name, a, b in ev:
            per_kernel.setdefault(name, []).append(a.elapsed_time(b))
    torch.cuda.synchronize()
    barrier(ws)
    launches = runner.dsa.launch_count() - launches0
    st, det = runner.dsa.device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} detail {det:#x}")
    return total_ms, per_kernel, launches


def time_part(runner, name, steps, warmup, ws):
    """Device time per step of one launch group run alone (flushed L2, same
    barriers as time_steps), in ms, max over ranks."""
    flush = Flusher()
    for _ in range(warmup):
        runner.step_part(name)
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        runner.step_part(name)
        b.record()
        b.synchronize()
        total += a.elapsed_time(b)
    torch.cuda.synchronize()
    barrier(ws)
    st, det = runner.dsa.device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} detail {det:#x}")
    return max_over_ranks(total / steps, ws)


def capture_step_graphs(runner, warmup):
    """Decode steps are a few microsecond launches, so the bench times them by
    CUDA-graph replay: the step is captured once, and each launch group once
    more on its own for the per-kernel split.  No collective here.  Returns
    ({"step", "indexer", "topk", "sparse_attn"} graphs, launches per step), or
    None when capture or replay fails or the replayed selection differs from
    the eager one (compared as sets per row)."""
    d = runner.dsa
    graphs = {}
    try:
        for _ in range(warmup):
            runner.step()
        torch.cuda.synchronize()
        if d.device_error()[0] != 0:
            return None
        ref = torch.sort(runner.outs.idx, dim=-1).values
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            runner.step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        n0 = d.launch_count()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            runner.step()
        launches = d.launch_count() - n0
        graphs["step"] = g
        for name in ("indexer", "topk", "sparse_attn"):
            gp = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gp, capture_error_mode="relaxed"):
                runner.step_part(name)
            graphs[name] = gp
        runner.outs.idx.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        if launches <= 0 or d.device_error()[0] != 0:
            return None
        if not torch.equal(torch.sort(runner.outs.idx, dim=-1).values, ref):
            return None
        return graphs, launches
    except Exception:
        return None


def time_graphs(graphs, steps, warmup, ws):
    """Replay timing of captured step graphs; same barriers and flushes as
    time_steps.  Returns (total_ms, per_kernel)."""
    flush = Flusher()
    for _ in range(warmup):
        graphs["step"].replay()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()

    def timed(g):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        return a.elapsed_time(b)

    total_ms = sum(timed(graphs["step"]) for _ in range(steps))
    per_kernel = {name: [timed(graphs[name]) for _ in range(steps)] for name in ("indexer", "topk", "sparse_attn")}
    torch.cuda.synchronize()
    barrier(ws)
    return total_ms, per_kernel


def kernel_report(wl, per_kernel, steps, peaks, peak_src, sustained):
    _, ap = causal_pairs(wl)
    ip = scored_pairs(wl)
    bf16 = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    kind = "sustained" if sustained else "burst"
    work = {
        # name: (algorithmic amount per step, unit, bound, peak, peak note)
        # decode: one query per sequence, so the indexer streams every key
        # once (D_I FP8 bytes + a 4-byte scale) and is bound by HBM
        "indexer": ((2.0 * wl.H_I * wl.D_I * ip / 1e12, "TFLOP/s", "tensor", bf16 * FP8_PER_BF16,
                     f"fp8 = {kind} bf16 x {FP8_PER_BF16:g} ({peak_src})") if not wl.decode else
                    (wl.B * wl.S * (wl.D_I + 4) / 1e9, "GB/s", "hbm", peaks["hbm_gbs"],
                     f"hbm, k_I + k_scale bytes ({peak_src})")),
        "topk": (4.0 * ip / 1e9, "GB/s", "hbm", peaks["hbm_gbs"], f"hbm ({peak_src})"),
        # prefill: the indexer and the selection fused (dsa_select); its work
        # is the indexer's, so the fraction is a lower bound on the indexer's
        "select": (2.0 * wl.H_I * wl.D_I * ip / 1e12, "TFLOP/s", "tensor", bf16 * FP8_PER_BF16,
                   f"indexer FLOP over the fused indexer + top-k time; fp8 = {kind} bf16 x {FP8_PER_BF16:g} "
                   f"({peak_src})"),
        "sparse_attn": ((2.0 * wl.H * (wl.d_k + wl.d_v) * ap / 1e12, "TFLOP/s", "tensor", bf16,
                         f"bf16 {kind} ({peak_src})") if not wl.decode else
                        (2.0 * wl.d_k * ap / 1e9, "GB/s", "hbm", peaks["hbm_gbs"], f"hbm, gathered KV bytes ({peak_src})")),
    }
    out = {}
    tot = sum(sum(v) for v in per_kernel.values())
    for name, times in per_kernel.items():
        ms = sum(times) / steps                       # per step
        launches = len(times) / steps
        amount, unit, bound, peak, note = work[name]
        achieved = amount / (ms / 1e3)
        out[name] = {"ms_per_step": ms, "launches_per_step": launches, "share": sum(times) / tot,
                     "bound": bound, "achieved": achieved, "unit": unit, "peak": peak,
                     "frac": achieved / peak, "peak_note": note,
                     "work_per_step": amount * (1e12 if unit == "TFLOP/s" else 1e9)}
    return out


def cpu_oracle_sample(wl, inp, budget_s=12.0, max_rows=4096):
    """The FP64 oracle as it stands, on evenly spread query rows of the same
    workload (one full path per row), until the time budget is used."""
    import numpy as np
    from oracle import dsa_oracle as O

    def u16(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    b = 0
    kd = O.e4m3_decode(inp["k_I"][b].cpu().numpy()) * inp["k_scale"][b].cpu().double().numpy()[:, None]
    kv = O.bf16_decode(u16(inp["kv"][b]))
    tau = O.default_tau(wl.d_k)
    n_target = max_rows
    rows = [int(wl.T * (i + 0.5) / n_target) for i in range(n_target)]
    rng = np.random.default_rng(0)
    rng.shuffle(rows)
    done = 0
    t0 = time.perf_counter()
    for t in rows:
        qd = O.e4m3_decode(inp["q_I"][b, t].cpu().numpy()) * inp["q_scale"][b, t].cpu().double().numpy()[:, None]
        w = inp["w"][b, t].cpu().double().numpy()
        q = O.bf16_decode(u16(inp["q"][b, t]))
        O.dsa_row(qd, w, kd, q, kv, O.query_pos(wl.T, wl.S, t), wl.k, wl.d_v, tau)
        done += 1
        if time.perf_counter() - t0 > budget_s and done >= 4:
            break
    el = time.perf_counter() - t0
    try:
        import threadpoolctl
        cores = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()) or 1
    except Exception:
        cores = os.cpu_count()
    return {"value": done / el * wl.B, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} query rows of {wl.name} spread evenly over positions 0..{wl.T - 1}, "
                      f"full path per row (indexer over pos+1 keys, top-k, attention), {el:.1f} s"}


def run_e2e(runner, steps, ws):
    """dsa_forward on pinned host buffers: H2D of the inputs, the call, D2H of
    out and lse, all inside the timed region."""
    wl = runner.wl
    host_in = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in runner.inp.items()}
    for k, v in runner.inp.items():
        host_in[k].copy_(v)
    host_out = torch.empty(runner.outs.out.shape, dtype=torch.bfloat16, pin_memory=True)
    host_lse = torch.empty(runner.outs.lse.shape, dtype=torch.float32, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = host_out.numel() * 2 + host_lse.numel() * 4

    def one():
        for k, v in host_in.items():
            runner.inp[k].copy_(v, non_blocking=True)
        runner.forward()
        host_out.copy_(runner.outs.out, non_blocking=True)
        host_lse.copy_(runner.outs.lse, non_blocking=True)

    one()
    torch.cuda.synchronize()
    barrier(ws)
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(steps):
        one()
    s1.record()
    s1.synchronize()
    ms = max_over_ranks(s0.elapsed_time(s1) / steps, ws)
    del host_in
    return ms, h2d, d2h


def run_e2e_pipelined(runner, steps, ws):
    """dsa_forward on pinned host buffers, one call per query block of
    q_block rows (a chunked prefill: seqlens = the block's end, the whole key
    cache as S), with the host->device copies of the next block's queries and
    the device->host copies of the finished blocks' outputs on two copy
    streams overlapping the compute.  Every step still copies all inputs in
    and out + lse back; the per-block calls run the same kernels over the
    same keys as one call over all rows (the first block's rows that keep
    every key go through the top-k's fill instead of the dense shortcut)."""
    d, wl = runner.dsa, runner.wl
    qb = wl.q_block
    blocks = [(s0, min(qb, wl.T - s0)) for s0 in range(0, wl.T, qb)]
    key_names = ("k_I", "k_scale", "kv")
    q_names = ("q_I", "q_scale", "w", "q")
    host_in = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in runner.inp.items()}
    for k, v in runner.inp.items():
        host_in[k].copy_(v)
    o = runner.outs
    host_out = torch.empty(o.out.shape, dtype=torch.bfloat16, pin_memory=True)
    host_lse = torch.empty(o.lse.shape, dtype=torch.float32, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = host_out.numel() * 2 + host_lse.numel() * 4
    ends = [torch.tensor([s0 + c], dtype=torch.int32, device="cuda") for s0, c in blocks]
    shapes = [d.make_shape(wl.with_(T=c, q_block=c), mode=d.DSA_PREFILL, seqlens=e)
              for (s0, c), e in zip(blocks, ends)]
    ws_blk = d.alloc_workspace(shapes[0])
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def one():
        main = torch.cuda.current_stream()
        for st in (s_in, s_cmp, s_out):
            st.wait_stream(main)
        ev_in = []
        with torch.cuda.stream(s_in):
            for n in key_names:
                runner.inp[n].copy_(host_in[n], non_blocking=True)
            for s0, c in blocks:
                for n in q_names:
                    runner.inp[n][:, s0:s0 + c].copy_(host_in[n][:, s0:s0 + c], non_blocking=True)
                ev_in.append(torch.cuda.Event())
                ev_in[-1].record(s_in)
        ev_done = []
        with torch.cuda.stream(s_cmp):
            for (s0, c), shape, ev in zip(blocks, shapes, ev_in):
                s_cmp.wait_event(ev)
                part = {n: runner.inp[n][:, s0:s0 + c] for n in q_names}
                part.update({n: runner.inp[n] for n in key_names})
                d.forward(shape, part, o.out[:, s0:s0 + c], o.lse[:, s0:s0 + c], o.idx[:, s0:s0 + c], ws_blk)
                ev_done.append(torch.cuda.Event())
                ev_done[-1].record(s_cmp)
        with torch.cuda.stream(s_out):
            for (s0, c), ev in zip(blocks, ev_done):
                s_out.wait_event(ev)
                host_out[:, s0:s0 + c].copy_(o.out[:, s0:s0 + c], non_blocking=True)
                host_lse[:, s0:s0 + c].copy_(o.lse[:, s0:s0 + c], non_blocking=True)
        main.wait_stream(s_out)

    one()
    torch.cuda.synchronize()
    st, det = d.device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} detail {det:#x}")
    barrier(ws)
    s0e = torch.cuda.Event(enable_timing=True)
    s1e = torch.cuda.Event(enable_timing=True)
    s0e.record()
    for _ in range(steps):
        one()
    s1e.record()
    s1e.synchronize()
    ms = max_over_ranks(s0e.elapsed_time(s1e) / steps, ws)
    del host_in
    return ms, h2d, d2h, len(blocks)


# ------------------------------------------------------------------ other forms of the path

class CallRunner:
    """A list of named launch groups run as one step (the time_steps protocol:
    .dsa, .step(ev))."""

    def __init__(self, dsa, groups):
        self.dsa = dsa
        self.groups = groups

    def step(self, ev=None):
        for name, fn in self.groups:
            if ev is None:
                fn()
                continue
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            ev.append((name, a, b))


def part_report(ms, amount, unit, bound, peak, note):
    achieved = amount / (ms / 1e3)
    return {"ms_per_step": ms, "bound": bound, "achieved": achieved, "unit": unit, "peak": peak,
            "frac": achieved / peak, "peak_note": note,
            "work_per_step": amount * (1e12 if unit == "TFLOP/s" else 1e9)}


def timed_groups(runner, steps, warmup, ws):
    total, per, launches = time_steps(runner, steps, warmup, ws)
    return (max_over_ranks(total / steps, ws), {n: sum(v) / steps for n, v in per.items()}, launches // steps)


def extra_paged_decode(wl, steps, warmup, ws, peaks, peak_src, contiguous_ms, page_size=64):
    """Decode over page pools (random page order) against the contiguous
    caches: the same work, so the ratio is the paging cost."""
    run = DsaRunner(wl, page_size=page_size)
    got = capture_step_graphs(run, warmup)
    if got is not None:
        total, kern = time_graphs(got[0], steps, warmup, ws)
        launches, timing = got[1], "cuda_graph_replay"
        got[0].clear()
        torch.cuda.synchronize()
    else:
        total, kern, launches = time_steps(run, steps, warmup, ws)
        launches //= steps
        timing = "eager"
    ms = max_over_ranks(total / steps, ws)
    rep = kernel_report(run.wl, kern, steps, peaks, peak_src, sustained=False)
    for r in rep.values():
        r.pop("share", None)
    del run
    return {"workload": f"{wl.name} paged", "page_size": page_size, "value": ws * wl.B * wl.T / (ms / 1e3),
            "unit": "tokens/s", "ms_per_step": ms, "timing": timing, "gpu_launches": launches,
            "vs_contiguous": ms / contiguous_ms if contiguous_ms else None, "kernels": rep}


def extra_dense(wl, steps, warmup, ws, peaks, peak_src):
    """dsa_dense_attn (every visible key) beside the sparse attention over the
    selected keys, on the same queries and cache; and dsa_forward on a prefill
    short enough that every row keeps all its visible keys (the whole call is
    the dense form)."""
    from long_context_05_b200 import dsa
    bf16 = peaks["bf16_tflops_sustained"]
    run = DsaRunner(wl)
    run.step()
    i, o = run.inp, run.outs
    dout = torch.empty_like(o.out)
    dlse = torch.empty_like(o.lse)
    cr = CallRunner(dsa, [("sparse_attn", lambda: dsa.sparse_attn(run.shape, i["q"], i["kv"], o.idx, o.out, o.lse,
                                                                  run.ws)),
                          ("dense_attn", lambda: dsa.dense_attn(run.shape, i["q"], i["kv"], dout, dlse, run.ws))])
    ms, per, launches = timed_groups(cr, steps, warmup, ws)
    ip, ap = causal_pairs(wl)
    fl = 2.0 * wl.H * (wl.d_k + wl.d_v)
    note = f"bf16 sustained ({peak_src})"
    res = {"workload": wl.name, "gpu_launches": launches,
           "sparse_attn": part_report(per["sparse_attn"], fl * ap / 1e12, "TFLOP/s", "tensor", bf16, note),
           "dense_attn": part_report(per["dense_attn"], fl * ip / 1e12, "TFLOP/s", "tensor", bf16, note)}
    res["dense_vs_sparse_ms"] = per["dense_attn"] / per["sparse_attn"]
    del run, cr
    # a short prefill: k covers every row, so dsa_forward runs the dense form
    swl = wl.with_(name=f"prefill_{wl.k // 1024}k_b4", B=4, T=wl.k, S=wl.k, q_block=wl.k)
    srun = DsaRunner(swl)
    cr = CallRunner(dsa, [("forward", srun.forward)])
    ms, per, launches = timed_groups(cr, steps, warmup, ws)
    ip, _ = causal_pairs(swl)
    res["short_prefill"] = {"workload": swl.name, "config": {"batch": swl.B, "seq_len": swl.T, "k": swl.k},
                            "value": ws * swl.B * swl.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
                            "gpu_launches": launches,
                            "roofline": part_report(ms, fl * ip / 1e12, "TFLOP/s", "tensor", bf16, note)}
    del srun, cr
    return res


def extra_train(wl, steps, warmup, ws, peaks, peak_src):
    """One indexer training step over all query rows, per query block: the
    indexer's scores, the KL target from the main attention, the KL loss and
    dL/dI, and the backward to q_I, w and k_I.  Sparse stage (the selected
    set, lse from the sparse attention) and warm-up (every visible key, lse
    from the dense attention)."""
    from long_context_05_b200 import dsa
    run = DsaRunner(wl)
    run.step()
    i, o = run.inp, run.outs
    qb = min(wl.q_block, wl.T)
    rows = wl.B * qb
    ld = run.ld
    target = torch.zeros(rows, ld, device="cuda")
    grad = torch.zeros(rows, ld, device="cuda")
    loss = torch.zeros(rows, device="cuda")
    dq = torch.zeros(wl.B, wl.T, wl.H_I, wl.D_I, device="cuda")
    dw = torch.zeros(wl.B, wl.T, wl.H_I, device="cuda")
    dk = torch.zeros(wl.B, wl.S, wl.D_I, device="cuda")
    dout = torch.empty_like(o.out)
    dlse = torch.empty_like(o.lse)
    dsa.dense_attn(run.shape, i["q"], i["kv"], dout, dlse, run.ws)
    sh = run.shape

    def groups(idx, lse):
        g = [("dk_zero", dk.zero_)]
        for q0 in range(0, wl.T, qb):
            cnt = min(qb, wl.T - q0)
            g += [("indexer", lambda q0=q0, cnt=cnt: dsa.indexer_scores(
                      sh, i["q_I"], i["q_scale"], i["w"], i["k_I"], i["k_scale"], q0, cnt, run.scores)),
                  ("kl_target", lambda q0=q0, cnt=cnt: dsa.kl_target(sh, i["q"], i["kv"], lse, q0, cnt, target, idx)),
                  ("indexer_kl", lambda q0=q0, cnt=cnt: dsa.indexer_kl(sh, run.scores, target, q0, cnt, grad, loss,
                                                                       idx)),
                  ("indexer_backward", lambda q0=q0, cnt=cnt: dsa.indexer_backward(
                      sh, i["q_I"], i["q_scale"], i["w"], i["k_I"], i["k_scale"], grad, q0, cnt, dq, dw, dk, idx))]
        return g

    ip, ap = causal_pairs(wl)
    bf16 = peaks["bf16_tflops_sustained"]
    res = {}
    for stage, idx, lse, pairs in (("sparse", o.idx, o.lse, ap), ("warmup_dense", None, dlse, ip)):
        cr = CallRunner(dsa, groups(idx, lse))
        ms, per, launches = timed_groups(cr, steps, warmup, ws)
        # per row: the set's scores and targets read, grad written over the visible keys
        kl_bytes = (8.0 * pairs + 4.0 * ip) if idx is not None else 12.0 * ip
        parts = {
            "indexer": part_report(per["indexer"], 2.0 * wl.H_I * wl.D_I * ip / 1e12, "TFLOP/s", "tensor",
                                   bf16 * FP8_PER_BF16, f"fp8 = sustained bf16 x {FP8_PER_BF16:g} ({peak_src})"),
            "kl_target": part_report(per["kl_target"], 2.0 * wl.H * wl.d_k * pairs / 1e12, "TFLOP/s", "tensor",
                                     bf16, f"bf16 sustained ({peak_src}); Q K^T of the set"),
            "indexer_kl": part_report(per["indexer_kl"], kl_bytes / 1e9, "GB/s", "hbm", peaks["hbm_gbs"],
                                      f"hbm ({peak_src}); scores + target of the set read, grad row written"),
            # tensor cores (D in FP8, dk and R in BF16 hi + lo); algorithmic
            # FLOP: D, dq and dk per pair.  Its dk additions into global
            # memory (512 B per pair) are reported beside it
            "indexer_backward": part_report(per["indexer_backward"], 6.0 * wl.H_I * wl.D_I * pairs / 1e12,
                                            "TFLOP/s", "tensor", bf16,
                                            f"bf16 sustained ({peak_src}); D, dq and dk per pair"),
        }
        parts["indexer_backward"]["dk_reduce_gbs"] = 4.0 * wl.D_I * pairs / (per["indexer_backward"] / 1e3) / 1e9
        res[stage] = {"ms_per_step": ms, "rows_per_s": ws * wl.B * wl.T / (ms / 1e3), "gpu_launches": launches,
                      "kernels": parts}
    st, det = dsa.device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} detail {det:#x}")
    del run
    res["workload"] = wl.name
    return res


def run_extras(args, ws, peaks, peak_src, contiguous_decode_ms):
    """The forms of the path beside the headline step, each timed on its own
    with the same warm-up, flushes and events: paged decode, the dense form,
    and the indexer's training step."""
    steps, warmup = max(2, args.steps), args.warmup
    out = {}
    if args.decode_workload != "none":
        out["paged_decode"] = extra_paged_decode(WORKLOADS[args.decode_workload], steps, warmup, ws, peaks, peak_src,
                                                 contiguous_decode_ms)
        torch.cuda.empty_cache()
    out["dense"] = extra_dense(WORKLOADS["prefill_8k"], steps, warmup, ws, peaks, peak_src)
    torch.cuda.empty_cache()
    out["train"] = extra_train(WORKLOADS["prefill_8k"], steps, warmup, ws, peaks, peak_src)
    torch.cuda.empty_cache()
    return out


def gpu_arm(args):
    ws, rank, local = dist_setup(args.gpus)
    from long_context_05_b200 import dsa
    dsa.lib()
    peaks, peak_src = load_peaks()
    wl = WORKLOADS[args.workload]
    wl_dec = WORKLOADS[args.decode_workload] if args.decode_workload != "none" else None

    clocks = ClockSampler(local)

    runner = DsaRunner(wl, seed_offset=rank)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(runner.wl, runner.inp, budget_s=args.cpu_seconds)

    clocks.start()
    total_ms, per_kernel, launches = time_steps(runner, args.steps, args.warmup, ws)
    ms_step = max_over_ranks(total_ms / args.steps, ws)
    # the fused selection, timed alone over the same blocks (every rank takes
    # the same branch: the workload is the same on all)
    fused_ms = None
    if runner.ws_fused is not None:
        fused_ms = time_part(runner, "select", args.steps, min(args.warmup, 1), ws)
    dec = None
    if wl_dec is not None:
        drun = DsaRunner(wl_dec, seed_offset=rank)
        got = capture_step_graphs(drun, args.warmup)
        # every rank takes the same path: graphs only if all ranks captured
        use_graph = max_over_ranks(0.0 if got is not None else 1.0, ws) == 0.0
        if use_graph:
            timing = "cuda_graph_replay"
            d_total, d_kern = time_graphs(got[0], args.steps, args.warmup, ws)
            d_launch = got[1]
        else:
            timing = "eager"
            d_total, d_kern, d_launch = time_steps(drun, args.steps, args.warmup, ws)
            d_launch //= args.steps
        if got is not None:
            got[0].clear()
            torch.cuda.synchronize()
        d_ms = max_over_ranks(d_total / args.steps, ws)
        d_rep = kernel_report(drun.wl, d_kern, args.steps, peaks, peak_src, sustained=False)
        d_top = max(d_rep.items(), key=lambda kv: kv[1]["ms_per_step"])
        dec = {"workload": wl_dec.name, "value": ws * wl_dec.B * wl_dec.T / (d_ms / 1e3), "unit": "tokens/s",
               "ms_per_step": d_ms, "gpu_launches": d_launch, "timing": timing,
               "config": {"batch": wl_dec.B, "context": wl_dec.S, "k": wl_dec.k, "H": wl_dec.H,
                          "H_I": wl_dec.H_I, "D_I": wl_dec.D_I, "d_k": wl_dec.d_k, "d_v": wl_dec.d_v},
               "roofline": {"kernel": d_top[0], "bound": d_top[1]["bound"], "achieved": d_top[1]["achieved"],
                            "peak": d_top[1]["peak"], "unit": d_top[1]["unit"], "frac": d_top[1]["frac"],
                            "traffic": None},
               "kernels": d_rep}
        del drun
    clk = clocks.stop()

    e2e = None
    need = sum(v.numel() * v.element_size() for v in runner.inp.values()) + runner.outs.out.numel() * 2
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = None
    if not args.no_e2e and avail is not None and avail < 2 * need * max(1, ws):
        e2e = {"skipped": f"host RAM available {avail / 2**30:.0f} GiB < 2 x {need / 2**30:.0f} GiB pinned per rank"}
    elif not args.no_e2e:
        if not wl.decode and wl.B == 1 and wl.T > wl.q_block:
            # a long prefill: per-block calls with the copies overlapping
            e_ms, h2d, d2h, nblk = run_e2e_pipelined(runner, args.e2e_steps, ws)
            how = f"dsa_forward per {wl.q_block}-row query block ({nblk} calls), copies on two streams overlapping"
        else:
            e_ms, h2d, d2h = run_e2e(runner, args.e2e_steps, ws)
            how = "one dsa_forward call between the copies"
        e2e = {"value": ws * wl.B * wl.T / (e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps, "how": how}

    rep = kernel_report(runner.wl, per_kernel, args.steps, peaks, peak_src, sustained=True)
    top = max(rep.items(), key=lambda kv: kv[1]["ms_per_step"])
    alternatives = None
    if fused_ms is not None:
        f = kernel_report(runner.wl, {"select": [fused_ms] * args.steps}, args.steps, peaks, peak_src,
                          sustained=True)["select"]
        f.pop("share", None)
        sel_ms = sum(rep[n]["ms_per_step"] for n in ("indexer", "topk") if n in rep)
        f["vs_indexer_topk"] = fused_ms / sel_ms if sel_ms > 0 else None
        f["workspace_bytes"] = int(runner.ws_fused.numel())
        f["score_tile_workspace_bytes"] = int(runner.ws.numel())
        alternatives = {"select_fused": f}
    # the other forms of the path, on one GPU only (each rank decides alike)
    extras = None
    if ws == 1 and not args.no_extras:
        del runner
        torch.cuda.empty_cache()
        xclk = ClockSampler(local)
        xclk.start()
        extras = run_extras(args, ws, peaks, peak_src, dec["ms_per_step"] if dec else None)
        extras["clocks"] = xclk.stop()
    tokens = ws * wl.B * wl.T
    line = {
        "metric": METRIC,
        "value": tokens / (ms_step / 1e3),
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8 indexer (f32 accumulate) / bf16 attention (f32 accumulate)",
        "data": "synthetic (seeded; needles + local-window bias), inputs larger than L2, L2 flushed between steps",
        "config": {"workload": wl.name, "batch": wl.B, "seq_len": wl.T, "context": wl.S, "k": wl.k,
                   "q_block": wl.q_block, "H_I": wl.H_I, "D_I": wl.D_I, "H": wl.H, "d_k": wl.d_k,
                   "d_v": wl.d_v, "parallelism": f"independent sequences x{ws}", "l2": "flushed between steps"},
        "gpu_launches": launches // args.steps,
        "roofline": {"kernel": top[0], "bound": top[1]["bound"], "achieved": top[1]["achieved"],
                     "peak": top[1]["peak"], "unit": top[1]["unit"], "frac": top[1]["frac"],
                     "traffic": measured_traffic(wl.name, top[0]),
                     "peak_note": top[1]["peak_note"]},
        "kernels": rep,
        "alternatives": alternatives,
        "decode": dec,
        "extras": extras,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clk,
        "peaks_source": peak_src,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def reference_arm(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(wl.with_(T=wl.T, S=wl.S), dev) if dev == "cuda" else None
    if inp is None:
        # generate on the host when there is no GPU; same shapes, CPU stream
        inp = make_inputs(wl, "cpu")
    vals = []
    cpu = None
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(wl, inp, budget_s=args.cpu_seconds / max(1, args.steps), max_rows=16)
        if i >= args.warmup:
            vals.append(r["value"])
            cpu = r
    v = statistics.mean(vals)
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * wl.B * wl.T / v, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.B, "seq_len": wl.T, "context": wl.S, "k": wl.k},
            "impl": "reference",
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cpu["cores"], "kind": "oracle",
                             "sample": cpu["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="dsa", choices=["dsa", "reference"])
    ap.add_argument("--workload", default=PREFILL, choices=sorted(WORKLOADS))
    ap.add_argument("--decode-workload", default=DECODE, choices=sorted(WORKLOADS) + ["none"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "dsa":
        print("note: warm-up raised to the minimum of 3 steps", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
