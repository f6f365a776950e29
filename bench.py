#!/usr/bin/env python
"""Benchmark of the SAS gated block-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config all|c1|c2|c3|c4|c5]
                    [--impl ours|reference]

Prints ONE JSON line (rank 0). The default (--config all) measures every
workload the metric is quoted on, each with the same K timed steps:
  c5  long-context decode (512K, batch 1, top-k 63): the headline record;
  c4  batched decode (batch 8, ragged 96K-128K, top-k 31);
  c2  decode (64K, batch 1, top-k 15), also through a paged cache;
  c5 with bf16 block summaries (the cheaper long-context selection);
  c3  prefill training step (N = 16384, GQA 32/8, top-k 31): summaries,
      selection, gated sparse forward and backward, selector backward.
The line's top level is the c5 record; "records" holds one full record per
workload (roofline, cpu_baseline, e2e, clocks, launches).

A decode step is block selection over the summaries (scores, gate, Top-K)
and split-K attention over the kept blocks plus the current block, for every
sequence and kv group; the summaries are cache state, built when blocks
complete, outside the step. Metric: GB/s of algorithmic bytes (summaries
scanned + kept K/V read + q/o). A prefill step's metric is TFLOP/s of
algorithmic FLOPs (kept block pairs, causal pairs exact on the diagonal
block, forward 4d and backward 10d per pair).

Timing: W warm-up steps and one untimed replay of the timed graphs, then
exactly K steps replayed from CUDA graphs and bracketed by CUDA events on the
launching stream (barrier + synchronize on both sides, max over ranks).
Decode steps rotate over L copies of the layer's cache and summaries so that
the bytes touched between reuses exceed 3x L2; prefill inputs exceed L2.
With N > 1 every rank runs its own replica (independent sequences, no
data-path collective): weak scaling.

cpu_baseline: the fp64 oracle on the host, on bounded samples of the same
workload, once on one core and once on all cores (a spawn process pool over
independent rows or query blocks). --impl reference times that oracle alone.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn decode GB/s vs HBM peak; prefill fwd+bwd TFLOP/s vs bf16 peak"
DEFAULT_STEPS = {"c1": 200, "c2": 100000, "c3": 200, "c4": 4000, "c5": 20000}
DEFAULT_WARMUP = {"c1": 10, "c2": 1000, "c3": 3, "c4": 100, "c5": 500}
# reference arm (the fp64 oracle on one core): steps without --steps, and the
# most steps it times (an oracle step takes tens of milliseconds)
REFERENCE_STEPS = 20
REFERENCE_MAX_STEPS = 1000
# (record name, config, options) of the default run; the first is the headline
ALL_RECORDS = (("c5", "c5", {}), ("c5_bf16_summaries", "c5", {"summary": "bf16"}),
               ("c4", "c4", {}), ("c2", "c2", {}), ("c2_paged", "c2", {"paged": True}),
               ("c3", "c3", {}), ("c3_tokens", "c3", {"tokens": True}))


# ----------------------------------------------------------------- helpers
def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    sm_max=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sm_max=1965.0, source="fallback")


def source_sha(name: str) -> str:
    """Hash of a kernel's source file and the shared device headers."""
    h = hashlib.sha256()
    for f in (name, "common.cuh", "ptx.cuh", "tc.cuh"):
        h.update(open(os.path.join(ROOT, "gated_block_sparse_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, source: str, workload: str | None = None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of the kernel (and on this workload when the
    record names one); else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    recs = json.load(open(p))
    rec = recs.get(f"{kernel}@{workload}") if workload else None
    rec = rec or recs.get(kernel)
    if not rec or rec.get("source_sha") != source_sha(source):
        return None
    if workload and rec.get("workload", workload) != workload:
        return None
    return rec.get("dram_bytes_per_launch")


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


class ClockSampler:
    """nvidia-smi samples every 100 ms; summarised over a wall-clock window."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
        self.f.flush()

    def summary(self, t0: float, t1: float) -> dict:
        rows = []
        try:
            for r in csv.reader(open(self.f.name)):
                if len(r) < 9:
                    continue
                ts = time.mktime(time.strptime(r[0].strip().split(".")[0], "%Y/%m/%d %H:%M:%S"))
                frac = float("0." + r[0].strip().split(".")[1]) if "." in r[0] else 0.0
                rows.append((ts + frac, [x.strip() for x in r[1:]]))
        except Exception:
            rows = []
        win = [x for t, x in rows if t0 - 0.15 <= t <= t1 + 0.15] or \
              [x for t, x in rows if t >= t0][:1] or [x for _, x in rows[-1:]]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for x in win for n, v in zip(names, x[4:8]) if v.lower() == "active"})
        sm = [float(x[0]) for x in win if x[0].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(win[0][1]) if win[0][1].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(win)}


_SAMPLER: ClockSampler | None = None


def clock_sampler(gpu_index: int) -> ClockSampler:
    """One sampler for the whole run, started before the first workload, so
    that a short timed region still has samples around it."""
    global _SAMPLER
    if _SAMPLER is None:
        _SAMPLER = ClockSampler(gpu_index)
        time.sleep(0.5)
    return _SAMPLER


def barrier(world):
    from gated_block_sparse_b200 import dist as D
    D.barrier(world)


def max_over_ranks(world, x: float) -> float:
    from gated_block_sparse_b200 import dist as D
    return D.max_over_ranks(world, x)


def timed_graphs(fn_step, n_steps: int, warmup: int, world: int, stream, chunk: int = 512,
                 clocks: ClockSampler | None = None):
    """Capture fn_step(i) for i in [0, chunk) into a graph (plus a tail graph)
    and time exactly n_steps steps after `warmup` untimed ones and one
    untimed replay of every graph the timed schedule uses (so the timed
    region holds no first launch of a graph). Returns (ms total, max over
    ranks; clock summary)."""
    import torch
    chunk = max(1, min(chunk, n_steps))
    graphs = {}

    def graph_of(n):
        if n not in graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    fn_step(i)
            graphs[n] = g
        return graphs[n]

    def run(n):
        full, tail = divmod(n, chunk)
        for _ in range(full):
            graph_of(chunk).replay()
        if tail:
            graph_of(tail).replay()

    with torch.cuda.stream(stream):
        run(max(3, warmup))
        graph_of(chunk).replay()
        if n_steps % chunk:
            graph_of(n_steps % chunk).replay()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.time()
        start.record(stream)
        run(n_steps)
        end.record(stream)
        torch.cuda.synchronize()
        t1 = time.time()
        barrier(world)
    ms = max_over_ranks(world, start.elapsed_time(end))
    return ms, (clocks.summary(t0, t1) if clocks else None)


def event_ms(fn, n: int, stream) -> float:
    """Device time of n eager calls of fn on `stream` (ms, after 3 warm-ups)."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
    return a.elapsed_time(b)


# ----------------------------------------------------------------- decode
def decode_bytes(c: dict, lens, summary: str = "f32") -> tuple[int, int, int]:
    """Algorithmic bytes of one decode step: (selection, attention, whole step).

    Selection reads each row's C summaries (C = (n-1)//64; 4 bytes per
    element, 2 with bf16 summaries) and q; attention reads the kk = min(k, C)
    kept blocks' and the current block's n-64C tokens of K and V, q, and
    writes o; the fused step reads q once.
    """
    C = [(int(n) - 1) // 64 for n in lens]
    kk = [min(c["topk"], x) for x in C]
    ncur = [int(n) - 64 * x for n, x in zip(lens, C)]
    d, Hkv, es = c["d"], c["Hkv"], 2 if c["dtype"] == "bf16" else 4
    ses = 2 if summary == "bf16" else 4
    qb = c["B"] * c["Hq"] * d * es
    sel = sum(Hkv * x * d * ses for x in C) + qb
    att = sum(Hkv * (k * 64 + nc) * d * es * 2 for k, nc in zip(kk, ncur)) + 2 * qb
    return sel, att, sel + att - qb


class DecodeWorkload:
    def __init__(self, name: str, summary: str = "f32", host=None):
        from gated_block_sparse_b200 import inputs
        self.name = name
        self.summary = summary
        self.c = inputs.CONFIGS[name]
        self.host = inputs.gen_config(name) if host is None else host
        c = self.c
        self.rows = c["B"] * c["Hkv"]
        self.sel_bytes, self.att_bytes, self.step_bytes = decode_bytes(
            c, self.host["lens"].numpy(), summary)

    def describe(self):
        from gated_block_sparse_b200 import inputs
        c = self.c
        return {"workload": f"{self.name}: {inputs.DESCRIPTIONS[self.name]}", "batch": c["B"],
                "q_heads": c["Hq"], "kv_heads": c["Hkv"], "head_dim": c["d"],
                "context": c["Lmax"] if c["lens"][0] == c["lens"][1] else list(c["lens"]),
                "topk": c["topk"], "gated": c["gated"], "block": 64,
                "summaries": "bf16" if self.summary == "bf16" else "fp32",
                "bytes_per_step": self.step_bytes, "selected_kv_bytes_per_step": self.att_bytes}


def bench_decode_ours(K: int, W: int, world: int, local: int, w: DecodeWorkload,
                      paged: bool = False, layers: int = 0) -> dict:
    import torch

    from gated_block_sparse_b200 import sas
    c = w.c
    dev = torch.device("cuda", local if world > 1 else 0)
    h = w.host
    q = h["q"].to(dev)
    lens = h["lens"].to(dev)
    kc0, vc0 = h["kc"].to(dev), h["vc"].to(dev)
    bf16_sum = w.summary == "bf16"
    ks0 = (sas.sas_block_summary_ex(kc0, torch.bfloat16) if bf16_sum
           else sas.sas_block_summary(kc0))
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per_layer = kc0.numel() * kc0.element_size() * 2 + ks0.numel() * ks0.element_size()
    free = torch.cuda.mem_get_info(dev)[0]
    L = max(2, math.ceil(3 * l2 / w.step_bytes))
    L = min(L, max(2, int(0.6 * free // per_layer)))
    if layers:
        L = layers
    kcs, vcs, kss = [kc0], [vc0], [ks0]
    for _ in range(L - 1):
        kcs.append(kc0.clone())
        vcs.append(vc0.clone())
        kss.append(ks0.clone())
    topk, Hkv = c["topk"], c["Hkv"]
    bt = None
    if paged:  # the same caches scattered into 64-token pages, random page order
        B_, _, Lmax_, d_ = kc0.shape
        nblk = Lmax_ // 64
        perm = torch.randperm(B_ * nblk, generator=torch.Generator().manual_seed(12345)).to(dev)
        bt = perm.view(B_, nblk).to(torch.int32).contiguous()

        def pages(x):
            p = torch.empty((B_ * nblk, Hkv, 64, d_), dtype=x.dtype, device=dev)
            p[perm] = x.view(B_, Hkv, nblk, 64, d_).permute(0, 2, 1, 3, 4).reshape(
                B_ * nblk, Hkv, 64, d_)
            return p
        for j in range(L):
            kcs[j], vcs[j] = pages(kcs[j]), pages(vcs[j])
            kss[j] = (sas.sas_block_summary_ex(kcs[j], torch.bfloat16) if bf16_sum
                      else sas.sas_block_summary(kcs[j])).view(B_ * nblk, Hkv, d_)
    o = torch.empty_like(q)
    stream = torch.cuda.Stream(dev)
    clocks = clock_sampler(dev.index if dev.index is not None else 0)

    def decode(j, qq, out):
        if bt is not None:  # sas_decode_paged_ex takes the summaries' dtype from kss[j]
            sas.sas_decode_paged_ex(qq, kcs[j], vcs[j], kss[j], bt, lens, topk,
                                    gated=c["gated"], out=out)
        elif bf16_sum:
            sas.sas_decode_ex(qq, kcs[j], vcs[j], lens, kss[j], topk, gated=c["gated"], out=out)
        else:
            sas.sas_decode(qq, kcs[j], vcs[j], lens, kss[j], topk, gated=c["gated"], out=out)

    def step(i):
        decode(i % L, q, o)

    ms, clk = timed_graphs(step, K, W, world, stream, clocks=clocks)

    # split path (contiguous caches, fp32 summaries): selection alone, attention alone
    split = None
    if bt is None and not bf16_sum:
        split = split_path_timing(sas, c, w, q, lens, kcs, vcs, kss, L, K, world, stream, o)
    peaks = measured_peaks()
    # the step is one launch of the cluster kernel: its duration is the step's
    kt = ms / K * 1e-3
    ach = w.step_bytes / kt / 1e9
    ach_sel = w.att_bytes / kt / 1e9
    variant = ("paged" if bt is not None else None, "bf16_summaries" if bf16_sum else None)
    variant = "_".join(v for v in variant if v) or None
    roof = {"bound": "hbm", "kernel": "k_decode_fused", "achieved": round(ach, 1),
            "peak": peaks["hbm"], "unit": "GB/s", "frac": round(ach / peaks["hbm"], 4),
            "traffic": (None if variant else
                        recorded_traffic("k_decode_fused", "k_decode_fused.cu", w.name)),
            "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)",
            "algorithmic_bytes_per_launch": w.step_bytes, "launch_us": round(kt * 1e6, 3),
            "selected_kv_bytes_per_launch": w.att_bytes,
            "achieved_selected_kv": round(ach_sel, 1),
            "frac_selected_kv": round(ach_sel / peaks["hbm"], 4),
            "split_path": split}
    rec = finish_decode(sas, c, w, q, lens, kcs, vcs, kss, L, K, W, world, stream, o, decode,
                        ms, clk, roof, l2, variant)
    del kcs, vcs, kss, kc0, vc0, ks0
    torch.cuda.empty_cache()
    return rec


def split_path_timing(sas, c, w, q, lens, kcs, vcs, kss, L, K, world, stream, o):
    import torch
    dev = q.device
    topk, Hkv = c["topk"], c["Hkv"]
    sel = [sas.sas_select(q, kss[j], Hkv, topk, "decode", lens=lens) for j in range(L)]
    sel_ws = torch.empty(max(16, sas.load_library().sas_select_workspace_size(
        c["B"], c["Hq"], Hkv, c["Lmax"], c["d"], topk, 1)), dtype=torch.uint8, device=dev)
    att_ws = torch.empty(max(16, sas.load_library().sas_decode_attend_workspace_size(
        c["B"], c["Hq"], Hkv, c["Lmax"], c["d"], topk)), dtype=torch.uint8, device=dev)
    sel_out = [(torch.empty_like(a), torch.empty_like(b), torch.empty_like(cc)) for a, b, cc in sel]

    def sel_step(i):
        j = i % L
        sas.sas_select(q, kss[j], Hkv, topk, "decode", lens=lens, out=sel_out[j], ws=sel_ws)

    def att_step(i):
        j = i % L
        sas.sas_decode_attend(q, kcs[j], vcs[j], lens, *sel[j], gated=c["gated"], out=o, ws=att_ws)

    ms_sel, _ = timed_graphs(sel_step, K, 10, world, stream)
    ms_att, _ = timed_graphs(att_step, K, 10, world, stream)
    t_sel, t_att = ms_sel / K * 1e-3, ms_att / K * 1e-3
    return {"k_select_decode": {"us": round(t_sel * 1e6, 3),
                                "GBps": round(w.sel_bytes / t_sel / 1e9, 1)},
            "k_decode_attend": {"us": round(t_att * 1e6, 3),
                                "GBps": round(w.att_bytes / t_att / 1e9, 1)}}


def finish_decode(sas, c, w, q, lens, kcs, vcs, kss, L, K, W, world, stream, o, decode, ms, clk,
                  roof, l2, variant) -> dict:
    import torch

    from gated_block_sparse_b200 import dist as D
    # end to end through the public API: pinned host q in, o out, every step
    qh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    qh.copy_(q.cpu())
    oh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    qd = torch.empty_like(q)
    E = max(K, 200)

    def e2e_step(i):
        j = i % L
        if variant:  # host copies through torch around the call
            qd.copy_(qh, non_blocking=True)
            decode(j, qd, o)
            oh.copy_(o, non_blocking=True)
        else:  # one C call: the step reads q from and writes o to pinned host memory
            sas.sas_decode_host(qh, qd, kcs[j], vcs[j], lens, kss[j], c["topk"], o, oh,
                                gated=c["gated"])

    # (a) eager: one public-API call per step from Python
    with torch.cuda.stream(stream):
        for i in range(20):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0 = time.perf_counter()
        e0.record(stream)
        for i in range(E):
            e2e_step(i)
        h1 = time.perf_counter()
        e1.record(stream)
        torch.cuda.synchronize()
    ms_eager = max_over_ranks(world, e0.elapsed_time(e1))
    # (b) for comparison, the same public-API step captured in a CUDA graph
    # (one per rotated layer copy) and launched once per step
    graphs = []
    with torch.cuda.stream(stream):
        for j in range(L):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                e2e_step(j)
            graphs.append(g)
        for i in range(2 * L):
            graphs[i % L].replay()
        torch.cuda.synchronize()
        barrier(world)
        e0.record(stream)
        for i in range(E):
            graphs[i % L].replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms_e2e = max_over_ranks(world, e0.elapsed_time(e1))
    del graphs
    # where a step's time goes: the host-side call alone (enqueue time per
    # eager step), a q copy alone and the kernel alone (the device-timed step)
    copy_ms = event_ms(lambda: qd.copy_(qh, non_blocking=True), E, stream)
    nb = q.numel() * q.element_size()
    api = ({"paged": "sas_decode_paged_ex with torch copies",
            "paged_bf16_summaries": "sas_decode_paged_ex with torch copies",
            "bf16_summaries": "sas_decode_ex with torch copies"}.get(variant) or
           "sas_decode_host (the step reading q from and writing o to pinned host memory)")
    value = D.whole_job_rate(w.step_bytes * K, world, ms) / 1e9
    cfg = {**w.describe(), "parallelism": f"replicas x{world}",
           "cache": ("paged: 64-token pages in a random page order"
                     if variant and variant.startswith("paged")
                     else "contiguous [B][Hkv][Lmax][d]"),
           "l2": f"rotating {L} layer copies of cache + summaries "
                 f"({w.step_bytes * L / 1e6:.0f} MB touched per rotation, L2 {l2 / 1e6:.0f} MB)"}
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if c["dtype"] == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) with planted relevant blocks)",
        "config": cfg,
        "roofline": roof,
        "e2e": {"value": round(D.whole_job_rate(w.step_bytes * E, world, ms_eager) / 1e9, 2),
                "unit": "GB/s", "h2d_bytes_per_step": nb, "d2h_bytes_per_step": nb,
                "path": f"pinned host q -> {api} via the Python binding -> pinned host o",
                "split_us_per_step": {"end_to_end": round(ms_eager / E * 1e3, 3),
                                      "host_call": round((h1 - h0) / E * 1e6, 3),
                                      "graph_launch_per_step": round(ms_e2e / E * 1e3, 3),
                                      "q_copy_in_alone": round(copy_ms / E * 1e3, 3),
                                      "kernel": round(ms / K * 1e3, 3)},
                "steps": E},
        "gpu_launches": K,
        "clocks": clk,
    }


# ----------------------------------------------------------------- prefill
def prefill_flops(idx_cnt, N: int, Hq: int, Hkv: int, d: int):
    """Algorithmic FLOPs of one forward and one backward (per sequence sum)."""
    import numpy as np
    cnt = np.asarray(idx_cnt)  # [B][Hkv][T]
    G = Hq // Hkv
    T = cnt.shape[-1]
    pairs = 0
    for t in range(T):
        nr = min(64, N - 64 * t)
        pairs += int(cnt[..., t].sum()) * G * nr * 64 + cnt.shape[0] * Hq * nr * (nr + 1) // 2
    return 4 * d * pairs, 10 * d * pairs


def prefill_flops_tokens(cnt_tok, N: int, Hq: int, Hkv: int, d: int):
    """Algorithmic FLOPs of one forward and one backward with per-token
    selection rows: every token i of every head sees 64 keys of each of its
    cnt_i kept blocks and the i % 64 + 1 causal keys of its own block."""
    import numpy as np
    cnt = np.asarray(cnt_tok)  # [B][Hkv][N]
    G = Hq // Hkv
    cur = (np.arange(N) % 64 + 1).astype(np.int64)
    pairs = int(G * (64 * cnt.astype(np.int64).sum() + cnt.shape[0] * cnt.shape[1] * cur.sum()))
    return 4 * d * pairs, 10 * d * pairs


def bench_prefill_ours(name: str, K: int, W: int, world: int, local: int, host=None,
                       tokens: bool = False) -> dict:
    import torch

    from gated_block_sparse_b200 import dist as D
    from gated_block_sparse_b200 import inputs, sas
    c = inputs.CONFIGS[name]
    dev = torch.device("cuda", local if world > 1 else 0)
    h = inputs.gen_config(name) if host is None else host
    q, k, v, do = (h[n].to(dev) for n in ("q", "k", "v", "do"))
    topk, Hkv = c["topk"], c["Hkv"]
    B, Hq, N, d = q.shape
    ks = sas.sas_block_summary(k)
    lib = sas.load_library()
    dt = 1 if c["dtype"] == "bf16" else 0
    if tokens:  # per-token selection rows (each query token its own block set)
        idx, cnt, logg = sas.sas_select_tokens(q, ks, Hkv, topk)
        o, lse = sas.sas_attn_fwd_tokens(q, k, v, idx, cnt, logg)
        bwd_ws = torch.empty(max(16, lib.sas_attn_bwd_tokens_workspace_size(B, Hq, Hkv, N, d)),
                             dtype=torch.uint8, device=dev)
        grads = sas.sas_attn_bwd_tokens(q, k, v, o, do, lse, idx, cnt, logg, ws=bwd_ws)
        sbw_ws = torch.empty(max(16, lib.sas_select_bwd_tokens_workspace_size(B, Hq, Hkv, N, d)),
                             dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        f_fwd, f_bwd = prefill_flops_tokens(cnt.cpu().numpy(), N, Hq, Hkv, d)
    else:
        idx, cnt, logg = sas.sas_select(q, ks, Hkv, topk, "prefill")
        o, lse = sas.sas_attn_fwd(q, k, v, idx, cnt, logg)
        grads = sas.sas_attn_bwd(q, k, v, o, do, lse, idx, cnt, logg)
        torch.cuda.synchronize()
        f_fwd, f_bwd = prefill_flops(cnt.cpu().numpy(), N, Hq, Hkv, d)
        bwd_ws = torch.empty(max(16, lib.sas_attn_bwd_workspace_size(B, Hq, Hkv, N, d, topk, dt)),
                             dtype=torch.uint8, device=dev)
        sbw_ws = torch.empty(max(16, lib.sas_select_bwd_workspace_size(B, Hq, Hkv, N, d)),
                             dtype=torch.uint8, device=dev)
    sel_ws = torch.empty(max(16, lib.sas_select_workspace_size(B, Hq, Hkv, N, d, topk, 0)),
                         dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    clocks = clock_sampler(dev.index if dev.index is not None else 0)

    def step(i):
        sas.sas_block_summary(k, out=ks)
        if tokens:
            sas.sas_select_tokens(q, ks, Hkv, topk, out=(idx, cnt, logg))
            sas.sas_attn_fwd_tokens(q, k, v, idx, cnt, logg, out=(o, lse))
            sas.sas_attn_bwd_tokens(q, k, v, o, do, lse, idx, cnt, logg, out=grads, ws=bwd_ws)
            sas.sas_select_bwd_tokens(q, ks, Hkv, idx, cnt, grads[3], grads[0], grads[1],
                                      ws=sbw_ws)
            return
        sas.sas_select(q, ks, Hkv, topk, "prefill", out=(idx, cnt, logg), ws=sel_ws)
        sas.sas_attn_fwd(q, k, v, idx, cnt, logg, out=(o, lse))
        sas.sas_attn_bwd(q, k, v, o, do, lse, idx, cnt, logg, out=grads, ws=bwd_ws)
        # the gradient through the selector (eq. 8), added into dq and dk
        sas.sas_select_bwd(q, ks, Hkv, idx, cnt, grads[3], grads[0], grads[1], ws=sbw_ws)

    ms, clk = timed_graphs(step, K, W, world, stream, chunk=8, clocks=clocks)

    def fwd_step(i):
        if tokens:
            sas.sas_attn_fwd_tokens(q, k, v, idx, cnt, logg, out=(o, lse))
        else:
            sas.sas_attn_fwd(q, k, v, idx, cnt, logg, out=(o, lse))

    def bwd_step(i):
        if tokens:
            sas.sas_attn_bwd_tokens(q, k, v, o, do, lse, idx, cnt, logg, out=grads, ws=bwd_ws)
        else:
            sas.sas_attn_bwd(q, k, v, o, do, lse, idx, cnt, logg, out=grads, ws=bwd_ws)

    def sbw_step(i):
        if tokens:
            sas.sas_select_bwd_tokens(q, ks, Hkv, idx, cnt, grads[3], grads[0], grads[1],
                                      ws=sbw_ws)
        else:
            sas.sas_select_bwd(q, ks, Hkv, idx, cnt, grads[3], grads[0], grads[1], ws=sbw_ws)

    Kp = max(3, K)
    ms_f, _ = timed_graphs(fwd_step, Kp, 2, world, stream, chunk=8)
    ms_b, _ = timed_graphs(bwd_step, Kp, 2, world, stream, chunk=8)
    ms_s, _ = timed_graphs(sbw_step, Kp, 2, world, stream, chunk=8)
    tf, tb = ms_f / Kp * 1e-3, ms_b / Kp * 1e-3
    peaks = measured_peaks()
    tensor = c["dtype"] == "bf16" and d == 128 and (Hq // Hkv) % 2 == 0
    if tensor:  # tcgen05 kernels, timed alone: the burst bf16 peak
        names = ("k_attn_fwd_tc", "k_attn_bwd_tc")
        srcs = ("k_attn_fwd_tc.cu", "k_attn_bwd_tc.cu")
        peak, bound = peaks["bf16"], "tensor"
        psrc = f"{peaks['source']} (MEASURED_PEAKS.json bf16_tflops, cuBLAS bf16 burst)"
    else:  # fp32 CUDA-core kernels
        names = ("k_attn_fwd_simt", "k_attn_bwd_simt")
        srcs = ("k_attn_simt.cu", "k_attn_simt.cu")
        peak, bound = 148 * 128 * 2 * peaks["sm_max"] * 1e6 / 1e12, "alu"
        psrc = "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x max SM clock"
    i = 1 if tb >= tf else 0
    kern, kf, kt = names[i], (f_fwd, f_bwd)[i], (tf, tb)[i]
    ach = kf / kt / 1e12
    roof = {"bound": bound, "kernel": kern, "achieved": round(ach, 2), "peak": round(peak, 1),
            "unit": "TFLOP/s", "frac": round(ach / peak, 4),
            "traffic": recorded_traffic(kern, srcs[i], name + ("_tokens" if tokens else "")),
            "peak_source": psrc,
            "algorithmic_flops_per_launch": kf, "launch_ms": round(kt * 1e3, 4),
            "fwd_ms": round(tf * 1e3, 4), "bwd_ms": round(tb * 1e3, 4),
            "fwd_tflops": round(f_fwd / tf / 1e12, 2), "bwd_tflops": round(f_bwd / tb / 1e12, 2),
            "fwd_frac": round(f_fwd / tf / 1e12 / peak, 4),
            "bwd_frac": round(f_bwd / tb / 1e12 / peak, 4),
            "fwd_plus_bwd_frac": round((f_fwd + f_bwd) / (tf + tb) / 1e12 / peak, 4),
            "select_bwd_ms": round(ms_s / Kp, 4)}

    # end to end: pinned host inputs in, gradients out
    pin = {n: torch.empty(h[n].shape, dtype=h[n].dtype, pin_memory=True) for n in ("q", "k", "v", "do")}
    for n in pin:
        pin[n].copy_(h[n])
    outs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o,) + tuple(grads)]
    E = max(3, min(K, 10))

    def copy_in():
        q.copy_(pin["q"], non_blocking=True)
        k.copy_(pin["k"], non_blocking=True)
        v.copy_(pin["v"], non_blocking=True)
        do.copy_(pin["do"], non_blocking=True)

    def copy_out():
        for dst, src in zip(outs, (o,) + tuple(grads)):
            dst.copy_(src, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            copy_in()
            step(0)
            copy_out()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(E):
            copy_in()
            step(0)
            copy_out()
        e1.record(stream)
        torch.cuda.synchronize()
    ms_e2e = max_over_ranks(world, e0.elapsed_time(e1))
    ms_in = event_ms(copy_in, E, stream)
    ms_out = event_ms(copy_out, E, stream)
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in outs)
    total = f_fwd + f_bwd
    rec = {
        "metric": METRIC, "value": round(D.whole_job_rate(total * K, world, ms) / 1e12, 4),
        "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if c["dtype"] == "bf16" else "f32", "data": "synthetic (seeded N(0,1), planted)",
        "config": {"workload": f"{name}: {inputs.DESCRIPTIONS[name]}"
                               + (", per-token selection rows" if tokens else ""),
                   "batch": B, "seq_len": N,
                   "q_heads": Hq, "kv_heads": Hkv, "head_dim": d, "topk": topk,
                   "flops_fwd": f_fwd, "flops_bwd": f_bwd, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2 (q+k+v+dO = {h2d / 1e6:.0f} MB)"},
        "roofline": roof,
        "e2e": {"value": round(total * E * world / (ms_e2e * 1e-3) / 1e12, 4), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "pinned host q, k, v, dO -> the step's five library calls -> pinned host "
                        "o, dq, dk, dv, dlogg",
                "split_ms_per_step": {"end_to_end": round(ms_e2e / E, 4),
                                      "copy_in": round(ms_in / E, 4),
                                      "copy_out": round(ms_out / E, 4),
                                      "step": round(ms / K, 4)},
                "steps": E},
        # block rows: summary, query means, selection, forward, backward, 2
        # conversions, selector backward (query means, rows, columns); token
        # rows: summary, selection, forward, backward, 2 conversions, selector
        # backward (rows, spread)
        "gpu_launches": (8 if tokens else 10) * K,
        "clocks": clk,
    }
    del q, k, v, do, grads, o, lse
    torch.cuda.empty_cache()
    return rec


# ----------------------------------------------------------------- oracle baselines
# The oracle (fp64 numpy, oracle/) timed on the host cores on bounded samples.
# One-core runs limit BLAS to one thread; all-core runs use a spawn process
# pool (one BLAS thread each) over independent decode rows or prefill query
# blocks, sharing the input tensors through shared memory.
def _one_thread():
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1)


def _decode_rows_worker(args):
    """Decode rows (b, r) of one workload, round-robin, for `seconds`; each
    row is one oracle decode step of a single-row problem. Returns (rows
    done, seconds)."""
    from oracle import sas_oracle as O
    rows, seconds, topk, gated, G = args
    with _one_thread():
        n, t0 = 0, time.perf_counter()
        while True:
            q, kc, vc, lens, ks = rows[n % len(rows)]
            O.decode(q, kc, vc, lens, ks, 1, topk, gated=gated)
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                return n, el


def _prefill_units_worker(args):
    """Prefill (kv group, query block) units, forward + backward of the
    group's heads, for `seconds`. Returns (FLOPs done, units done, seconds)."""
    from oracle import sas_oracle as O
    units, seconds, d = args
    with _one_thread():
        flops, n, t0 = 0, 0, time.perf_counter()
        while True:
            q, k, v, do, idx, cnt, logg, t, G, N = units[n % len(units)]
            O.query_block(q, k, v, do, idx, cnt, logg, 0, 0, t)
            nr = min(64, N - 64 * t)
            flops += 14 * d * (int(cnt[0, 0, t]) * G * nr * 64 + G * nr * (nr + 1) // 2)
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                return flops, n, el


def _pool_map(fn, tasks):
    import torch.multiprocessing as tmp
    with tmp.get_context("spawn").Pool(len(tasks)) as pool:
        return pool.map(fn, tasks)


def cpu_baseline_decode(w: DecodeWorkload, seconds: float, all_cores: bool = True) -> dict:
    """The fp64 oracle on whole decode steps of the workload (one core), and
    on all cores over its independent rows."""
    from oracle import sas_oracle as O
    c = w.c
    h = w.host
    with _one_thread():
        ks = O.block_summary(h["kc"], lens=h["lens"].numpy())  # cache state, as on the GPU
        if w.summary == "bf16":
            ks = O.round_bf16(ks)
        lens = h["lens"].numpy()
        n, t0 = 0, time.perf_counter()
        while True:
            O.decode(h["q"], h["kc"], h["vc"], lens, ks, c["Hkv"], c["topk"], gated=c["gated"])
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    one = w.step_bytes * n / el / 1e9
    res = {"value": round(one, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "steps": n, "seconds": round(el, 2),
           "sample": f"{n} whole decode steps of {w.name} (all {w.rows} rows), fp64 numpy "
                     f"oracle, 1 BLAS thread; summaries precomputed as on the GPU",
           "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    ncpu = os.cpu_count() or 1
    if all_cores and ncpu > 1:
        G = c["Hq"] // c["Hkv"]
        rows = []
        for b in range(c["B"]):
            for r in range(c["Hkv"]):
                rows.append((h["q"][b:b + 1, r * G:(r + 1) * G].clone(),
                             h["kc"][b:b + 1, r:r + 1].clone(), h["vc"][b:b + 1, r:r + 1].clone(),
                             lens[b:b + 1].copy(), ks[b:b + 1, r:r + 1].copy()))
        P = min(ncpu, len(rows))
        tasks = [(rows[j::P], seconds, c["topk"], c["gated"], G) for j in range(P)]
        out = _pool_map(_decode_rows_worker, tasks)
        done = sum(x[0] for x in out)
        span = max(x[1] for x in out)
        rate = done / w.rows / span * w.step_bytes / 1e9
        res["all_cores"] = {"value": round(rate, 4), "unit": "GB/s", "cores": P,
                            "rows": done, "seconds": round(span, 2),
                            "sample": f"{P} processes (spawn, 1 BLAS thread each) each running "
                                      f"its share of the {w.rows} rows for {seconds:g} s; rate = "
                                      f"rows done / rows per step / slowest process's time"}
    return res


def reference_arm(cfg: str, summary: str, K: int, W: int) -> dict:
    """The oracle as the reference arm: W untimed and K timed steps on one
    core (one BLAS thread), each step a bounded sample of the workload: a
    whole decode step (all rows) for decode workloads, one (sequence, kv
    group, query block) unit's forward and backward, latest blocks first and
    cycling, for prefill."""
    from gated_block_sparse_b200 import inputs
    from oracle import sas_oracle as O
    c = inputs.CONFIGS[cfg]
    with _one_thread():
        if c["kind"] == "decode":
            w = DecodeWorkload(cfg, summary)
            h = w.host
            ks = O.block_summary(h["kc"], lens=h["lens"].numpy())
            if summary == "bf16":
                ks = O.round_bf16(ks)
            lens = h["lens"].numpy()

            def step(i):
                O.decode(h["q"], h["kc"], h["vc"], lens, ks, c["Hkv"], c["topk"], gated=c["gated"])
                return w.step_bytes
            unit, scale_to, what = "GB/s", 1e9, f"a whole decode step of {cfg} (all {w.rows} rows)"
        else:
            h = inputs.gen_config(cfg)
            N, d, G = c["N"], c["d"], c["Hq"] // c["Hkv"]
            ks = O.block_summary(h["k"])
            idx, cnt, logg, _ = O.select_prefill(h["q"], ks, c["Hkv"], c["topk"])
            T = idx.shape[2]
            order = [(b, r, t) for t in range(T - 1, -1, -1) for b in range(c["B"])
                     for r in range(c["Hkv"])]

            def step(i):
                b, r, t = order[i % len(order)]
                O.query_block(h["q"], h["k"], h["v"], h["do"], idx, cnt, logg, b, r, t)
                nr = min(64, N - 64 * t)
                return 14 * d * (int(cnt[b, r, t]) * G * nr * 64 + G * nr * (nr + 1) // 2)
            unit, scale_to = "TFLOP/s", 1e12
            what = (f"one (sequence, kv group, query block) unit of {cfg}, forward + backward "
                    "of all heads of the group")
        for i in range(W):
            step(i)
        work, t0 = 0, time.perf_counter()
        for i in range(K):
            work += step(W + i)
        el = time.perf_counter() - t0
    value = round(work / el / scale_to, 6)
    return {"value": value, "unit": unit, "steps": K, "warmup": W, "seconds": round(el, 3),
            "cpu_baseline": {"value": value, "unit": unit, "cores": 1, "kind": "oracle",
                             "sample": f"{K} steps, each {what}; fp64 numpy oracle, 1 BLAS thread",
                             "cpu_model": cpu_model(), "nproc": os.cpu_count()}}


def cpu_baseline_prefill(name: str, seconds: float, host=None, all_cores: bool = True) -> dict:
    """The oracle's forward+backward on whole query blocks of the workload
    (one core), and on all cores over (kv group, query block) units."""
    from gated_block_sparse_b200 import inputs
    from oracle import sas_oracle as O
    c = inputs.CONFIGS[name]
    h = inputs.gen_config(name) if host is None else host
    N, d = c["N"], c["d"]
    G = c["Hq"] // c["Hkv"]
    with _one_thread():
        ks = O.block_summary(h["k"])
        idx, cnt, logg, _ = O.select_prefill(h["q"], ks, c["Hkv"], c["topk"])
        T = idx.shape[2]
        n, flops, t0 = 0, 0, time.perf_counter()
        order = [(b, r, t) for t in range(T - 1, -1, -1) for b in range(c["B"])
                 for r in range(c["Hkv"])]
        for (b, r, t) in order:
            O.query_block(h["q"], h["k"], h["v"], h["do"], idx, cnt, logg, b, r, t)
            nr = min(64, N - 64 * t)
            pairs = int(cnt[b, r, t]) * G * nr * 64 + G * nr * (nr + 1) // 2
            flops += 14 * d * pairs
            n += 1
            if time.perf_counter() - t0 >= seconds:
                break
        el = time.perf_counter() - t0
    res = {"value": round(flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
           "seconds": round(el, 2),
           "sample": f"{n} of {len(order)} (sequence, kv group, query block) units of {name} "
                     "(forward + backward, all heads of the group, latest query blocks first), "
                     "fp64 numpy oracle, 1 BLAS thread",
           "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    ncpu = os.cpu_count() or 1
    if all_cores and ncpu > 1 and c["B"] == 1:
        P = ncpu
        units = []
        for t in range(T - 1, -1, -1):
            for r in range(c["Hkv"]):
                units.append((r, t))
        groups = {}
        for r in range(c["Hkv"]):
            groups[r] = (h["q"][:, r * G:(r + 1) * G].clone(), h["k"][:, r:r + 1].clone(),
                         h["v"][:, r:r + 1].clone(), h["do"][:, r * G:(r + 1) * G].clone(),
                         idx[:, r:r + 1].copy(), cnt[:, r:r + 1].copy(), logg[:, r:r + 1].copy())
        share = [[groups[r] + (t, G, N) for (r, t) in units[j::P][:64]] for j in range(P)]
        share = [s for s in share if s]
        out = _pool_map(_prefill_units_worker, [(s, seconds, d) for s in share])
        fl = sum(x[0] for x in out)
        span = max(x[2] for x in out)
        res["all_cores"] = {"value": round(fl / span / 1e12, 6), "unit": "TFLOP/s",
                            "cores": len(share), "units": sum(x[1] for x in out),
                            "seconds": round(span, 2),
                            "sample": f"{len(share)} processes (spawn, 1 BLAS thread each), each "
                                      f"cycling over up to 64 of the latest (kv group, query "
                                      f"block) units for {seconds:g} s; rate = FLOPs done / "
                                      f"slowest process's time"}
    return res


def cpu_baseline_prefill_tokens(name: str, seconds: float, host=None) -> dict:
    """The per-token oracle (selection, forward, backward) on a prefix of the
    workload: the first n tokens of every head (n grows by 64-token blocks
    while a pass stays within the time), so the sample keeps the workload's
    shapes and selection rule at shorter history."""
    from gated_block_sparse_b200 import inputs
    from oracle import sas_oracle as O
    c = inputs.CONFIGS[name]
    h = inputs.gen_config(name) if host is None else host
    d, Hkv, topk = c["d"], c["Hkv"], c["topk"]
    G = c["Hq"] // Hkv
    n, flops, el, passes = 256, 0, 0.0, 0
    with _one_thread():
        while True:
            x = {k_: h[k_][:, :, :n] for k_ in ("q", "k", "v", "do")}
            t0 = time.perf_counter()
            idx, cnt, logg, _ = O.select_prefill_tokens(x["q"], O.block_summary(x["k"]), Hkv, topk)
            O.attn_fwd_tokens(x["q"], x["k"], x["v"], idx, cnt, logg)
            O.attn_bwd_tokens(x["q"], x["k"], x["v"], x["do"], idx, cnt, logg)
            dt_ = time.perf_counter() - t0
            cur = sum(i % 64 + 1 for i in range(n))
            flops += 14 * d * G * (64 * int(cnt.sum()) + Hkv * cur)
            el += dt_
            passes += 1
            if el >= seconds or n >= c["N"]:
                break
            n = min(c["N"], 2 * n)
    return {"value": round(flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "seconds": round(el, 2),
            "sample": f"{passes} pass(es) over prefixes of {name}, from its first 256 tokens "
                      f"(doubling) to its first {n} tokens of every head: per-token selection, "
                      "forward and backward, fp64 numpy oracle, 1 BLAS thread",
            "cpu_model": cpu_model(), "nproc": os.cpu_count()}


# ----------------------------------------------------------------- main
def run_one(name: str, cfg: str, opts: dict, K: int, W: int, world: int, rank: int, local: int,
            cpu_seconds: float, hosts: dict, baselines: dict) -> dict:
    from gated_block_sparse_b200 import inputs
    c = inputs.CONFIGS[cfg]
    if cfg not in hosts:
        hosts.clear()  # one workload's inputs on the host at a time
        hosts[cfg] = inputs.gen_config(cfg)
    if c["kind"] == "decode":
        w = DecodeWorkload(cfg, opts.get("summary", "f32"), host=hosts[cfg])
        rec = bench_decode_ours(K, W, world, local, w, paged=opts.get("paged", False),
                                layers=opts.get("layers", 0))
        if rank == 0:
            key = (cfg, w.summary)
            if key not in baselines:
                baselines[key] = cpu_baseline_decode(w, cpu_seconds)
            rec["cpu_baseline"] = baselines[key]
    elif opts.get("tokens"):
        rec = bench_prefill_ours(cfg, K, W, world, local, host=hosts[cfg], tokens=True)
        if rank == 0:
            rec["cpu_baseline"] = cpu_baseline_prefill_tokens(cfg, cpu_seconds, host=hosts[cfg])
        rec["config"]["variant"] = "per-token selection (sas_select_tokens, *_tokens)"
    else:
        rec = bench_prefill_ours(cfg, K, W, world, local, host=hosts[cfg])
        if rank == 0:
            rec["cpu_baseline"] = cpu_baseline_prefill(cfg, cpu_seconds, host=hosts[cfg])
    parts = []
    if opts.get("paged"):
        parts.append("paged KV cache")
    if opts.get("summary") == "bf16":
        parts.append("bf16 block summaries")
    if parts:
        rec["config"]["variant"] = " + ".join(parts) + (
            " (sas_decode_paged_ex)" if opts.get("paged") else " (sas_decode_ex)")
    return rec


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--config", default="all", choices=["all", "c1", "c2", "c3", "c4", "c5"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=None,
                    help="oracle baseline sample per config and core setting "
                         "(default 4 s with --config all, 10 s otherwise)")
    ap.add_argument("--paged", action="store_true",
                    help="decode: read the caches through 64-token pages (sas_decode_paged)")
    ap.add_argument("--summary", default="f32", choices=["f32", "bf16"],
                    help="decode: store block summaries in fp32 or bf16 (sas_decode_ex)")
    ap.add_argument("--tokens", action="store_true",
                    help="prefill: per-token selection rows (sas_select_tokens, *_tokens)")
    ap.add_argument("--layers", type=int, default=0,
                    help="decode: number of rotated layer copies (default: enough for 3x L2)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    cpu_s = args.cpu_seconds or (4.0 if args.config == "all" else 10.0)

    if args.config == "all":
        plan = ALL_RECORDS
    else:
        opts = {"paged": args.paged, "summary": args.summary, "layers": args.layers,
                "tokens": args.tokens}
        plan = ((args.config, args.config, opts),)

    if args.impl == "reference":
        if rank != 0:
            return
        from gated_block_sparse_b200 import inputs
        name, cfg, opts = plan[0]
        K = min(args.steps or REFERENCE_STEPS, REFERENCE_MAX_STEPS)
        W = min(args.warmup if args.warmup is not None else 1, REFERENCE_MAX_STEPS)
        ref = reference_arm(cfg, opts.get("summary", "f32"), K, W)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": ref["value"], "unit": ref["unit"],
            "n_gpus": args.gpus, "steps": K, "warmup": W,
            "ms_per_step": ref["seconds"] * 1e3 / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded, same generator)",
            "config": {"workload": f"{cfg}: {inputs.DESCRIPTIONS[cfg]}"},
            "cpu_baseline": ref["cpu_baseline"],
            "e2e": {"value": ref["value"], "unit": ref["unit"], "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return

    from gated_block_sparse_b200 import dist as D
    world, rank, local = D.setup()
    clock_sampler(local if world > 1 else 0)
    records, hosts, baselines = {}, {}, {}
    for name, cfg, opts in plan:
        K = args.steps or DEFAULT_STEPS[cfg]
        W = max(3, args.warmup if args.warmup is not None else DEFAULT_WARMUP[cfg])
        records[name] = run_one(name, cfg, opts, K, W, world, rank, local, cpu_s, hosts, baselines)
    if rank == 0:
        head = dict(records[plan[0][0]])
        if len(plan) > 1:
            head["records"] = records
            head["config"] = dict(head["config"], headline=plan[0][0],
                                  records=[n for n, _, _ in plan])
        print(json.dumps(head))
    if _SAMPLER is not None:
        _SAMPLER.stop()
    D.teardown(world)


if __name__ == "__main__":
    main()
