"""Benchmark of the fused-attention hot path on B200.

One step = one pass of every operation on the path over its own seeded,
HBM-resident synthetic input (the five workloads):
  tiny      tiny causal self-attention         B1 Hq2 Hkv2 S128 D64     (frt_attn_fwd)
  prefill   Llama-3-8B-shaped causal prefill   B1 Hq32 Hkv8 S4096 D128  (frt_attn_fwd)
  paged     paged GQA decode                   B4 Hq64 Hkv8 D128 ps16, lens U[1024,32768]
                                               (frt_attn_decode_paged: streaming kernel,
                                               then the dependent LSE merge kernel)
  long      long-context split-KV decode       B1 Hq32 Hkv4 Skv262144 D128 ps16
  contig    single-token GQA decode            B1 Hq32 Hkv8 Skv4096 D128 (frt_attn_fwd, Sq=1:
                                               one launch, clusters merge in shared memory)
Each step's working set (~0.9 GB) exceeds the 126 MB L2, and every call's
inputs are evicted by the calls before it, so no call starts L2-warm.

Prints ONE JSON line (rank 0).  `value` is whole-job steps per second; the
per-call microseconds, TFLOP/s, GB/s and roofline fractions are under
"calls"; "roofline" describes the dominant kernel; "extras" holds calls
outside the step (the FP8-cache decode on the two paged workloads, cross
attention, the prefill through strided views), timed the same way.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (fp64, OpenMP) on the host cores: each
step is one full pass of the oracle over the same five workloads (rank 0
only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from flash_attention_tiled_b200 import inputs  # noqa: E402

METRIC = ("attn prefill TFLOP/s & decode KV GB/s vs B200 roofline; "
          "µs/call at batch 1")
WORKLOAD = ("tiny causal (B1 H2 S128 D64) + llama3-8b causal prefill 4k (B1 Hq32 Hkv8 D128) "
            "+ paged GQA decode (B4 Hq64 Hkv8 D128 ps16 lens U[1024,32768]) + 256k split-KV "
            "decode (B1 Hq32 Hkv4 D128 ps16) + 4k GQA decode (B1 Hq32 Hkv8 D128)")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PREROLL_S = 1.5          # untimed step replays under the clock sampler before the timed steps
REF_STEP_S_EST = 5.0     # one full oracle step on 16 host cores (seconds, for run planning)
REF_BUDGET_S = 240.0     # the reference arm's planned length


def source_sha() -> str:
    """Hash of the CUDA sources' code (comments and whitespace removed), to tell
    whether profiled counters still apply: a comment edit keeps them, a code
    change retires them."""
    import glob
    import hashlib
    import re
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "flash_attention_tiled_b200", "csrc", "*"))):
        if not f.endswith((".cu", ".cuh", ".h")):
            continue
        with open(f, encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(os.path.basename(f).encode())
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def profiled_traffic():
    """Per-call DRAM traffic (bytes per launch) from the committed ncu summary,
    or {} if the kernels changed since it was taken."""
    import re
    path = os.path.join(ROOT, "profiles", "dram_traffic__bench_calls.md")
    try:
        text = open(path).read()
    except OSError:
        return {}
    m_sha = re.search(r"^source-sha256: (\w+)", text, re.M)
    m_tr = re.search(r"^traffic_bytes: (.*)$", text, re.M)
    if not m_sha or not m_tr or m_sha.group(1) != source_sha():
        return {}
    return {k: float(v) for k, v in (kv.split("=") for kv in m_tr.group(1).split())}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------- work figures
def prefill_flops(w) -> float:
    """4*D flops per visible (query, key) pair per query head (2 for Q.K^T,
    2 for P.V; exp not counted); masked pairs are not counted."""
    off = w.Skv - w.Sq
    if w.causal:
        pairs = sum(max(0, min(w.Skv, i + off + 1)) for i in range(w.Sq))
    else:
        pairs = w.Sq * w.Skv
    return 4.0 * w.D * pairs * w.Hq * w.B


def prefill_bytes(w) -> float:
    q = w.B * w.Hq * w.Sq * w.D * 2
    kv = 2 * w.B * w.Hkv * w.Skv * w.D * 2
    return q + kv + q + w.B * w.Hq * w.Sq * 4          # Q, K, V, O, LSE


def decode_bytes(B, Hq, Hkv, D, total_tokens) -> float:
    """K and V of every cached token read once per KV head, plus q, o, lse."""
    return 2.0 * total_tokens * Hkv * D * 2 + B * Hq * D * 2 * 2 + B * Hq * 4


def decode_flops(Hq, D, total_tokens) -> float:
    return 4.0 * D * Hq * total_tokens


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# -------------------------------------------------------------- our arm
class Step:
    """The five calls of one step, with inputs resident on the device."""

    ALL = ("tiny", "prefill", "paged", "long", "contig")
    # the paged workloads with their cache stored as e4m3 (not part of the
    # configured step; --calls may name them, e.g. for a profile)
    FP8 = ("paged_fp8", "long_fp8")
    # kernels each call launches: prefill_kernel; decode_splitkv_kernel then
    # decode_merge_kernel (paged); the cluster-mode decode kernel alone (contig)
    LAUNCHES = {"tiny": 1, "prefill": 1, "paged": 2, "long": 2, "contig": 1, "paged_fp8": 2,
                "long_fp8": 2}

    def __init__(self, device, names=ALL):
        from flash_attention_tiled_b200 import frt
        self.frt = frt
        self.dev = device
        self.NAMES = tuple(names)
        W = inputs.WORKLOADS
        self.w_tn = W["tiny_causal"]
        self.w_pf = W["llama3_8b_prefill_4k"]
        self.w_pg = W["paged_gqa_decode_b4"]
        self.w_lg = W["long_splitkv_decode_256k"]
        self.w_ct = W["gqa_decode_4k"]
        wl = {"tiny": self.w_tn, "prefill": self.w_pf, "paged": self.w_pg, "long": self.w_lg,
              "contig": self.w_ct, "paged_fp8": self.w_pg, "long_fp8": self.w_lg}

        def make(n):
            w = wl[n]
            if n in Step.FP8:
                return inputs.paged_fp8(w.B, w.Hq, w.Hkv, w.D, len_range=w.len_range,
                                        page_size=w.page_size, seed=w.seed)
            return inputs.make(w)

        self.host = {n: make(n) for n in self.NAMES}
        self.d = {k: {n: (t.to(device) if isinstance(t, torch.Tensor) else t)
                      for n, t in v.items()} for k, v in self.host.items()}
        if "paged" in self.NAMES:
            self.tokens_pg = int(self.host["paged"]["seq_lens"].sum())
        if "long" in self.NAMES:
            self.tokens_lg = int(self.host["long"]["seq_lens"].sum())
        self.tokens = {n: int(self.host[n]["seq_lens"].sum()) for n in self.NAMES
                       if n in Step.FP8}
        # outputs, allocated once
        shapes = {"tiny": (self.w_tn.B, self.w_tn.Hq, self.w_tn.Sq),
                  "prefill": (self.w_pf.B, self.w_pf.Hq, self.w_pf.Sq),
                  "paged": (self.w_pg.B, self.w_pg.Hq), "long": (self.w_lg.B, self.w_lg.Hq),
                  "contig": (self.w_ct.B, self.w_ct.Hq, 1),
                  "paged_fp8": (self.w_pg.B, self.w_pg.Hq), "long_fp8": (self.w_lg.B, self.w_lg.Hq)}
        self.out = {n: (torch.empty_like(self.d[n]["q"]), torch.empty(shapes[n], device=device))
                    for n in self.NAMES}

    def call(self, name, d=None, out=None):
        d = self.d[name] if d is None else d
        o, l = self.out[name] if out is None else out
        f = self.frt
        if name == "tiny":
            f.attn_fwd(d["q"], d["k"], d["v"], causal=True, scale=self.w_tn.scale, out=o, lse=l)
        elif name == "prefill":
            f.attn_fwd(d["q"], d["k"], d["v"], causal=True, scale=self.w_pf.scale, out=o, lse=l)
        elif name == "contig":
            f.attn_fwd(d["q"], d["k"], d["v"], causal=False, scale=self.w_ct.scale, out=o, lse=l)
        elif name in Step.FP8:
            w = self.w_pg if name == "paged_fp8" else self.w_lg
            f.attn_decode_paged_fp8(d["q"], d["k_pages"], d["v_pages"], d["k_scale"], d["v_scale"],
                                    d["block_table"], d["seq_lens"], scale=w.scale, out=o, lse=l)
        else:
            w = self.w_pg if name == "paged" else self.w_lg
            f.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"],
                                d["seq_lens"], scale=w.scale, out=o, lse=l)

    def work(self):
        """Algorithmic (flops, bytes) of each call."""
        out = {}
        for n in self.NAMES:
            if n == "tiny":
                out[n] = (prefill_flops(self.w_tn), prefill_bytes(self.w_tn))
            elif n == "prefill":
                out[n] = (prefill_flops(self.w_pf), prefill_bytes(self.w_pf))
            elif n == "paged":
                out[n] = (decode_flops(self.w_pg.Hq, 128, self.tokens_pg),
                          decode_bytes(self.w_pg.B, self.w_pg.Hq, self.w_pg.Hkv, 128,
                                       self.tokens_pg))
            elif n == "long":
                out[n] = (decode_flops(self.w_lg.Hq, 128, self.tokens_lg),
                          decode_bytes(1, self.w_lg.Hq, self.w_lg.Hkv, 128, self.tokens_lg))
            elif n in Step.FP8:
                w, t = (self.w_pg if n == "paged_fp8" else self.w_lg), self.tokens[n]
                # one byte per cached K/V element
                out[n] = (decode_flops(w.Hq, 128, t),
                          decode_bytes(w.B, w.Hq, w.Hkv, 128, t) - 2.0 * t * w.Hkv * 128)
            else:
                out[n] = (decode_flops(self.w_ct.Hq, 128, self.w_ct.Skv),
                          decode_bytes(1, self.w_ct.Hq, self.w_ct.Hkv, 128, self.w_ct.Skv))
        return out


# ----------------------------------------------------------- rank plumbing
def sync_ranks(world: int) -> None:
    """Barrier over all ranks (a no-op for one process)."""
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest value any rank holds: every rank gets the same answer.  The
    tensor lives on `device` (CUDA for NCCL, CPU for gloo)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, steps: int, total_ms: float) -> float:
    """Whole-job steps per second: every rank ran `steps` steps, and the job
    took as long as its slowest rank (`total_ms`, max over ranks)."""
    return world * steps / (total_ms * 1e-3)


def run_ours(args, rank, world, local_rank):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    st = Step(device, args.calls)
    names = st.NAMES
    # Everything runs on one dedicated stream; the step and each call are
    # captured once as CUDA graphs, so the device time measured is the
    # kernels' and not the host's launch overhead.
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            for n in names:
                st.call(n)
    torch.cuda.synchronize(device)
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        for n in names:
            st.call(n)
    # Per-call timing graphs: R x (L2 flush, call) and R x (L2 flush) alone;
    # a call's device time is the difference divided by R, so neither the
    # graph launch nor the flush is counted.  The flush writes a buffer of
    # twice the L2 size, then reads another one: the write evicts the call's
    # inputs, the read evicts the written lines, so their write-back to HBM
    # happens inside the flush and is not charged to the call.
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush_w = torch.empty(max(2 * l2, 1 << 20) // 4, dtype=torch.float32, device=device)
    flush_r = torch.ones(max(2 * l2, 1 << 20) // 4, dtype=torch.float32, device=device)
    flush_acc = torch.empty((), dtype=torch.float32, device=device)

    def flush():
        flush_w.fill_(1.0)
        torch.sum(flush_r, dim=0, out=flush_acc)

    R = 20
    g_flush = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_flush, stream=stream):
        for _ in range(R):
            flush()
    g_call = {}
    for n in names:
        g_call[n] = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_call[n], stream=stream):
            for _ in range(R):
                flush()
                st.call(n)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g_step.replay()
    torch.cuda.synchronize(device)

    sync_ranks(world)
    torch.cuda.synchronize(device)
    # The clock sampler (nvidia-smi, one sample per 100 ms) runs through a
    # pre-roll of untimed step replays lasting PREROLL_S seconds and then
    # through the K timed steps, which alone are too short to be sampled.
    sampler = ClockSampler(device.index if device.index is not None else 0)
    preroll = 0
    with sampler, torch.cuda.stream(stream):
        t_end = time.perf_counter() + PREROLL_S
        while time.perf_counter() < t_end:
            for _ in range(50):
                g_step.replay()
            preroll += 50
            torch.cuda.synchronize(device)
        sync_ranks(world)
        torch.cuda.synchronize(device)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(args.steps):
            g_step.replay()
        end.record(stream)
        torch.cuda.synchronize(device)
    sync_ranks(world)
    total_ms = max_over_ranks(start.elapsed_time(end), world, device)
    ms_per_step = total_ms / args.steps

    # per-call device time, each call starting with a flushed L2
    def graph_ms(g, reps=5):
        ts = []
        with torch.cuda.stream(stream):
            g.replay()
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                ts.append((a, b))
            torch.cuda.synchronize(device)
        return float(np.median([a.elapsed_time(b) for a, b in ts]))

    t_flush = graph_ms(g_flush)
    per_call_ms = {n: max(graph_ms(g_call[n]) - t_flush, 1e-6) / R for n in names}
    # the tiny call once more as a host program makes it: 200 eager calls
    # through the binding back to back (host marshalling and launch included)
    eager_us = None
    if "tiny" in names:
        with torch.cuda.stream(stream):
            for _ in range(20):
                st.call("tiny")
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(200):
                st.call("tiny")
            b.record(stream)
            torch.cuda.synchronize(device)
        eager_us = a.elapsed_time(b) / 200 * 1e3
    # the contiguous decode once more with its inputs left in L2: R calls back
    # to back, no flush (reported beside the flushed figure, labelled L2-hot)
    hot_ms = None
    if "contig" in names and not args.no_extras:
        g_hot = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_hot, stream=stream):
            for _ in range(R):
                st.call("contig")
        hot_ms = graph_ms(g_hot) / R
        del g_hot

    # ---- the FP8-cache decode on the two paged workloads (not part of the
    # step: the step is the configured workload), timed the same way
    extras = None
    if not args.no_extras:
        extras = run_fp8_extras(device, stream, flush, R, graph_ms, t_flush)
        extras.update(run_tile_extras(device, stream, flush, R, graph_ms, t_flush))

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        with torch.cuda.stream(stream):
            e2e = run_e2e(st, args, device)
        # whole job, as long as its slowest rank (every rank takes this step);
        # the byte counts are per step of one rank
        ms = max_over_ranks(e2e["ms_per_step"], world, device)
        e2e["ms_per_step"] = round(ms, 3)
        e2e["value"] = round(job_rate(world, 1, ms), 3)
    del g_step, g_call, g_flush

    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    work = st.work()
    calls = {}
    for n in names:
        fl, by = work[n]
        us = per_call_ms[n] * 1e3
        rec = {"us": round(us, 2), "tflops": round(fl / us * 1e-6, 1),
               "gbs": round(by / us * 1e-3, 1), "flop": fl, "bytes": by}
        if n in ("prefill", "tiny"):
            rec["bound"] = "tensor" if n == "prefill" else "latency"
            rec["frac"] = round(rec["tflops"] / peaks["bf16_tflops"], 4)
        else:
            rec["bound"] = "hbm"
            rec["frac"] = round(rec["gbs"] / peaks["hbm_gbs"], 4)
        if n == "tiny" and eager_us is not None:
            rec["eager"] = {"us": round(eager_us, 2),
                            "note": "200 eager calls back to back through the Python binding"}
        if n == "contig" and hot_ms is not None:
            rec["l2_hot"] = {"us": round(hot_ms * 1e3, 2),
                             "gbs": round(by / (hot_ms * 1e3) * 1e-3, 1),
                             "note": "inputs L2-resident: 20 calls back to back, no flush"}
        calls[n] = rec
    # The dominant kernel is the one with the largest share of a step: the
    # decode kernel serves three calls, the prefill kernel one.  A decode
    # call's time also holds its small merge kernel (timed together, so the
    # streaming kernel's fraction is if anything understated).
    kernel_of = {"tiny": "prefill_kernel<64>", "prefill": "prefill_kernel<128>",
                 "paged": "decode_splitkv_kernel<128>",
                 "long": "decode_splitkv_kernel<128>",
                 "contig": "decode_splitkv_kernel<128> (cluster mode)",
                 "paged_fp8": "decode_splitkv_kernel<128> (e4m3 cache)",
                 "long_fp8": "decode_splitkv_kernel<128> (e4m3 cache)"}
    per_kernel = {}
    for n in names:
        k = kernel_of[n]
        t, fl, by, cnt = per_kernel.get(k, (0.0, 0.0, 0.0, 0))
        per_kernel[k] = (t + per_call_ms[n], fl + work[n][0], by + work[n][1], cnt + 1)
    dom = max(per_kernel, key=lambda k: per_kernel[k][0])
    t_ms, fl, by, cnt = per_kernel[dom]
    if dom.startswith("prefill"):
        roof = {"bound": "tensor", "achieved": round(fl / (t_ms * 1e-3) * 1e-12, 1),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": round(by / (t_ms * 1e-3) * 1e-9, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    roof["kernel"] = dom
    roof["launches_per_step"] = cnt
    roof["avg_launch_us"] = round(t_ms * 1e3 / cnt, 2)
    roof["peak_source"] = f"{peak_src} (burst figure: each kernel runs < 1 ms)"
    tr = profiled_traffic()
    dom_calls = [n for n in names if kernel_of[n] == dom]
    roof["traffic"] = (round(sum(tr[n] for n in dom_calls) / len(dom_calls))
                       if tr and all(n in tr for n in dom_calls) else None)
    roof["traffic_unit"] = "bytes per launch (ncu dram read + write, profiles/)"
    roof["algorithmic_bytes_per_launch"] = round(by / cnt)
    roof["share_of_step"] = round(t_ms / sum(v[0] for v in per_kernel.values()), 3)

    cpu = None   # the oracle on the host cores: rank 0 of a one-GPU run only
    if not args.no_cpu_baseline and world == 1 and tuple(names) == Step.ALL:
        cpu = cpu_baseline(st)
    line = {
        "metric": METRIC,
        "value": round(job_rate(world, args.steps, total_ms), 2),
        "unit": "step/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V, shuffled page tables)",
        "config": {"workload": WORKLOAD, "global_batch": None, "seq_len": 4096,
                   "parallelism": f"replicas x{world}",
                   "timing": "step = one CUDA graph of the five calls, replayed K times; "
                             "per-call times: a graph of 20 x (L2 flush, call) minus a "
                             "graph of 20 flushes, divided by 20",
                   "l2": "step working set ~0.9 GB > 126 MB L2 and every call's inputs are "
                         "evicted by the calls before it; per-call timings flush L2 "
                         "before each call (2x L2 size written, then another 2x L2 "
                         "read so the written lines are clean)"},
        "calls": calls,
        "extras": extras,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": sum(Step.LAUNCHES[n] for n in names) * args.steps * world,   # all ranks
        "clocks": dict(sampler.summary(), window=(
            f"{PREROLL_S:.1f} s of untimed step replays ({preroll} steps) immediately before "
            f"the timed region, and the timed region")),
    }
    return line


def run_fp8_extras(device, stream, flush, R, graph_ms, t_flush):
    """Per-call µs and GB/s of frt_attn_decode_paged_fp8 on the paged B4 and
    256k workloads with the cache stored as e4m3 (per-KV-head scales); L2
    flushed before each call as for the step's calls."""
    from flash_attention_tiled_b200 import frt
    peaks, _ = load_peaks()
    res = {}
    for name, wname in (("paged_fp8", "paged_gqa_decode_b4"), ("long_fp8", "long_splitkv_decode_256k")):
        w = inputs.WORKLOADS[wname]
        x = inputs.paged_fp8(w.B, w.Hq, w.Hkv, w.D, len_range=w.len_range, page_size=w.page_size,
                             seed=w.seed)
        d = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        o = torch.empty_like(d["q"])
        lse = torch.empty((w.B, w.Hq), device=device)

        def call():
            frt.attn_decode_paged_fp8(d["q"], d["k_pages"], d["v_pages"], d["k_scale"],
                                      d["v_scale"], d["block_table"], d["seq_lens"],
                                      scale=w.scale, out=o, lse=lse)

        with torch.cuda.stream(stream):
            for _ in range(3):
                call()
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(R):
                flush()
                call()
        us = max(graph_ms(g) - t_flush, 1e-6) / R * 1e3
        tokens = int(x["seq_lens"].sum())
        # one byte per cached K/V element, plus q, o and lse
        nbytes = 2.0 * tokens * w.Hkv * w.D + w.B * w.Hq * w.D * 2 * 2 + w.B * w.Hq * 4
        gbs = nbytes / us * 1e-3
        res[name] = {"us": round(us, 2), "gbs": round(gbs, 1), "bytes": nbytes, "bound": "hbm",
                     "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "cache": "e4m3 codes, per-KV-head fp32 scale", "workload": wname}
        del g, d, x
        torch.cuda.empty_cache()
    return res


def run_tile_extras(device, stream, flush, R, graph_ms, t_flush):
    """Per-call µs and TFLOP/s of the tile kernel on two more shapes: cross
    attention (1024 queries over 4096 keys, non-causal, GQA 32/8, D 128) and
    the Llama-3-8B causal prefill read through views of a fused
    [B, S, Hq + 2 Hkv, D] projection output (frt_attn_fwd_strided)."""
    from flash_attention_tiled_b200 import frt
    peaks, _ = load_peaks()
    gen = torch.Generator("cpu").manual_seed(2024)
    res = {}
    w = inputs.WORKLOADS["llama3_8b_prefill_4k"]
    cases = []
    # cross attention: contiguous [B,H,S,D] tensors
    Sq, Skv = 1024, 4096
    q = torch.randn(1, 32, Sq, 128, generator=gen).to(torch.bfloat16).to(device)
    k = torch.randn(1, 8, Skv, 128, generator=gen).to(torch.bfloat16).to(device)
    v = torch.randn(1, 8, Skv, 128, generator=gen).to(torch.bfloat16).to(device)
    o = torch.empty_like(q)
    lse = torch.empty((1, 32, Sq), device=device)
    cases.append(("cross_attn", lambda: frt.attn_fwd(q, k, v, causal=False, out=o, lse=lse),
                  4.0 * 128 * Sq * Skv * 32, "B1 Hq32 Hkv8 Sq1024 Skv4096 D128, non-causal"))
    # the Llama-3-8B prefill from a fused projection output
    x = torch.randn(w.B, w.Sq, w.Hq + 2 * w.Hkv, w.D, generator=gen).to(torch.bfloat16).to(device)
    qs = x[:, :, :w.Hq].permute(0, 2, 1, 3)
    ks = x[:, :, w.Hq:w.Hq + w.Hkv].permute(0, 2, 1, 3)
    vs = x[:, :, w.Hq + w.Hkv:].permute(0, 2, 1, 3)
    os_ = torch.empty(w.B, w.Sq, w.Hq, w.D, dtype=torch.bfloat16, device=device).permute(0, 2, 1, 3)
    lse2 = torch.empty((w.B, w.Hq, w.Sq), device=device)
    cases.append(("prefill_strided",
                  lambda: frt.attn_fwd_strided(qs, ks, vs, causal=True, scale=w.scale, out=os_,
                                               lse=lse2),
                  prefill_flops(w), "Llama-3-8B causal 4k, Q/K/V/O as views of [B,S,H,D] buffers"))
    for name, call, flop, desc in cases:
        with torch.cuda.stream(stream):
            for _ in range(3):
                call()
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(R):
                flush()
                call()
        us = max(graph_ms(g) - t_flush, 1e-6) / R * 1e3
        tf = flop / us * 1e-6
        res[name] = {"us": round(us, 2), "tflops": round(tf, 1), "flop": flop, "bound": "tensor",
                     "frac": round(tf / peaks["bf16_tflops"], 4), "workload": desc}
        del g
    return res


def run_e2e(st: Step, args, device):
    """Same step through the public API with pinned host inputs: H2D copy of
    every call's inputs, the call, and a D2H read of its outputs, per step."""
    names = st.NAMES
    host = {n: {k: (t.pin_memory() if isinstance(t, torch.Tensor) else t)
                for k, t in st.host[n].items()} for n in names}
    outs_h = {n: tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in st.out[n])
              for n in names}
    scratch = {n: {k: torch.empty_like(t) if isinstance(t, torch.Tensor) else t
                   for k, t in st.d[n].items()} for n in names}
    h2d = sum(t.numel() * t.element_size() for n in names for t in host[n].values()
              if isinstance(t, torch.Tensor))
    d2h = sum(t.numel() * t.element_size() for n in names for t in outs_h[n])
    stream = torch.cuda.current_stream(device)
    steps = max(1, min(args.steps, 10))

    def one():
        for n in names:
            for k, t in host[n].items():
                if isinstance(t, torch.Tensor):
                    scratch[n][k].copy_(t, non_blocking=True)
            st.call(n, d=scratch[n])
            for h, dv in zip(outs_h[n], st.out[n]):
                h.copy_(dv, non_blocking=True)

    one()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        one()
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / steps
    return {"value": round(1e3 / ms, 3), "unit": "step/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 3), "steps": steps}


# ------------------------------------------------------------- oracle arm
def cpu_baseline(st: Step | None, host=None):
    """One full step of the oracle on the host cores: every call of the step
    at its full size (the fp64 oracle as it stands, OpenMP over its
    (sequence, head) rows), timed by wall clock."""
    import oracle
    W = inputs.WORKLOADS
    if host is None:
        host = st.host
    legs = {}
    t0 = time.perf_counter()
    for key, name in (("tiny", "tiny_causal"), ("prefill", "llama3_8b_prefill_4k"),
                      ("contig", "gqa_decode_4k")):
        w, x = W[name], host[key]
        ts = time.perf_counter()
        oracle.attn_fwd(x["q"], x["k"], x["v"], w.causal, w.scale)
        legs[key] = time.perf_counter() - ts
    for key, name in (("paged", "paged_gqa_decode_b4"), ("long", "long_splitkv_decode_256k")):
        w, x = W[name], host[key]
        ts = time.perf_counter()
        oracle.attn_decode_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"],
                                 x["seq_lens"], w.scale)
        legs[key] = time.perf_counter() - ts
    total = time.perf_counter() - t0
    return {"value": round(1.0 / total, 6), "unit": "step/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": "one full step: all five calls at full size, nothing extrapolated",
            "s_per_step": round(total, 3),
            "s_per_call": {k: round(v, 4) for k, v in legs.items()}}


def reference_plan(steps: int, warmup: int):
    """(timed, untimed) oracle steps of the reference arm: the GPU arm's K and W
    when they fit the planned length, else as many timed steps as fit."""
    budget = max(1, int(REF_BUDGET_S // REF_STEP_S_EST))
    timed = max(1, min(steps, budget))
    return timed, max(0, min(warmup, budget - timed))


def reference_host_inputs():
    return {"tiny": inputs.make("tiny_causal"), "prefill": inputs.make("llama3_8b_prefill_4k"),
            "paged": inputs.make("paged_gqa_decode_b4"),
            "long": inputs.make("long_splitkv_decode_256k"), "contig": inputs.make("gqa_decode_4k")}


def run_reference(args, rank):
    if rank != 0:
        return None
    host = reference_host_inputs()
    for _ in range(args.warmup_ref):
        cpu_baseline(None, host=host)
    vals = [cpu_baseline(None, host=host) for _ in range(args.steps_ref)]
    s_per_step = float(np.mean([v["s_per_step"] for v in vals]))
    cb = vals[-1]
    value = round(1.0 / s_per_step, 6)
    cb["value"] = value
    cb["s_per_step"] = round(s_per_step, 3)
    return {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "step/s", "n_gpus": 1,
        "steps": args.steps_ref, "warmup": args.warmup_ref,
        "ms_per_step": round(s_per_step * 1e3, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V, shuffled page tables)",
        "config": {"workload": WORKLOAD, "global_batch": None, "seq_len": 4096,
                   "parallelism": "host cores (OpenMP)",
                   "timing": "wall clock around each full oracle step"},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "step/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the FP8-cache decode, cross-attention and strided-prefill "
                         "measurements")
    ap.add_argument("--calls", default=",".join(Step.ALL),
                    help="comma-separated subset of the step's calls (profiling runs)")
    args = ap.parse_args()
    args.calls = tuple(c for c in args.calls.split(",") if c)
    if not set(args.calls) <= set(Step.ALL + Step.FP8):
        ap.error(f"--calls must be a subset of {Step.ALL + Step.FP8}")
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # every step is one full oracle pass (~5 s on 16 host cores): K timed
        # steps after W untimed ones, as many as the GPU arm runs, unless that
        # would take more than ~4 minutes (the default K of 2000 would)
        args.steps_ref, args.warmup_ref = reference_plan(args.steps, args.warmup)
        line = run_reference(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120),
            device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
