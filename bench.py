#!/usr/bin/env python
"""Benchmark of the per-rank context-parallel attention hot path on B200.

One step = one pass of the Ulysses path over the S=44160 video-latent workload:
P=8 virtual ranks x [5520 tokens][16 heads][128] bf16 Q/K/V shards in, non-causal
attention over 8 head groups x 2 heads x S=44160 x D=128, O shards + LSE out.  Two step
variants of the same work are timed: `fused` (the default headline: one tcgen05 kernel
whose addressing does the re-partitions) and `plain` (3 seq2head permutes -> attention ->
head2seq).  The metric is attention TFLOPS (4*B*H*S^2*D per step) over the whole step;
the attention kernel's own roofline, the permutes' and the (O, LSE) merge's HBM rooflines,
the other workloads' attention and an end-to-end number through host buffers are
reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--step fused|plain] [--qk-norm] [--profile] [--no-cpu-baseline]

Under torchrun (N > 1) every rank runs its own replica (weak scaling, no data-path
collective); the timed region is bracketed by barriers and the max over ranks is used.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from context_long_sequence_non_b200 import workloads as W  # noqa: E402

METRIC = "non-causal bf16 attention TFLOPS at S=44160 on 1 B200; % of dense BF16 peak"
UNIT = "TFLOP/s"
WORKLOAD = W.WORKLOADS[4]
# DRAM bytes (read + write) per launch of each attention kernel on this workload, from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the kernel and by the
# SHA-256 of the kernel sources the capture was taken with, comments and whitespace removed
# (an edit to either leaves the kernel as it was).  When the code hashes to something else
# the figure no longer describes the kernel that runs, and the line reports traffic null
# until a new capture is recorded here.
ATTN_SOURCES = ("context_long_sequence_non_b200/csrc/attn_sm100.cu",
                "context_long_sequence_non_b200/csrc/sm100_ptx.cuh",
                "context_long_sequence_non_b200/csrc/tail_plan.cu")  # the launch's work split
ATTN_TRAFFIC = {
    "attn_fwd_sm100_kernel<128,0,2>": {  # the fused Ulysses kernel (tail-split launch)
        "sources_sha256": "69c968bdd07bfb40a30b821b95feb7d06a3b168ef5b06bc8e2d4e4c379fca5b3",
        "bytes": 590_219_264 + 182_754_048,
    },
    "attn_fwd_sm100_kernel<128,0,0>": {  # the plain form, in the 5-launch step
        "sources_sha256": "69c968bdd07bfb40a30b821b95feb7d06a3b168ef5b06bc8e2d4e4c379fca5b3",
        "bytes": 584_683_520 + 167_802_880,
    },
}
AUX_REPS = 15  # bursts per auxiliary measurement (median reported, with the range)
AUX_IDLE_S = 1.0  # idle between the timed steps and the auxiliary measurements
L2_NOTE = ("inputs larger than L2: each step streams 543 MB of Q/K/V shards plus 724 MB of "
           "permute traffic through the 126 MB L2")


def code_only(text):
    """C/C++/CUDA source with its comments and all whitespace removed."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return re.sub(r"\s+", "", text)


def attn_sources_sha256():
    import hashlib

    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(code_only(f.read()).encode())
    return h.hexdigest()


def attn_traffic(kernel):
    """ncu DRAM bytes per launch for ``kernel``, or None when no capture matches its
    current sources."""
    rec = ATTN_TRAFFIC.get(kernel)
    if rec is None or rec["sources_sha256"] != attn_sources_sha256():
        return None
    return rec["bytes"]


def workload_config(qk_norm=False, step="fused"):
    w = WORKLOAD
    if step == "fused":
        return {
            "workload": ("ulysses-cp8-s44160: P=8 virtual ranks x [5520 tokens][16 heads][128] "
                         "bf16 Q/K/V shards in, O shards + fp32 LSE out; the Ulysses re-partitions "
                         "(seq2head of Q/K/V, head2seq of O) done by the attention kernel's own "
                         "addressing (non-causal attention over 8 head groups x 2 heads, "
                         "S=44160, D=128, fp32 accumulate, bf16 O); the 104 work items of the "
                         "kernel's last, partial wave run as 4 key ranges each, folded by a "
                         "combine kernel (2 launches per step); equal to rounding to the 3x "
                         "seq2head + attention + head2seq launches"),
            "B": w.B, "H": w.H, "S": w.Sq, "D": w.D, "P": w.P, "step": "fused",
            "inputs": "iid N(0,1), torch.Generator seed 4000, rounded to bf16",
            "l2": L2_NOTE,
        }
    if qk_norm:
        return {
            "workload": ("ulysses-cp8-s44160 with Q/K RMSNorm: P=8 virtual ranks x [5520 tokens]"
                         "[16 heads][128] bf16 Q/K/V, one seq2head launch for Q/K/V with the "
                         "RMSNorm of every Q and K head row fused in (eps 1e-6, float32 weights) + "
                         "non-causal attention + head2seq"),
            "B": w.B, "H": w.H, "S": w.Sq, "D": w.D, "P": w.P,
            "inputs": "iid N(0,1), torch.Generator seed 4000, rounded to bf16; weights 1+0.1 N(0,1)",
            "l2": L2_NOTE,
        }
    return {
        "workload": (f"ulysses-cp8-s44160: P=8 virtual ranks x [5520 tokens][16 heads][128] bf16 "
                     f"Q/K/V, 3x seq2head + non-causal attention (8 head groups x 2 heads, "
                     f"S=44160, D=128, fp32 accumulate, bf16 O + fp32 LSE) + head2seq"),
        "B": w.B, "H": w.H, "S": w.Sq, "D": w.D, "P": w.P, "step": "plain",
        "inputs": "iid N(0,1), torch.Generator seed 4000, rounded to bf16",
        "l2": L2_NOTE,
    }


# --------------------------------------------------------------------------- distributed


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_group(world, backend):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist

    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def aggregate(dist, elapsed_ms: float, units: float, device=None):
    """Max of the timed region over ranks and the sum of the work units of all ranks."""
    if dist is None:
        return elapsed_ms, units
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms during the timed region.

    nvidia-smi can take a second or more to print its first sample, so its output is read
    on a thread and ``start`` returns only once the first sample has arrived (or after
    ``wait_s``): the timed region that follows is then covered from its first moment."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path: str | None = None):
        self.gpu_index, self.proc, self.path = gpu_index, None, path
        self.lines, self.reader = [], None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def start(self, wait_s: float = 10.0):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < wait_s and self.proc.poll() is None:
            time.sleep(0.02)

    def stop(self, t_begin: float | None = None, t_end: float | None = None):
        """Stop sampling; summarise the samples taken inside [t_begin, t_end] (epoch s), or
        the ones nearest to it (within 1 s) when the region was too short to catch one."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)  # one more sample after the region
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
            self.proc.wait()
        if self.reader is not None:
            self.reader.join(timeout=5)
        out = "".join(self.lines)
        if self.path:
            with open(self.path, "w") as f:
                f.write(out)
        import datetime

        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        parsed = []
        for r in (r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8):
            try:
                ts = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
                parsed.append((ts, float(r[1]), float(r[2]), float(r[3]),
                               [n for n, val in zip(names, r[5:9])
                                if val.strip().lower() == "active"]))
            except ValueError:
                continue
        window = "samples inside the timed region"
        chosen = parsed
        if t_begin is not None:
            chosen = [x for x in parsed if t_begin <= x[0] <= t_end]
            if not chosen:
                chosen = [x for x in parsed if t_begin - 1.0 <= x[0] <= t_end + 1.0]
                window = "samples within 1 s of the timed region (none inside it)"
        sm = [x[1] for x in chosen]
        reasons = sorted({n for x in chosen for n in x[4]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": chosen[-1][2] if chosen else None,
                "sm_mhz_min": min(sm) if sm else None, "reasons": reasons,
                "samples": len(sm), "power_w_max": max(x[3] for x in chosen) if chosen else None,
                "window": window}


# --------------------------------------------------------------------------- peaks


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# --------------------------------------------------------------------------- our arm


def run_ours(args, world, rank, local):
    import context_long_sequence_non_b200 as cp
    from context_long_sequence_non_b200 import _binding as Bd
    from context_long_sequence_non_b200.paths import UlyssesPlan

    torch.cuda.set_device(local)
    dist = init_group(world, "nccl")
    dev = torch.device("cuda", local)
    w = WORKLOAD
    P, S_l, H = w.P, w.Sq // w.P, w.H * w.P
    x = W.make_inputs(w)
    global _INPUTS
    _INPUTS = x
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    plan = UlyssesPlan(P, S_l, H, w.D, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = w.attn_flops
    if args.qk_norm:  # the sample's Q/K RMSNorm fused into one Q/K/V seq2head launch
        gq = W.norm_weights(w.D, seed=41).to(dev)
        gk = W.norm_weights(w.D, seed=42).to(dev)

    def plain_step(ev_attn=None):
        if args.qk_norm:
            cp.seq2head_qkv_norm(q, k, v, P, gq, gk, out=(plan.qh, plan.kh, plan.vh))
        else:
            cp.seq2head(q, P, out=plan.qh)
            cp.seq2head(k, P, out=plan.kh)
            cp.seq2head(v, P, out=plan.vh)
        if ev_attn is not None:
            ev_attn[0].record(stream)
        cp.fwd(plan.qh, plan.kh, plan.vh, out=plan.oh, lse=plan.lse, scale=w.softmax_scale)
        if ev_attn is not None:
            ev_attn[1].record(stream)
        cp.head2seq(plan.oh, P, out=plan.out)

    # the fused pass's tail split: the work items of the last wave run as key ranges whose
    # fp32 partials a combine kernel folds (workspace allocated once, outside the timing)
    ws_bytes = cp.ulysses_workspace_bytes(P, S_l, H, w.D)
    ws_u = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    def fused_step(ev_attn=None):
        # sharded Q/K/V in, sharded O + LSE out: the work of plain_step (equal to rounding),
        # the re-partitions done by the attention kernel's addressing
        if ev_attn is not None:
            ev_attn[0].record(stream)
        cp.ulysses_fwd_split(q, k, v, P, out=plan.out, lse=plan.lse, scale=w.softmax_scale,
                             workspace=ws_u)
        if ev_attn is not None:
            ev_attn[1].record(stream)

    def timed_steps(step, tag):
        """W untimed warm-up steps, then exactly K timed steps bracketed by a barrier and a
        device synchronize on both sides; CUDA events on the launching stream around the
        whole region and around each attention launch; clocks sampled during it."""
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        if Bd.device_error() != 0:
            raise RuntimeError(f"bounded wait ran out during the {tag} warm-up")
        path = (args.clocks_csv.replace("{rank}", str(rank)).replace("{step}", tag)
                if args.clocks_csv else None)
        clocks = ClockSampler(local, path)
        attn_events = [(torch.cuda.Event(enable_timing=True),
                        torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        clocks.start()  # returns once nvidia-smi is reporting
        wall0 = time.time()
        t0.record(stream)
        for i in range(args.steps):
            step(attn_events[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        wall1 = time.time()
        clk = clocks.stop(wall0, wall1)
        if dist is not None:
            dist.barrier()
        elapsed_ms = t0.elapsed_time(t1)
        attn_ms = statistics.mean(a.elapsed_time(b) for a, b in attn_events)
        if Bd.device_error() != 0:
            raise RuntimeError(f"bounded wait ran out during the {tag} timed region")
        max_ms, total_flops = aggregate(dist, elapsed_ms, flops * args.steps,
                                        device=dev if dist is not None else None)
        return max_ms, total_flops, attn_ms, clk

    peaks = measured_peaks()
    variants = {
        "fused": (fused_step, 2 if ws_bytes > 0 else 1, "attn_fwd_sm100_kernel<128,0,2>",
                  "cpattn_ulysses_fwd_split: one attention kernel (sharded Q/K/V in, sharded "
                  "O + LSE out) whose last wave's items run as key ranges, and the combine of "
                  "their partials"),
        "plain": (plain_step, 3 if args.qk_norm else 5, "attn_fwd_sm100_kernel<128,0,0>",
                  ("seq2head_qkv_norm + cpattn_fwd + head2seq" if args.qk_norm else
                   "3x cpattn_seq2head + cpattn_fwd + cpattn_head2seq")),
    }
    head = "plain" if args.qk_norm else args.step
    # profiler runs time the headline variant only, so a launch list holds one step kind
    order = [head] + [n for n in variants
                      if n != head and not args.qk_norm and not args.profile]
    results = {}
    for name in order:
        fn, launches, kernel, what = variants[name]
        max_ms, total_flops, attn_ms, clk = timed_steps(fn, name)
        value = total_flops / (max_ms * 1e-3) / 1e12
        results[name] = {"value": round(value, 2), "unit": UNIT,
                         "ms_per_step": round(max_ms / args.steps, 4),
                         "attn_kernel": kernel, "attn_ms": round(attn_ms, 4),
                         "attn_TFLOP/s": round(flops / (attn_ms * 1e-3) / 1e12, 2),
                         "gpu_launches": launches * args.steps, "what": what, "clocks": clk,
                         "_raw": (max_ms, total_flops, attn_ms)}

    if args.profile:  # profiler runs: the timed steps only, nothing else launched
        aux, e2e = None, None
    else:
        # ---- auxiliary kernels, each timed alone (L2 flushed before each burst), after a
        # short idle so that they do not inherit the power-capped clock of the loop above
        time.sleep(AUX_IDLE_S)
        aux_clocks = ClockSampler(local, None)
        aux_clocks.start()
        wall_a0 = time.time()
        aux = aux_kernels(cp, w, q, plan, dev, stream)
        aux["next"] = next_paths(cp, w, q, k, v, plan, dev, stream)
        aux["clocks"] = aux_clocks.stop(wall_a0, time.time())
        aux["idle_before_s"] = AUX_IDLE_S
        # ---- end to end through the public API with host buffers
        e2e = e2e_run(cp, UlyssesPlan, w, x, dev, stream, args, dist=dist, world=world)

    hr = results[head]
    max_ms, total_flops, attn_ms = hr.pop("_raw")
    for r in results.values():
        r.pop("_raw", None)
    value = total_flops / (max_ms * 1e-3) / 1e12
    achieved = flops / (attn_ms * 1e-3) / 1e12
    long_run = max_ms > 1000.0
    peak = peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]
    kernel = hr["attn_kernel"]
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(max_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(args.qk_norm, head),
        "frac_of_dense_bf16_peak": round(value / peak, 4),
        "roofline": {
            "bound": "tensor", "kernel": kernel,
            "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "peak_kind": (f"{peaks['source']} cuBLAS bf16 "
                          f"{'sustained' if long_run else 'burst'}"),
            "algorithmic_flops_per_launch": flops,
            "avg_launch_ms": round(attn_ms, 4),
            "timed": ("the cpattn_ulysses_fwd_split call: the attention kernel and the combine "
                      "of its split items' partials, so `achieved` slightly understates the "
                      "kernel alone" if head == "fused" else "the attention kernel alone"),
            "traffic": attn_traffic(kernel),
            "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
            "traffic_source": ("ncu capture of this kernel, recorded with the SHA-256 of its "
                               "sources; null when the sources have changed since"),
            "sources_sha256": attn_sources_sha256(),
            # Q, K, V read once and O written once (four equal bf16 tensors) + fp32 LSE
            "algorithmic_bytes_per_launch": 4 * q.numel() * q.element_size()
            + plan.lse.numel() * 4,
        },
        "step_variants": results,
        "aux": aux,
        "e2e": e2e,
        "gpu_launches": hr["gpu_launches"],
        "clocks": hr["clocks"],
    }
    if rank == 0 and world == 1 and not (args.no_cpu_baseline or args.profile):
        line["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def flush_l2(buf):
    """Evict L2: write a buffer 4x the 126 MB L2, then read it back, so the timed kernel
    starts with a cold, clean L2 (no dirty lines of the flush left to write back)."""
    buf.zero_()
    buf.sum(dtype=torch.int32)


def aux_kernels(cp, w, q, plan, dev, stream):
    """seq2head / head2seq / merge alone: achieved HBM GB/s (bytes read + written once).

    Each kernel is timed as a burst of back-to-back launches on distinct buffers (as in
    the step: three seq2heads in a row; a ring step's seven merges in a row), after an L2
    flush, and reported per launch; the burst's buffers exceed L2 so every launch streams
    from HBM.
    """
    peaks = measured_peaks()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)  # 4x the 126 MB L2
    out = {}

    spread = {}

    def timed(fns, reps=AUX_REPS):
        ts = []
        for _ in range(reps):
            flush_l2(flush)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for fn in fns:
                fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b) / len(fns))
        spread["last"] = (min(ts), max(ts))
        return statistics.median(ts)

    def entry(ms, nbytes, **kw):
        gbs = nbytes / ms / 1e6
        lo, hi = spread["last"]
        return {"ms": round(ms, 4), "bytes": nbytes, "GB/s": round(gbs, 1),
                "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
                "frac_range": [round(nbytes / hi / 1e6 / peaks["hbm_gbs"], 4),
                               round(nbytes / lo / 1e6 / peaks["hbm_gbs"], 4)],
                "reps": AUX_REPS, **kw}

    P = w.P
    tensor_bytes = q.numel() * q.element_size()
    extra = [torch.empty_like(q) for _ in range(2)]
    srcs = [q] + extra
    dsts = [plan.qh, plan.kh, plan.vh]
    ms = timed([lambda s_=s_, d_=d_: cp.seq2head(s_, P, out=d_) for s_, d_ in zip(srcs, dsts)])
    out["seq2head"] = entry(ms, 2 * tensor_bytes, burst=3)
    outs = [plan.out] + extra
    ms = timed([lambda s_=s_, d_=d_: cp.head2seq(s_, P, out=d_)
                for s_, d_ in zip([plan.qh, plan.kh, plan.vh], outs)])
    out["head2seq"] = entry(ms, 2 * tensor_bytes, burst=3)
    del extra
    # ring-step merges on one rank's partials: [5520][16][128] bf16 + LSE [16][5520], 7 in a row
    S, Hm, D = 5520, 16, 128
    g = torch.Generator(device="cpu").manual_seed(31)
    sets = []
    for _ in range(7):
        oa = torch.randn(1, S, Hm, D, generator=g).to(torch.bfloat16).to(dev)
        ob = torch.randn(1, S, Hm, D, generator=g).to(torch.bfloat16).to(dev)
        la = torch.randn(1, Hm, S, generator=g).to(dev)
        lb = torch.randn(1, Hm, S, generator=g).to(dev)
        sets.append((oa, la, ob, lb, torch.empty_like(oa), torch.empty_like(la)))
    ms = timed([lambda t=t: cp.merge(t[0], t[1], t[2], t[3], out=t[4], lse=t[5]) for t in sets])
    oa, la = sets[0][0], sets[0][1]
    mbytes = 3 * oa.numel() * 2 + 3 * la.numel() * 4
    out["merge"] = entry(ms, mbytes, burst=7,
                         shape="[1][5520][16][128] bf16 x3 + LSE [1][16][5520] f32 x3")
    out["hbm_peak_gbs"] = peaks["hbm_gbs"]
    out["l2"] = ("512 MB buffer written then read before each burst; each burst's buffers "
                 "exceed L2")
    out["timing"] = (f"median of {AUX_REPS} bursts, each timed with CUDA events and reported "
                     f"per launch; frac_range = the slowest and fastest burst")
    return out


def next_paths(cp, w, q, k, v, plan, dev, stream):
    """The fused forms of the path, timed alone after an L2 flush (median of 5):
    Ulysses in one kernel, the batched Q/K/V seq2head, and one rank's Ring Attention step
    (Q slice of 5520 tokens over 8 K/V chunks of 5520, 16 heads) with the merge fused into
    the attention epilogue versus separate partials + merge kernel."""
    peaks = measured_peaks()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def timed(fn, reps=AUX_REPS):
        ts = []
        for _ in range(reps):
            flush_l2(flush)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    res = {}
    # the bandwidth kernels first, right after the idle, before the attention entries heat
    # the GPU into its power cap (their issue-bound forms follow the SM clock)
    ms = timed(lambda: cp.seq2head_qkv(q, k, v, w.P, out=(plan.qh, plan.kh, plan.vh)))
    nbytes = 3 * 2 * q.numel() * q.element_size()
    res["seq2head_qkv"] = {"ms": round(ms, 4), "bytes": nbytes,
                           "GB/s": round(nbytes / ms / 1e6, 1),
                           "frac_of_hbm": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 4)}
    # the sample's Q/K RMSNorm fused into that launch (same bytes), and standalone in place
    gq = W.norm_weights(w.D, seed=41).to(dev)
    gk = W.norm_weights(w.D, seed=42).to(dev)
    ms = timed(lambda: cp.seq2head_qkv_norm(q, k, v, w.P, gq, gk, out=(plan.qh, plan.kh, plan.vh)))
    res["seq2head_qkv_norm"] = {"ms": round(ms, 4), "bytes": nbytes,
                                "GB/s": round(nbytes / ms / 1e6, 1),
                                "frac_of_hbm": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 4),
                                "what": "seq2head of Q, K, V with RMSNorm of Q and K head rows"}
    qn = q.clone()
    nb1 = 2 * qn.numel() * qn.element_size()
    ms = timed(lambda: cp.rmsnorm(qn, gq, out=qn))
    res["rmsnorm"] = {"ms": round(ms, 4), "bytes": nb1, "GB/s": round(nb1 / ms / 1e6, 1),
                      "frac_of_hbm": round(nb1 / ms / 1e6 / peaks["hbm_gbs"], 4),
                      "what": "RMSNorm of [8][5520][16][128] bf16 head rows, in place"}
    del qn
    # the image-DiT joint sequence: B=1, H=24, S=4608 (4096 image + 512 text tokens), D=128
    w2 = W.WORKLOADS[2]
    x2 = W.make_inputs(w2)
    q2, k2, v2 = (x2[n].to(dev) for n in ("q", "k", "v"))
    ms2 = timed(lambda: cp.fwd(q2, k2, v2, scale=w2.softmax_scale))
    res["image_dit_4608"] = {"workload": "B1 H24 S4608 D128 bf16 (4096 image + 512 text tokens)",
                             "ms": round(ms2, 4), "TFLOP/s": round(w2.attn_flops / ms2 / 1e9, 2),
                             "frac_of_burst": round(w2.attn_flops / ms2 / 1e9 / peaks["bf16_tflops"], 4),
                             "ctas": 18 * 24, "waves_on_148_sms": round(18 * 24 / 148, 2)}
    del q2, k2, v2, x2
    # the long joint video + text sequence with large logits: B=1, H=16, S=47152, D=128,
    # Q/K ~ N(0, 9) (the softmax-stability stress case)
    w5 = W.WORKLOADS[5]
    x5 = W.make_inputs(w5)
    q5, k5, v5 = (x5[n].to(dev) for n in ("q", "k", "v"))
    ms5 = timed(lambda: cp.fwd(q5, k5, v5, scale=w5.softmax_scale), reps=5)
    res["video_text_47152_sigma3"] = {
        "workload": "B1 H16 S47152 D128 bf16, Q/K ~ N(0,9), V ~ N(0,1)", "ms": round(ms5, 4),
        "TFLOP/s": round(w5.attn_flops / ms5 / 1e9, 2),
        "frac_of_burst": round(w5.attn_flops / ms5 / 1e9 / peaks["bf16_tflops"], 4), "reps": 5}
    del q5, k5, v5, x5
    # the fused pass without and with its tail split, their launches alternating (measured
    # one after the other, the second would inherit the first's heat)
    ws_u = torch.empty(max(cp.ulysses_workspace_bytes(w.P, w.Sq // w.P, w.H * w.P, w.D), 256),
                       dtype=torch.uint8, device=dev)
    pair = (lambda: cp.ulysses_fwd(q, k, v, w.P, out=plan.out, lse=plan.lse),
            lambda: cp.ulysses_fwd_split(q, k, v, w.P, out=plan.out, lse=plan.lse,
                                         workspace=ws_u))
    ts = ([], [])
    for _ in range(AUX_REPS):
        for i_, fn in enumerate(pair):
            ts[i_].append(timed(fn, reps=1))
    ms, ms_s = statistics.median(ts[0]), statistics.median(ts[1])
    res["ulysses_fused"] = {"ms": round(ms, 4), "TFLOP/s": round(w.attn_flops / ms / 1e9, 2),
                            "what": ("seq2head x3 + attention + head2seq as one kernel "
                                     "(cpattn_ulysses_fwd, no tail split)")}
    res["ulysses_fused_split"] = {"ms": round(ms_s, 4),
                                  "TFLOP/s": round(w.attn_flops / ms_s / 1e9, 2),
                                  "what": ("the same with the tail split (cpattn_ulysses_fwd_split,"
                                           " the headline step's call); launches alternating "
                                           "with the unsplit one")}
    del ws_u
    w3 = W.WORKLOADS[3]
    x3 = W.make_inputs(w3)
    q3, k3, v3 = (x3[n].to(dev) for n in ("q", "k", "v"))
    bounds = [0]
    for c in x3["chunks"]:
        bounds.append(bounds[-1] + c)
    kc = [k3[:, a:b].contiguous() for a, b in zip(bounds, bounds[1:])]
    vc = [v3[:, a:b].contiguous() for a, b in zip(bounds, bounds[1:])]
    n_split = cp.split_suggest(1, w3.H, w3.Sq, x3["chunks"][0])
    ms_f = timed(lambda: cp.ring_attention(q3, kc, vc, scale=w3.softmax_scale, fused=True))
    ms_u = timed(lambda: cp.ring_attention(q3, kc, vc, scale=w3.softmax_scale, fused=False))
    ms_s = timed(lambda: cp.ring_attention(q3, kc, vc, scale=w3.softmax_scale, fused=True,
                                           n_split=n_split))
    ms_t = timed(lambda: cp.ring_attention(q3, kc, vc, scale=w3.softmax_scale, fused=True,
                                           n_split=0))
    # the same tail-split step recorded once into a CUDA graph and replayed, as a serving
    # loop runs it (no host work between its launches)
    ring_t = lambda: cp.ring_attention(q3, kc, vc, scale=w3.softmax_scale, fused=True, n_split=0)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        ring_t()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        ring_t()
    ms_g = timed(graph.replay)
    del graph
    # AllGather-KV-like: a short query slice (512 tokens, 16 heads) against all 44160 keys --
    # 32 CTAs for 148 SMs, the case split-KV is for
    g = torch.Generator(device="cpu").manual_seed(41)
    qs = W.randn((1, 512, 16, 128), g, 1.0, "bf16").to(dev)
    ks = k3.reshape(1, -1, 16, 128)[:, :44160].contiguous()
    vs = v3.reshape(1, -1, 16, 128)[:, :44160].contiguous()
    flops_s = 4.0 * 16 * 512 * 44160 * 128
    ns = cp.split_suggest(1, 16, 512, 44160)
    ms_1 = timed(lambda: cp.fwd(qs, ks, vs))
    ws = torch.empty(cp.split_workspace_bytes(1, 16, 512, 128, ns), dtype=torch.uint8, device=dev)
    ms_n = timed(lambda: cp.fwd_split(qs, ks, vs, n_split=ns, workspace=ws))
    res["split_kv_short_q"] = {"workload": "Q [1][512][16][128] over 44160 keys", "n_split": ns,
                               "single_ms": round(ms_1, 4),
                               "single_TFLOP/s": round(flops_s / ms_1 / 1e9, 2),
                               "split_ms": round(ms_n, 4),
                               "split_TFLOP/s": round(flops_s / ms_n / 1e9, 2)}
    res["ring_step"] = {
        "workload": "Q [1][5520][16][128] over 8 K/V chunks of 5520 tokens, bf16 accumulator",
        "fused_ms": round(ms_f, 4), "fused_TFLOP/s": round(w3.attn_flops / ms_f / 1e9, 2),
        "unfused_ms": round(ms_u, 4), "unfused_TFLOP/s": round(w3.attn_flops / ms_u / 1e9, 2),
        "split_kv": n_split, "split_ms": round(ms_s, 4),
        "split_TFLOP/s": round(w3.attn_flops / ms_s / 1e9, 2),
        "tail_split_ms": round(ms_t, 4), "tail_split_TFLOP/s": round(w3.attn_flops / ms_t / 1e9, 2),
        "tail_split_frac_of_burst": round(w3.attn_flops / ms_t / 1e9 / peaks["bf16_tflops"], 4),
        "tail_split": ("352 items on 148 SMs: 296 whole, the 56 of the last wave as 2 key "
                       "ranges each, folded into the accumulator by a combine kernel"),
        "tail_split_graph_ms": round(ms_g, 4),
        "tail_split_graph_TFLOP/s": round(w3.attn_flops / ms_g / 1e9, 2),
        "tail_split_graph_frac_of_burst": round(w3.attn_flops / ms_g / 1e9 / peaks["bf16_tflops"], 4),
        "launches_fused": 8, "launches_unfused": 15, "launches_split": 16,
        "launches_tail_split": 16}
    return res


def e2e_run(cp, UlyssesPlan, w, x, dev, stream, args, dist=None, world=1):
    """Same metric end to end with pinned host buffers: every step copies its Q/K/V shards
    host -> device and its O and LSE device -> host inside the timed region.

    The reported value goes through the C ABI's host-buffer call (cpattn_ulysses_host via
    ``UlyssesHostPass``): inside each call the head groups go in chunks, and the upload of
    one chunk and the download of another overlap the attention of a third.  Calls run
    back to back on one stream, each ordered after the previous one.  Also reported:
    ``streamer`` (``UlyssesStreamer``: whole steps overlapped with their neighbours' copies
    on three streams, as a serving loop would run them) and ``serial`` (copy in, compute,
    copy out, one step after another)."""
    from context_long_sequence_non_b200.paths import UlyssesHostPass, UlyssesStreamer

    P, S_l, H = w.P, w.Sq // w.P, w.H * w.P
    hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
    plan = UlyssesPlan(P, S_l, H, w.D, device=dev)
    ho = torch.empty(plan.out.shape, dtype=plan.out.dtype).pin_memory()
    hl = torch.empty(plan.lse.shape, dtype=plan.lse.dtype).pin_memory()
    n = max(3, min(args.steps, 10))
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()

    def timed(fn, start_stream=None, end_stream=None):
        for _ in range(2):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(start_stream or stream)
        for _ in range(n):
            fn()
        b.record(end_stream or stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / n

    tf = lambda ms: round(w.attn_flops / (ms * 1e-3) / 1e12, 2)

    # through the C ABI: host shards in, host O/LSE out, copies pipelined inside the call
    hp = UlyssesHostPass(P, S_l, H, w.D, device=dev)
    ms_single = timed(lambda: hp.run(hq, hk, hv, ho, hl, scale=w.softmax_scale))
    del hp
    # the same call double-buffered as a serving loop runs it: two passes (two device
    # buffer sets, two host output sets) alternate on two streams, so one step's first
    # upload and last download overlap its neighbours' attention
    hps = [UlyssesHostPass(P, S_l, H, w.D, device=dev) for _ in range(2)]
    houts = [(ho, hl), (torch.empty_like(ho).pin_memory(), torch.empty_like(hl).pin_memory())]
    strs = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    kk = [0]

    def host_step():
        i = kk[0] % 2
        strs[i].wait_stream(stream) if kk[0] < 2 else None
        hps[i].run(hq, hk, hv, *houts[i], scale=w.softmax_scale, stream=strs[i])
        kk[0] += 1

    def host_timed():
        for _ in range(2):
            host_step()
        torch.cuda.synchronize(dev)
        kk[0] = 0
        if dist is not None:  # every rank's timed region starts together
            dist.barrier()
            torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            host_step()
        for st in strs:
            stream.wait_stream(st)
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / n

    ms_host = host_timed()
    del hps
    # the whole job: the max of the ranks' timed regions, the work and copies of all ranks
    ms_all, flops_all = aggregate(dist, ms_host * n, w.attn_flops * n,
                                  device=dev if dist is not None else None)
    ms_job = ms_all / n

    dq, dk, dv = (torch.empty_like(hq, device=dev) for _ in range(3))

    def serial_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        plan.run(dq, dk, dv, scale=w.softmax_scale)
        ho.copy_(plan.out, non_blocking=True)
        hl.copy_(plan.lse, non_blocking=True)

    ms_serial = timed(serial_step)
    del plan, dq, dk, dv

    # whole steps overlapped: two host output sets so a step's download never races the next
    streamer = UlyssesStreamer(P, S_l, H, w.D, device=dev, depth=2)
    outs = [(ho, hl), (torch.empty_like(ho).pin_memory(), torch.empty_like(hl).pin_memory())]
    k = [0]

    def stream_step():
        streamer.submit(hq, hk, hv, *outs[k[0] % 2], scale=w.softmax_scale)
        k[0] += 1

    ms_streamer = timed(stream_step, streamer.upload, streamer.download)
    return {"value": round(flops_all / n / (ms_job * 1e-3) / 1e12, 2), "unit": UNIT,
            "ms_per_step": round(ms_job, 4), "n_gpus": world,
            "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world, "steps": n,
            "mode": ("C ABI cpattn_ulysses_host (UlyssesHostPass): pinned host Q/K/V shards in, "
                     "host O + LSE out; one chunk per head group (8), uploads and downloads "
                     "overlapping the attention inside each call; two passes alternating on "
                     "two streams (double-buffered serving loop)"),
            "per_rank": "single_stream, streamer and serial are this rank's own (rank 0)",
            "single_stream": {"value": tf(ms_single), "ms_per_step": round(ms_single, 4),
                              "mode": "the same call back to back on one stream"},
            "streamer": {"value": tf(ms_streamer), "ms_per_step": round(ms_streamer, 4),
                         "mode": "UlyssesStreamer: neighbouring steps' copies overlap compute "
                                 "(2 buffer sets, upload/compute/download streams)"},
            "serial": {"value": tf(ms_serial), "ms_per_step": round(ms_serial, 4),
                       "mode": "copy in, compute (5 launches), copy out, one step after another"}}


# --------------------------------------------------------------------------- CPU oracle


# Query rows per oracle sample, for the CPU baseline and the reference arm alike: about
# 128 rows per head, so each head's products are real matrix products (a handful of rows
# per head would time BLAS at matrix-vector efficiency and understate the oracle).
ORACLE_ROWS = 2048


def oracle_sample(n_rows, seed):
    """The fp64 oracle on ``n_rows`` sampled query rows of the Ulysses workload (each row
    attends over all 44160 keys of its head).  Returns (seconds, flops, cores)."""
    import oracle

    cores = oracle.set_threads()
    w = WORKLOAD
    x = _oracle_inputs()
    S_l, H = w.Sq // w.P, w.H * w.P
    full = lambda t: t.reshape(1, w.P * S_l, H, w.D)
    g = torch.Generator(device="cpu").manual_seed(seed)
    hs = torch.randint(0, H, (n_rows,), generator=g).tolist()
    ts = torch.randint(0, w.Sq, (n_rows,), generator=g).tolist()
    rows = [(0, h, t) for h, t in zip(hs, ts)]
    t = time.perf_counter()
    oracle.attention_rows(full(x["q"]), full(x["k"]), full(x["v"]), w.softmax_scale, rows)
    dt = time.perf_counter() - t
    return dt, 4.0 * len(rows) * w.Skv * w.D, cores


_INPUTS = None


def _oracle_inputs():
    global _INPUTS
    if _INPUTS is None:
        _INPUTS = W.make_inputs(WORKLOAD)
    return _INPUTS


def _sample_text(rows, spent):
    return (f"{rows} query rows of the S=44160 Ulysses workload in samples of {ORACLE_ROWS} "
            f"(~{ORACLE_ROWS // 16} per head), each row over all 44160 keys, fp64 NumPy/BLAS, "
            f"{spent:.1f} s")


def cpu_baseline(budget_s=15.0):
    oracle_sample(ORACLE_ROWS // 8, seed=99)  # untimed: BLAS threads and page-in
    spent, flops, cores, rounds = 0.0, 0.0, 1, 0
    while spent < budget_s and rounds < 40:
        dt, f, cores = oracle_sample(ORACLE_ROWS, seed=100 + rounds)
        spent += dt
        flops += f
        rounds += 1
    return {"value": round(flops / spent / 1e12, 6), "unit": UNIT, "cores": cores,
            "kind": "oracle", "sample": _sample_text(rounds * ORACLE_ROWS, spent)}


def oracle_per_config(row_sample=2048):
    """The fp64 oracle timed on each configuration's own inputs on the host cores (one JSON
    line).  Configs 1 and 2 run in full; config 3 as one of its eight K/V chunks plus one
    merge, scaled to the eight chunks and seven merges; configs 4 and 5 on ``row_sample``
    sampled query rows, scaled to all rows.  Each entry says which."""
    import oracle

    cores = oracle.set_threads()
    out = {"kind": "oracle", "cores": cores, "configs": {}}
    for n, w in W.WORKLOADS.items():
        x = W.make_inputs(w)
        flops = w.attn_flops
        if w.kind == "chunked":  # fp32, two chunks folded by the merge
            t = time.perf_counter()
            c = x["chunks"][0]
            oa, la = oracle.attention(x["q"], x["k"][:, :c], x["v"][:, :c], w.softmax_scale)
            ob, lb = oracle.attention(x["q"], x["k"][:, c:], x["v"][:, c:], w.softmax_scale)
            oracle.merge(oa, la, ob, lb)
            sec, how = time.perf_counter() - t, "full: two chunks and their merge"
        elif w.kind == "single" and flops < 1e12:
            t = time.perf_counter()
            oracle.attention(x["q"], x["k"], x["v"], w.softmax_scale)
            sec, how = time.perf_counter() - t, "full"
        elif w.kind == "ring":
            c = x["chunks"][0]
            t = time.perf_counter()
            oa, la = oracle.attention(x["q"], x["k"][:, :c], x["v"][:, :c], w.softmax_scale)
            t1 = time.perf_counter()
            oracle.merge(oa, la, oa, la)
            t2 = time.perf_counter()
            sec = 8 * (t1 - t) + 7 * (t2 - t1)
            how = "one of the 8 chunks and one merge, timed and scaled to 8 chunks + 7 merges"
        else:  # the long sequences (Ulysses, joint video + text): sampled rows, all keys
            S = w.Sq
            H = w.H * w.P if w.kind == "ulysses" else w.H
            full = (lambda t: t.reshape(1, S, H, w.D)) if w.kind == "ulysses" else (lambda t: t)
            g = torch.Generator(device="cpu").manual_seed(500 + n)
            hs = torch.randint(0, H, (row_sample,), generator=g).tolist()
            ts = torch.randint(0, S, (row_sample,), generator=g).tolist()
            rows = [(0, h, i) for h, i in zip(hs, ts)]
            oracle.attention_rows(full(x["q"]), full(x["k"]), full(x["v"]), w.softmax_scale,
                                  rows[: row_sample // 8])  # untimed: page-in, BLAS threads
            t = time.perf_counter()
            oracle.attention_rows(full(x["q"]), full(x["k"]), full(x["v"]), w.softmax_scale, rows)
            dt = time.perf_counter() - t
            sec = dt * (H * S) / row_sample
            how = f"{row_sample} sampled query rows over all {S} keys, scaled to all {H * S} rows"
        out["configs"][w.name] = {"seconds": round(sec, 3), "flops": flops,
                                  "TFLOP/s": round(flops / sec / 1e12, 6), "how": how}
        del x
    return out


def run_reference(args, world, rank):
    if rank != 0:
        return  # the CPU oracle arm runs on rank 0 only
    for i in range(args.warmup):
        oracle_sample(ORACLE_ROWS // 8, seed=1 + i)
    tot_t, tot_f, cores = 0.0, 0.0, 1
    for i in range(args.steps):
        dt, f, cores = oracle_sample(ORACLE_ROWS, seed=1000 + i)
        tot_t += dt
        tot_f += f
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot_t / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(step=args.step),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores,
                         "kind": "oracle",
                         "sample": "one step = " + _sample_text(ORACLE_ROWS, tot_t / args.steps)},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-configs", action="store_true",
                    help="time the CPU oracle on every configuration (host only) and exit")
    ap.add_argument("--profile", action="store_true",
                    help="for profiler captures: run only warm-up + timed steps (no aux "
                         "kernels, no end-to-end pass, no CPU baseline)")
    ap.add_argument("--clocks-csv", default=None, metavar="PATH",
                    help="also write the raw nvidia-smi samples of each timed region to PATH "
                         "('{rank}' and '{step}' are replaced by the rank and step variant)")
    ap.add_argument("--qk-norm", action="store_true",
                    help="step variant: Q/K RMSNorm fused into one Q/K/V seq2head launch "
                         "(not the headline step; for profiling that kernel)")
    ap.add_argument("--step", choices=("fused", "plain"), default="fused",
                    help="the headline step: 'fused' = the Ulysses pass as one kernel "
                         "(cpattn_ulysses_fwd), 'plain' = 3x seq2head + attention + head2seq; "
                         "the other variant is timed the same way and reported beside it")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    world, rank, local = dist_env()
    if args.oracle_configs:  # the oracle's own timing table (host cores only, no GPU work)
        if rank == 0:
            print(json.dumps(oracle_per_config()), flush=True)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
