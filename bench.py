#!/usr/bin/env python
"""Throughput of exact attention, forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

One step = one pass of the whole hot path over one batch: fa_fwd (O, lse) then fa_bwd's three
launches (prep, main, dQ convert).  Metric: attention TFLOP/s, forward FLOPs 4 N^2 d B H (halved
when causal), backward 2.5x forward; the step's value counts forward + backward.  Inputs are
seeded synthetic bf16 tensors of the workload's shape, resident in HBM; L2 is flushed (a 256 MiB
write) before every timed step, outside the step's events.  Every launch is timed with CUDA events
on the stream it runs on.  Under torchrun (N > 1) each rank runs the same workload on its own GPU
(the path splits over (batch, head) with no exchange, so ranks are independent replicas); the
step time is the max over ranks and the value counts all ranks' work.

--impl reference times the host-side fp64 oracle (the plain definition) on this machine's cores
over a bounded sample of the same workload; rank 0 only.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_68_b200.workloads import HEADLINE, WORKLOADS  # noqa: E402

METRIC = "attention TFLOP/s fwd & fwd+bwd (bf16, N=4096, d=128) vs B200 tensor peak"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"bf16_tflops": d["bf16_tflops"], "bf16_tflops_sustained": d["bf16_tflops_sustained"],
                "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def config_of(w, world):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "key_padding": w.key_len_range is not None, "dropout_p": w.dropout_p, "dtype": w.dtype,
            "parallelism": f"replicas{world}" if world > 1 else "single-gpu",
            "l2": "flushed (256 MiB write) before each timed step, outside the events"}


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- dist helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def aggregate(step_ms_local, flops_per_step_local, world, reduce_max, reduce_sum):
    """Whole-job figures: the slowest rank's time and every rank's work.

    ``reduce_max`` / ``reduce_sum`` combine one float across ranks (identity when world == 1).
    Returns (ms_per_step, total_flops_per_step, tflops)."""
    ms = reduce_max(step_ms_local)
    flops = reduce_sum(flops_per_step_local)
    return ms, flops, flops / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,utilization.gpu")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # the raw samples go to FA_BENCH_CLOCKS_DIR when set (to keep them), else the temp directory
        log_dir = os.environ.get("FA_BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(log_dir, f"fa_bench_clocks_rank{gpu_index}_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as fh:
            lines = fh.readlines()
        if not os.environ.get("FA_BENCH_CLOCKS_DIR"):
            os.remove(self.path)
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                             "active": parts[4], "hw": parts[5], "hwt": parts[6], "swt": parts[7],
                             "pcap": parts[8], "util": float(parts[9])})
            except ValueError:
                continue
        if not rows:
            return None
        busy = [r for r in rows if r["util"] > 0] or rows
        reasons = set()
        for r in busy:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in busy), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(busy), "power_w_max": max(r["power"] for r in rows)}


# ----------------------------------------------------------------------------- native arm
def run_native(args, w, world, rank, local):
    import torch
    from exact_io_aware_68_b200 import _lib
    from exact_io_aware_68_b200.inputs import make_inputs

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lib = _lib.load()

    x = make_inputs(w, exact=False)
    B, H, N, d = w.B, w.H, w.N, w.d

    def up(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v, do = (up(x[n]) for n in ("q", "k", "v", "do"))
    key_lens = None if x["key_lens"] is None else torch.from_numpy(x["key_lens"]).to(dev)
    kl_ptr = None if key_lens is None else key_lens.data_ptr()
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(lib.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    scale, causal, p, seed = w.scale, int(w.causal), w.dropout_p, w.seed

    def launches(tensors, events=None):
        qq, kk, vv, dd, oo, ll, gq, gk, gv = tensors
        calls = [
            ("fa_fwd", (qq, kk, vv, oo, ll, B, H, N, d, scale, causal, kl_ptr, p, seed, sp)),
            ("fa_bwd_prep", (oo, dd, B, H, N, d, ws.data_ptr(), ws.numel(), sp)),
            ("fa_bwd_main", (qq, kk, vv, ll, dd, gk, gv, B, H, N, d, scale, causal, kl_ptr, p, seed,
                             ws.data_ptr(), ws.numel(), sp)),
            ("fa_bwd_dq_convert", (gq, B, H, N, d, scale, ws.data_ptr(), ws.numel(), sp)),
        ]
        for i, (name, a) in enumerate(calls):
            _lib.call(name, *a)
            if events is not None:
                events[i + 1].record(stream)

    dev_tensors = tuple(t.data_ptr() for t in (q, k, v, do, o, lse, dq, dk, dv))
    names = ["fa_fwd", "fa_bwd_prep", "fa_bwd_main", "fa_bwd_dq_convert"]

    for _ in range(args.warmup):
        flush.zero_()
        launches(dev_tensors)
    _lib.call("fa_check", sp)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for s in range(args.steps):
        flush.zero_()
        ev[s][0].record(stream)
        launches(dev_tensors, ev[s])
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop()
    _lib.call("fa_check", sp)
    per_kernel = {n: [] for n in names}
    step_ms = []
    for s in range(args.steps):
        for i, n in enumerate(names):
            per_kernel[n].append(ev[s][i].elapsed_time(ev[s][i + 1]))
        step_ms.append(ev[s][0].elapsed_time(ev[s][4]))
    fwd_ms_local = statistics.mean(per_kernel["fa_fwd"])
    step_ms_local = statistics.mean(step_ms)

    # ---- end to end through the public API, host buffers (pinned), copies inside the timed region
    host = {n: torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in ("q", "k", "v", "do")}
    outs = {n: torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory() for n in ("o", "dq", "dk", "dv")}
    out_lse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs.values()) + out_lse.numel() * 4
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        q.copy_(host["q"], non_blocking=True)
        k.copy_(host["k"], non_blocking=True)
        v.copy_(host["v"], non_blocking=True)
        do.copy_(host["do"], non_blocking=True)
        launches(dev_tensors)
        outs["o"].copy_(o, non_blocking=True)
        out_lse.copy_(lse, non_blocking=True)
        outs["dq"].copy_(dq, non_blocking=True)
        outs["dk"].copy_(dk, non_blocking=True)
        outs["dv"].copy_(dv, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms_local = e0.elapsed_time(e1) / e2e_steps
    _lib.call("fa_check", sp)

    if dist is not None:
        def rmax(v):
            t = torch.tensor([v], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            return float(t.item())

        def rsum(v):
            t = torch.tensor([v], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.SUM)
            return float(t.item())
    else:
        rmax = rsum = float

    ms, flops, tflops = aggregate(step_ms_local, w.fwd_bwd_flops(), world, rmax, rsum)
    fwd_ms, fwd_flops, fwd_tflops = aggregate(fwd_ms_local, w.fwd_flops(), world, rmax, rsum)
    e2e_ms, _, e2e_tflops = aggregate(e2e_ms_local, w.fwd_bwd_flops(), world, rmax, rsum)
    kernel_ms = {n: rmax(statistics.mean(per_kernel[n])) for n in names}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    pk = peaks()
    kflops = {"fa_fwd": w.fwd_flops(), "fa_bwd_main": 2.5 * w.fwd_flops()}
    # algorithmic HBM bytes of the two HBM-bound launches
    rows = B * H * N
    kbytes = {"fa_bwd_prep": rows * d * 2 * 2 + rows * d * 4 + rows * 4,
              "fa_bwd_dq_convert": rows * d * 4 + rows * d * 2}
    kernels = {}
    for n in names:
        entry = {"avg_ms": round(kernel_ms[n], 5), "share": round(kernel_ms[n] / sum(kernel_ms.values()), 4)}
        if n in kflops:
            ach = kflops[n] / (kernel_ms[n] * 1e-3) / 1e12
            entry.update({"bound": "tensor", "achieved_tflops": round(ach, 1),
                          "frac_of_measured_peak": round(ach / pk["bf16_tflops"], 4)})
        else:
            ach = kbytes[n] / (kernel_ms[n] * 1e-3) / 1e9
            entry.update({"bound": "hbm", "achieved_gbs": round(ach, 1),
                          "frac_of_measured_peak": round(ach / pk["hbm_gbs"], 4)})
        kernels[n] = entry
    dom = max(kflops, key=lambda n: kernel_ms[n])
    dom_ach = kflops[dom] / (kernel_ms[dom] * 1e-3) / 1e12
    traffic = load_traffic(dom, w.name)
    line = {
        "metric": METRIC, "value": round(tflops, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
        "config": config_of(w, world),
        "fwd_tflops": round(fwd_tflops, 2), "fwd_ms": round(fwd_ms, 5),
        "fwd_frac_of_peak": round(fwd_tflops / world / pk["bf16_tflops"], 4),
        "fwd_bwd_frac_of_peak": round(tflops / world / pk["bf16_tflops"], 4),
        "peak_source": f"{pk['source']} bf16 {pk['bf16_tflops']} TFLOP/s (burst), HBM {pk['hbm_gbs']} GB/s",
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": round(dom_ach, 1), "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(dom_ach / pk["bf16_tflops"], 4), "traffic": traffic,
                     "algorithmic_flops_per_launch": kflops[dom]},
        "kernels": kernels,
        "e2e": {"value": round(e2e_tflops, 2), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds)
    return line


def csrc_hash(src_dir=None):
    """Hash of the kernel code, to tell whether a stored ncu figure still describes it. Comments
    and whitespace are left out, so editing a comment keeps the figures valid. The sources hold no
    string literal with comment markers."""
    import glob
    import hashlib
    import re

    src_dir = src_dir or os.path.join(ROOT, "exact_io_aware_68_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(src_dir, "*"))):
        with open(f, encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(os.path.basename(f).encode())
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def load_traffic(kernel, workload):
    """dram bytes (read + write) per launch of ``kernel`` from the committed ncu summary; None when
    there is none or the kernel sources changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if e is None or e.get("csrc_hash") != csrc_hash():
        return None
    return e["dram_bytes"]


# ----------------------------------------------------------------------------- oracle timing
def cpu_baseline(w, budget_s=15.0, heads=None):
    """The fp64 oracle as it stands, timed on this host over whole (b, h) heads of the workload.

    Forward + backward of head after head until ``budget_s`` seconds pass (at least one head);
    the metric counts the workload's nominal FLOPs of the heads done."""
    import oracle
    from exact_io_aware_68_b200.inputs import make_inputs
    from exact_io_aware_68_b200.workloads import Workload

    cores = host_cores()
    one = Workload(w.name, w.dtype, 1, 1, w.N, w.d, w.causal, seed=w.seed, factor=w.factor,
                   key_len_range=w.key_len_range, dropout_p=w.dropout_p)
    x = make_inputs(one)
    done, t0 = 0, time.perf_counter()
    limit = heads if heads is not None else 10 ** 9
    while done < limit:
        if w.N > 16384:   # long contexts: query rows a block at a time (full-row softmax per block)
            oracle.backward_head_blocked(x["q64"], x["k64"], x["v64"], x["do64"], x["scale"], w.causal,
                                         x["key_lens"], w.dropout_p, w.seed, 0, 0, block=256)
        else:
            oracle.forward(x["q64"], x["k64"], x["v64"], x["scale"], w.causal, x["key_lens"], w.dropout_p, w.seed)
            oracle.backward(x["q64"], x["k64"], x["v64"], x["do64"], x["scale"], w.causal, x["key_lens"],
                            w.dropout_p, w.seed)
        done += 1
        if heads is None and time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    flops = w.fwd_bwd_flops() / (w.B * w.H) * done
    return {"value": round(flops / dt / 1e12, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} of {w.B * w.H} (b,h) heads of {w.name}, forward + backward, fp64 numpy",
            "seconds": round(dt, 2)}


def run_reference(args, w, world, rank):
    if rank != 0:
        return None
    cb = cpu_baseline(w, budget_s=args.cpu_seconds)
    steps = []
    for _ in range(args.warmup):
        cpu_baseline(w, heads=1)
    for _ in range(args.steps):
        r = cpu_baseline(w, heads=1)
        steps.append(r["seconds"])
    ms = statistics.mean(steps) * 1e3
    value = (w.fwd_bwd_flops() / (w.B * w.H)) / (ms * 1e-3) / 1e12
    return {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
            "config": config_of(w, 1), "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cb["cores"], "kind": "oracle",
                             "sample": f"each step: one (b,h) head of {w.name}, forward + backward, fp64 numpy"},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=HEADLINE, choices=[n for n, w in WORKLOADS.items() if w.dtype == "bf16"])
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        line = run_reference(args, w, world, rank)
    else:
        line = run_native(args, w, world, rank, local)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
