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
    """SM clock, power and clock-event reasons of one GPU, polled through NVML every ``period_s``
    from a host thread while the timed region runs (the host has queued the work, so the GPU is busy
    for the whole window)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index, period_s=0.001):
        self.gpu, self.period = gpu_index, period_s
        self.rows, self.thread, self.stop_flag = [], None, False

    def start(self):
        try:
            import threading

            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.thread = None
            return

        def poll():
            while not self.stop_flag:
                try:
                    self.rows.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                      pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                      pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
                except Exception:
                    pass
                time.sleep(self.period)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join()
        rows = [r for r in self.rows if not (r[2] & 0x1)] or self.rows   # drop samples flagged GPU idle
        if not rows:
            return None
        reasons = sorted({name for _, _, bits in rows for bit, name in self.REASONS.items() if bits & bit})
        mhz = [r[0] for r in rows]
        return {"sm_mhz": statistics.median(mhz), "sm_mhz_min": min(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(rows), "power_w_max": round(max(r[1] for r in rows), 1),
                "source": "NVML, polled every 1 ms during the timed steps"}


# Dense bf16 tensor-core rate of tcgen05 kind::f16 per SM and clock (a 128 x 128 x 16 MMA every
# 64 cycles; back-to-back MMAs measured 8190 on this part), and NVIDIA's published dense bf16
# figure for HGX B200.
TC_FLOP_PER_CLK_SM = 8192
DATASHEET_BF16_TFLOPS = 2250.0


def clock_peak_tflops(sm_mhz, sms):
    """Tensor-core peak at the sampled SM clock: 8192 FLOP per clock per SM, `sms` SMs."""
    return TC_FLOP_PER_CLK_SM * sms * sm_mhz * 1e6 / 1e12


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
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

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
        calls = [("fa_fwd", (qq, kk, vv, oo, ll, B, H, N, d, scale, causal, kl_ptr, p, seed, sp))]
        if args.separate_dq:   # dK, dV and dQ in separate passes: one ABI call, three launches
            calls.append(("fa_bwd_split", (qq, kk, vv, oo, ll, dd, gq, gk, gv, B, H, N, d, scale, causal, kl_ptr, p,
                                           seed, ws.data_ptr(), ws.numel(), sp)))
        else:
            calls += [
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
    names = ["fa_fwd", "fa_bwd_split"] if args.separate_dq else ["fa_fwd", "fa_bwd_prep", "fa_bwd_main",
                                                                   "fa_bwd_dq_convert"]

    for _ in range(args.warmup):
        flush.zero_()
        launches(dev_tensors)
    _lib.call("fa_check", sp)

    def timed(n_steps):
        """n_steps steps, each launch timed with CUDA events, L2 flushed before each step."""
        sampler = ClockSampler(local)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(n_steps)]
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        sampler.start()
        for s in range(n_steps):
            flush.zero_()
            ev[s][0].record(stream)
            launches(dev_tensors, ev[s])
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        clk = sampler.stop()
        _lib.call("fa_check", sp)
        pk_ms = {n: [] for n in names}
        st_ms = []
        for s in range(n_steps):
            for i, n in enumerate(names):
                pk_ms[n].append(ev[s][i].elapsed_time(ev[s][i + 1]))
            st_ms.append(ev[s][0].elapsed_time(ev[s][len(names)]))
        return pk_ms, st_ms, clk

    per_kernel, step_ms, clocks = timed(args.steps)
    fwd_ms_local = statistics.mean(per_kernel["fa_fwd"])
    step_ms_local = statistics.mean(step_ms)
    # the same steps again, back to back, many more of them: the figure once power management has
    # settled (reported beside the headline value, which is the short run above)
    sustained = None
    if args.sustained_steps > 0:
        s_pk, s_step, s_clk = timed(args.sustained_steps)
        sustained = (statistics.mean(s_step), statistics.mean(s_pk["fa_fwd"]), s_clk)

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
    if sustained is not None:
        s_ms, _, s_tflops = aggregate(sustained[0], w.fwd_bwd_flops(), world, rmax, rsum)
        _, _, s_fwd_tflops = aggregate(sustained[1], w.fwd_flops(), world, rmax, rsum)
    fwd_ms, fwd_flops, fwd_tflops = aggregate(fwd_ms_local, w.fwd_flops(), world, rmax, rsum)
    e2e_ms, _, e2e_tflops = aggregate(e2e_ms_local, w.fwd_bwd_flops(), world, rmax, rsum)
    kernel_ms = {n: rmax(statistics.mean(per_kernel[n])) for n in names}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    pk = peaks()
    kflops = {"fa_fwd": w.fwd_flops(), "fa_bwd_split" if args.separate_dq else "fa_bwd_main": 2.5 * w.fwd_flops()}
    kbytes = algorithmic_bytes(B, H, N, d)
    kernels = {}
    for n in names:
        entry = {"avg_ms": round(kernel_ms[n], 5), "share": round(kernel_ms[n] / sum(kernel_ms.values()), 4)}
        gbs = kbytes[n] / (kernel_ms[n] * 1e-3) / 1e9
        ncu = load_ncu(n, w.name)
        if n in kflops:
            ach = kflops[n] / (kernel_ms[n] * 1e-3) / 1e12
            entry.update({"bound": "tensor", "achieved_tflops": round(ach, 1),
                          "frac_of_measured_peak": round(ach / pk["bf16_tflops"], 4),
                          "hbm_gbs": round(gbs, 1), "hbm_frac_of_measured_peak": round(gbs / pk["hbm_gbs"], 4),
                          "algorithmic_bytes": kbytes[n],
                          "tensor_pipe_active_pct": None if ncu is None else ncu.get("tensor_active_pct")})
        else:
            entry.update({"bound": "hbm", "achieved_gbs": round(gbs, 1),
                          "frac_of_measured_peak": round(gbs / pk["hbm_gbs"], 4), "algorithmic_bytes": kbytes[n]})
        if ncu is not None:
            entry["dram_bytes_ncu"] = ncu.get("dram_bytes")
        kernels[n] = entry
    dom = max(kflops, key=lambda n: kernel_ms[n])
    dom_ach = kflops[dom] / (kernel_ms[dom] * 1e-3) / 1e12
    dom_ncu = load_ncu(dom, w.name)
    mhz = clocks["sm_mhz"] if clocks else None
    line = {
        "metric": METRIC, "value": round(tflops, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
        "config": config_of(w, world),
        "fwd_tflops": round(fwd_tflops, 2), "fwd_ms": round(fwd_ms, 5),
        "fwd_frac_of_peak": round(fwd_tflops / world / pk["bf16_tflops"], 4),
        "fwd_bwd_frac_of_peak": round(tflops / world / pk["bf16_tflops"], 4),
        "frac_of_datasheet": {"fwd": round(fwd_tflops / world / DATASHEET_BF16_TFLOPS, 4),
                              "fwd_bwd": round(tflops / world / DATASHEET_BF16_TFLOPS, 4)},
        "frac_of_clock_peak": None if mhz is None else {
            "fwd": round(fwd_tflops / world / clock_peak_tflops(mhz, sms), 4),
            "fwd_bwd": round(tflops / world / clock_peak_tflops(mhz, sms), 4),
            "peak_tflops": round(clock_peak_tflops(mhz, sms), 1), "sm_mhz": mhz, "sms": sms},
        "peak_source": (f"targets use the {pk['source']} bf16 peak {pk['bf16_tflops']} TFLOP/s (cuBLAS burst); "
                        f"HBM {pk['hbm_gbs']} GB/s {pk['source']}; frac_of_datasheet divides by NVIDIA's dense bf16 "
                        f"{DATASHEET_BF16_TFLOPS} TFLOP/s (HGX B200); frac_of_clock_peak by 8192 FLOP/clk/SM x {sms} SMs "
                        "at the median sampled SM clock"),
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": round(dom_ach, 1), "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(dom_ach / pk["bf16_tflops"], 4),
                     "traffic": None if dom_ncu is None else dom_ncu.get("dram_bytes"),
                     "algorithmic_flops_per_launch": kflops[dom], "peak_kind": "burst (kernel timed per launch)"},
        "kernels": kernels,
        "e2e": {"value": round(e2e_tflops, 2), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": 4 * args.steps,   # fused: fwd, prep, main, convert; split: fwd, prep, main, dQ pass
        "clocks": clocks,
    }
    if sustained is not None:
        line["sustained"] = {"steps": args.sustained_steps, "value": round(s_tflops, 2), "unit": UNIT,
                             "ms_per_step": round(s_ms, 5), "fwd_tflops": round(s_fwd_tflops, 2),
                             "clocks": sustained[2],
                             "note": "the same step repeated back to back after the timed region"}
    if x["key_lens"] is not None and not w.causal:
        # key padding: every query row sees len_b keys, so the work done is sum_b len_b * N per head
        # instead of the nominal N^2 (the metric's value stays the nominal count)
        eff = float(np.sum(x["key_lens"].astype(np.float64))) / (B * N)
        line["effective"] = {"fraction_of_nominal_flops": round(eff, 4),
                             "fwd_bwd_tflops": round(tflops * eff, 2), "fwd_tflops": round(fwd_tflops * eff, 2),
                             "note": "FLOPs counted over the allowed keys only: 4 d H N sum_b len_b forward"}
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


def load_ncu(kernel, workload):
    """The committed ncu figures of ``kernel`` on ``workload`` (dram bytes read + written per launch,
    tensor-pipe active %); None when there are none or the kernel sources changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if e is None or e.get("csrc_hash") != csrc_hash():
        return None
    return e


def algorithmic_bytes(B, H, N, d):
    """Bytes each launch must move at least (the method's own traffic, no re-reads):
    fa_fwd reads Q, K, V and writes O (bf16) and lse (fp32); fa_bwd_prep reads O and dO and writes D
    and clears the fp32 dQ accumulator; fa_bwd_main reads Q, K, V, dO, lse, D and writes dK, dV (its
    fp32 dQ reductions, 4 B per element and key tile, are the method's choice and not counted);
    fa_bwd_dq_convert reads the accumulator and writes dQ."""
    e, rows = B * H * N * d, B * H * N
    return {"fa_fwd": 4 * 2 * e + 4 * rows,
            "fa_bwd_prep": 2 * 2 * e + 4 * e + 4 * rows,
            "fa_bwd_main": 6 * 2 * e + 2 * 4 * rows,
            "fa_bwd_dq_convert": 4 * e + 2 * e,
            # the whole backward with dQ in its own pass: read Q, K, V, O, dO, lse; write dQ, dK, dV (+ D)
            "fa_bwd_split": 8 * 2 * e + 2 * 4 * rows}


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


# ----------------------------------------------------------------------------- decode-shaped forward
def run_decode(args, world, rank, local):
    """fa_fwd_decode on Nq new rows per head against a cache of Nkv keys (HBM-bound): one step is one
    call (split + combine launches) over inputs resident in HBM, L2 flushed before each step."""
    import torch
    from exact_io_aware_68_b200 import _lib
    from exact_io_aware_68_b200.inputs import make_decode_inputs

    B, H, Nq, Nkv, d = args.decode
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lib = _lib.load()
    x = make_decode_inputs(B, H, Nq, Nkv, d, seed=7, exact=False)

    def up(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = up(x["q"]), up(x["k"]), up(x["v"])
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(lib.fa_fwd_decode_workspace_size(B, H, Nq, Nkv, d), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    a = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Nq, Nkv, d, x["scale"],
         int(args.decode_causal), None, ws.data_ptr(), ws.numel(), stream.cuda_stream)
    for _ in range(args.warmup):
        flush.zero_()
        _lib.call("fa_fwd_decode", *a)
    _lib.call("fa_check", stream.cuda_stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    torch.cuda.synchronize(dev)
    sampler.start()
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        _lib.call("fa_fwd_decode", *a)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    _lib.call("fa_check", stream.cuda_stream)
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    if rank != 0:
        return None
    pk = peaks()
    kv_bytes = 2 * B * H * Nkv * d * 2                      # K and V, bf16, read once
    alg_bytes = kv_bytes + 2 * B * H * Nq * d * 2 + 4 * B * H * Nq   # + q read, o written, lse written
    flops = 4.0 * B * H * Nq * Nkv * d                     # upper bound (no causal discount: Nq << Nkv)
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    return {"metric": "decode-shaped attention forward, HBM GB/s (K and V read once)", "value": round(gbs, 1),
            "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
            "config": {"workload": f"decode_{B}x{H}_q{Nq}_kv{Nkv}x{d}", "B": B, "H": H, "Nq": Nq, "Nkv": Nkv, "d": d,
                       "causal": bool(args.decode_causal),
                       "l2": "flushed (256 MiB write) before each timed step, outside the events"},
            "roofline": {"kernel": "fa_fwd_decode", "bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4), "traffic": None,
                         "algorithmic_bytes_per_launch": alg_bytes},
            "tflops": round(flops / (ms * 1e-3) / 1e12, 2), "gpu_launches": 2 * args.steps, "clocks": clocks}


# ----------------------------------------------------------------------------- memory against N
def memory_table(args, local):
    """Device memory and HBM bytes of exact attention against N, fused (this library) beside a
    materialising forward + backward made of torch ops (cuBLAS GEMMs, a softmax kernel): the O(N)
    versus O(N^2) claim of "48 FlashAttention" (block "PyTorch FlashAttention под капотом sdpa") and
    the memory comparison of "Flash Attention：如何通过硬件感知优化重塑注意力机制的未来" (section 2.1).
    The materialising arm is a comparison only; it runs where its N x N tensors fit.
    One JSON line per N: peak bytes allocated during the call beyond the inputs, and the algorithmic
    HBM bytes (fused: Q, K, V, O, dO, dQ, dK, dV, lse, D; materialising: adds S, P, dP, dS written
    and read once each, fp32)."""
    import torch
    from exact_io_aware_68_b200 import api

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B, H, d = 1, 16, 64
    for N in (512, 1024, 2048, 4096, 8192, 16384, 32768, 65536):
        g = torch.Generator(device=dev).manual_seed(N)
        q, k, v, do = (torch.randn((B, H, N, d), device=dev, generator=g, dtype=torch.float32).to(torch.bfloat16)
                       for _ in range(4))
        e = B * H * N * d
        row = {"N": N, "B": B, "H": H, "d": d}
        torch.cuda.synchronize(dev)
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        o, lse = api.attention_fwd(q, k, v, None, True)
        api.attention_bwd(q, k, v, o, lse, do, None, True)
        t1.record()
        torch.cuda.synchronize(dev)
        row["fused_peak_bytes"] = torch.cuda.max_memory_allocated(dev) - base
        row["fused_hbm_bytes"] = 8 * e + 4 * B * H * N + 16 * e + 8 * B * H * N
        row["fused_ms"] = round(t0.elapsed_time(t1), 3)
        del o, lse
        nn = B * H * N * N
        row["materialising_hbm_bytes"] = row["fused_hbm_bytes"] + 4 * 2 * 4 * nn   # S, P, dP, dS: fp32, write + read
        need = 4 * 4 * nn + 8 * e
        free = torch.cuda.mem_get_info(dev)[0]
        if need < 0.8 * free:
            qf, kf, vf = (t.float().requires_grad_() for t in (q, k, v))
            torch.cuda.synchronize(dev)
            base = torch.cuda.memory_allocated(dev)
            torch.cuda.reset_peak_memory_stats(dev)
            t0.record()
            s_ = (qf @ kf.transpose(-1, -2)) / d ** 0.5
            s_ = s_.masked_fill(torch.ones(N, N, dtype=torch.bool, device=dev).triu(1), float("-inf"))
            p_ = torch.softmax(s_, dim=-1)
            o_ = p_ @ vf
            o_.backward(do.float())
            t1.record()
            torch.cuda.synchronize(dev)
            row["materialising_peak_bytes"] = torch.cuda.max_memory_allocated(dev) - base
            row["materialising_ms"] = round(t0.elapsed_time(t1), 3)
            del qf, kf, vf, s_, p_, o_
        else:
            row["materialising_peak_bytes"] = None
            row["materialising_note"] = f"N x N fp32 tensors need {need / 2**30:.0f} GiB: not run"
        row["nxn_fp32_bytes_per_tensor"] = 4 * nn
        print(json.dumps(row), flush=True)
        del q, k, v, do
        torch.cuda.empty_cache()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--sustained-steps", type=int, default=200,
                    help="after the timed steps, time this many more back to back and report them as "
                         "'sustained' (0: skip)")
    ap.add_argument("--workload", default=HEADLINE, choices=[n for n, w in WORKLOADS.items() if w.dtype == "bf16"])
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--separate-dq", action="store_true",
                    help="backward through fa_bwd_split (dQ in a pass of its own) instead of the fused dQ")
    ap.add_argument("--decode", type=int, nargs=5, metavar=("B", "H", "NQ", "NKV", "D"),
                    help="time the decode-shaped forward instead (Nq rows against a cache of Nkv keys)")
    ap.add_argument("--decode-causal", type=int, default=1)
    ap.add_argument("--memory-table", action="store_true",
                    help="print device memory and HBM bytes against N, fused beside materialising, and exit")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if args.memory_table:
        if rank == 0:
            memory_table(args, local)
        return
    w = WORKLOADS[args.workload]
    if args.decode is not None:
        line = run_decode(args, world, rank, local) if args.impl == "native" else None
    elif args.impl == "reference":
        line = run_reference(args, w, world, rank)
    else:
        line = run_native(args, w, world, rank, local)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
