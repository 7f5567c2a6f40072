"""Benchmark: WKV fwd+bwd channel-tokens/s and achieved HBM GB/s on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libwkv|reference]
                [--workload rwkv169m|rwkv1b5_bf16|longctx|decode14b] [--gate | --token-shift]

A step is one pass of the whole hot path over one batch of the workload:
``wkv_forward`` (writing the checkpoints) followed by ``wkv_backward`` on the
same inputs, through the C ABI, inputs resident in HBM.  The default
workload is the RWKV-4 169M-shaped layer (B8 T1024 C768 fp32, seeded
synthetic inputs).  L2 is flushed (a 2x-L2 buffer is written) before every
timed step, outside the timed events; each step is bracketed by CUDA events
on the launching stream and the per-step times are summed.  ``--gate`` times
the gated calls instead (``wkv_forward_gated`` / ``wkv_backward_gated``,
o = sigmoid(r) * wkv, with a seeded N(0, 1) gate input r); ``--token-shift``
times the token shift (three interpolations) on the workload's layer shape.

Multi-GPU (torchrun): every rank runs an independent replica of the workload
on its own GPU (the operator has no cross-sequence exchange; weak scaling);
ranks are timed on the device and the maximum over ranks is reported.

``--impl reference`` times the float64 CPU oracle (the only reference this
operator has) on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rwkv_linear_rnn_b200 import workloads  # noqa: E402

# algorithmic bytes per channel-token (per channel-step for the decode step)
# (gated: the forward also reads r; the backward reads r and writes grad_r)
ALG_BYTES = {("fwd", "f32"): 12, ("fwd", "bf16"): 6, ("bwd", "f32"): 20, ("bwd", "bf16"): 10,
             ("fwd_gated", "f32"): 16, ("fwd_gated", "bf16"): 8, ("bwd_gated", "f32"): 28,
             ("bwd_gated", "bf16"): 14, ("step", "f32"): 36}


# Kernels each call launches on 16-byte aligned rows (all bench workloads),
# per kernel selector: (kernel names, launches per call).
FWD_PLAN = {"auto": ("fwd_seg_kernel", 1), "segment": ("fwd_seg_kernel", 1),
            "cluster": ("fwd_clu_kernel", 1)}
BWD_PLAN = {"auto": ("bwd_seg_kernel", 1),
            "segment": ("bwd_seg_kernel", 1)}
KERNEL_IDS = {"auto": 0, "segment": 6, "cluster": 7}

# DRAM bytes (read + write) per launch of the backward's main kernel from one
# ncu capture of this bench's workload (cold L2; gk/gv lines still dirty in
# L2 at kernel end are not counted).  Keyed by (workload, kernel, gated); a
# kernel changed since its capture has no entry (traffic reported as null).
TRAFFIC = {("rwkv169m", "bwd_seg_kernel", False): 78_219_776 + 416_768,
           ("rwkv169m", "bwd_seg_kernel", True): 112_421_120 + 24_960_768}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def stop(self, window=None):
        """Summary of the samples that arrived inside `window` (monotonic
        start, end of the timed region); all samples if none did."""
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        inside = [ln for t, ln in self.lines if window and window[0] <= t <= window[1]]
        scope = "timed region"
        if not inside:
            inside, scope = [ln for _, ln in self.lines], "whole sampler run (no sample inside the timed region)"
        for ln in inside:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "scope": scope}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, dist, device) -> float:
    """The maximum of a per-rank time over all ranks (every rank calls this
    in the same order); identity without a process group."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: int, n_ranks: int, ms_per_step: float) -> float:
    """Whole-job throughput: the units every rank processed in one step over
    the slowest rank's step time (weak scaling, replicas)."""
    return n_ranks * units_per_rank / (ms_per_step * 1e-3)


def cpu_baseline(wl_name: str, min_seconds: float = 10.0, gate: bool = False):
    """Time the oracle (float64 recurrence fwd + reverse bwd, gated or not)
    on the host."""
    import oracle
    wl = workloads.WORKLOADS[wl_name]
    what = "gated fwd+bwd" if gate else "fwd+bwd"
    if wl_name == "rwkv169m":
        inp = workloads.generate(wl, gate=gate)
        sample = f"full rwkv169m workload (B8 T1024 C768) {what}, repeated"
    else:  # a channel slice of the big workloads keeps the sample bounded
        C = 256
        inp = workloads.generate(wl, C=C, T=min(wl.T, 4096), grad=True, gate=gate)
        sample = f"{wl_name} with C={C}, T={inp['T']} {what}, repeated"
    names = ("w", "u", "k", "v", "r", "gy") if gate else ("w", "u", "k", "v", "gy")
    args = [np.asarray(inp[n], np.float64) for n in names]
    units = inp["B"] * inp["T"] * inp["C"]
    times = []
    t_end = time.perf_counter() + min_seconds
    while time.perf_counter() < t_end or len(times) < 3:
        t0 = time.perf_counter()
        if gate:
            oracle.fwd_gated(*args[:5])
            oracle.bwd_gated(*args)
        else:
            oracle.fwd_recur(*args[:4], want_y=True)
            oracle.bwd_recur(*args)
        times.append(time.perf_counter() - t0)
    med = statistics.median(times)
    return {"value": units / med, "unit": "channel-tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{sample} x{len(times)}, median"}


def metric_name(gate: bool) -> str:
    what = "gated WKV" if gate else "WKV"
    return f"{what} fwd+bwd channel-tokens/s (HBM GB/s and % of roofline alongside)"


def token_shift_cpu_baseline(wl_name: str, min_seconds: float):
    """Time the token-shift oracle (float64 numpy, forward + backward of the
    three interpolations) on the workload's layer shape."""
    from oracle import tokenshift as ots
    wl = workloads.WORKLOADS[wl_name]
    B, T, C, n = wl.B, min(wl.T, 4096), wl.C, 3
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    x = rng.standard_normal((B, T, C))
    xp = rng.standard_normal((B, C))
    mu = rng.random((n, C))
    g = rng.standard_normal((n, B, T, C))
    times = []
    t_end = time.perf_counter() + min_seconds
    while time.perf_counter() < t_end or len(times) < 3:
        t0 = time.perf_counter()
        ots.shift(x, mu, xp)
        ots.shift_bwd(x, mu, g, xp)
        times.append(time.perf_counter() - t0)
    med = statistics.median(times)
    return {"value": B * T * C / med, "unit": "channel-tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{wl_name} token shift (B{B} T{T} C{C}, n=3) fwd+bwd x{len(times)}, median"}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    if args.token_shift:
        cb = token_shift_cpu_baseline(args.workload, min_seconds=max(1.0, 2.0 * args.steps))
        wl = workloads.WORKLOADS[args.workload]
        line = {"metric": "token-shift fwd+bwd channel-tokens/s (3 interpolations; HBM GB/s alongside)",
                "value": cb["value"], "unit": "channel-tokens/s", "n_gpus": 1, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": wl.channel_tokens / cb["value"] * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded)", "impl": "reference",
                "config": {"workload": args.workload, "op": "token_shift", "B": wl.B, "T": wl.T, "C": wl.C,
                           "n": 3},
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "channel-tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    cb = cpu_baseline(args.workload, min_seconds=max(1.0, 2.0 * args.steps), gate=args.gate)
    wl = workloads.WORKLOADS[args.workload]
    line = {"metric": metric_name(args.gate),
            "value": cb["value"], "unit": "channel-tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": wl.channel_tokens / cb["value"] * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": args.workload, "B": wl.B, "T": wl.T, "C": wl.C,
                       **({"gate": True} if args.gate else {})},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "channel-tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_libwkv(args):
    import torch
    import rwkv_linear_rnn_b200 as W
    from rwkv_linear_rnn_b200 import abi

    ws_n, rank, local = dist_env()
    dist = None
    if ws_n > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = workloads.WORKLOADS[args.workload]
    if "bwd" not in wl.ops:
        raise SystemExit(f"workload {args.workload} has no backward; pick a fwd+bwd workload")
    inp = workloads.generate(wl, seed=wl.seed + 1000 * rank, gate=args.gate)
    B, T, C = inp["B"], inp["T"], inp["C"]
    dt = W.WKV_BF16 if inp["dtype"] == "bf16" else W.WKV_F32
    tdt = torch.bfloat16 if dt == W.WKV_BF16 else torch.float32

    def to_dev(name):
        if dt == W.WKV_BF16 and name in ("k", "v", "gy", "r"):
            return torch.from_numpy(inp[name + "_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(inp[name]).to(dev)

    w, u, k, v, gy = (to_dev(n) for n in ("w", "u", "k", "v", "gy"))
    r = to_dev("r") if args.gate else None
    gr = torch.empty_like(k) if args.gate else None
    y = torch.empty_like(k)
    gk = torch.empty_like(k)
    gv = torch.empty_like(v)
    gw = torch.empty(C, device=dev)
    gu = torch.empty(C, device=dev)
    ckpt = torch.empty(W.wkv_ckpt_size(B, T, C) // 4, device=dev)
    nws = W.wkv_workspace_size(W.WKV_OP_BACKWARD, B, T, C, dt)
    wsb = torch.zeros(nws, dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_w = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(2 * l2 // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # write 2x L2 (evicts everything), then read another 2x L2 so the
        # lines left behind are clean: the timed kernels neither hit their
        # inputs in L2 nor pay for write-backs of the flush
        flush_w.zero_()
        flush_r.sum()
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    P = lambda t: t.data_ptr()

    fopt = abi.Options(kernel=KERNEL_IDS[args.fwd_kernel])
    bopt = abi.Options(kernel=KERNEL_IDS[args.bwd_kernel])

    def fwd():
        if args.gate:
            abi.check(abi.wkv_forward_gated_ex(B, T, C, dt, P(w), P(u), P(k), P(v), P(r), 0, P(y), 0,
                                               P(ckpt), P(wsb), nws, sp, fopt))
        else:
            abi.check(abi.wkv_forward_ex(B, T, C, dt, P(w), P(u), P(k), P(v), 0, P(y), 0, P(ckpt),
                                         P(wsb), nws, sp, fopt))

    def bwd():
        if args.gate:
            abi.check(abi.wkv_backward_gated_ex(B, T, C, dt, P(w), P(u), P(k), P(v), P(r), P(gy), 0,
                                                P(ckpt), P(gw), P(gu), P(gk), P(gv), P(gr), P(wsb),
                                                nws, sp, bopt))
        else:
            abi.check(abi.wkv_backward_ex(B, T, C, dt, P(w), P(u), P(k), P(v), P(gy), 0, P(ckpt),
                                          P(gw), P(gu), P(gk), P(gv), P(wsb), nws, sp, bopt))

    for _ in range(args.warmup):
        flush_l2()
        fwd()
        bwd()
    torch.cuda.synchronize()
    if abi.wkv_get_status(P(wsb), sp) != 0:
        raise SystemExit("device-side status error during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)  # nvidia-smi is sampling before the timed region starts
    t_begin = time.monotonic()
    for i in range(K):
        flush_l2()
        ev[i][0].record(stream)
        fwd()
        ev[i][1].record(stream)
        bwd()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop(window=(t_begin, time.monotonic()))
    if dist:
        dist.barrier()
    t_fwd = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    t_bwd = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    total_ms = max_over_ranks(sum(t_fwd) + sum(t_bwd), dist, dev)
    status = abi.wkv_get_status(P(wsb), sp)

    # e2e: pinned host buffers, every step's copies inside the timed region,
    # through the same ABI.  Steps are pipelined over three streams (PCIe is
    # full duplex): step i+1's inputs are copied in while step i computes and
    # step i's results are copied out; device inputs and outputs are double
    # buffered, and the events order each buffer's reuse.
    e2e = None
    if not args.no_e2e:
        in_names = ["k", "v", "gy"] + (["r"] if args.gate else [])
        out_names = ["y", "gk", "gv", "gw", "gu"] + (["gr"] if args.gate else [])
        dev_now = {"k": k, "v": v, "gy": gy, "r": r, "y": y, "gk": gk, "gv": gv, "gw": gw, "gu": gu, "gr": gr}
        host_in = {n: dev_now[n].cpu().pin_memory() for n in in_names}
        host_out = {n: torch.empty_like(dev_now[n], device="cpu").pin_memory() for n in out_names}
        sets = [{n: torch.empty_like(dev_now[n]) for n in in_names + out_names} for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out.values())
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def step_on(bs, sp_):
            if args.gate:
                abi.check(abi.wkv_forward_gated_ex(B, T, C, dt, P(w), P(u), P(bs["k"]), P(bs["v"]), P(bs["r"]), 0,
                                                   P(bs["y"]), 0, P(ckpt), P(wsb), nws, sp_, fopt))
                abi.check(abi.wkv_backward_gated_ex(B, T, C, dt, P(w), P(u), P(bs["k"]), P(bs["v"]), P(bs["r"]),
                                                    P(bs["gy"]), 0, P(ckpt), P(bs["gw"]), P(bs["gu"]),
                                                    P(bs["gk"]), P(bs["gv"]), P(bs["gr"]), P(wsb), nws, sp_,
                                                    bopt))
            else:
                abi.check(abi.wkv_forward_ex(B, T, C, dt, P(w), P(u), P(bs["k"]), P(bs["v"]), 0, P(bs["y"]), 0,
                                             P(ckpt), P(wsb), nws, sp_, fopt))
                abi.check(abi.wkv_backward_ex(B, T, C, dt, P(w), P(u), P(bs["k"]), P(bs["v"]), P(bs["gy"]), 0,
                                              P(ckpt), P(bs["gw"]), P(bs["gu"]), P(bs["gk"]), P(bs["gv"]),
                                              P(wsb), nws, sp_, bopt))

        def pipeline(nsteps, timed):
            ev = lambda: torch.cuda.Event(enable_timing=timed)
            in_done, cmp_done, out_done = [], [], []
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(s_in)
            for i in range(nsteps):
                bs = sets[i % 2]
                with torch.cuda.stream(s_in):  # inputs of step i (after step i-2 has read this set)
                    if i >= 2:
                        s_in.wait_event(cmp_done[i - 2])
                    for n in in_names:
                        bs[n].copy_(host_in[n], non_blocking=True)
                    in_done.append(ev()); in_done[-1].record(s_in)
                s_cmp.wait_event(in_done[i])  # compute (after step i-2's results are copied out)
                if i >= 2:
                    s_cmp.wait_event(out_done[i - 2])
                step_on(bs, s_cmp.cuda_stream)
                cmp_done.append(ev()); cmp_done[-1].record(s_cmp)
                with torch.cuda.stream(s_out):  # results of step i
                    s_out.wait_event(cmp_done[i])
                    for n in out_names:
                        host_out[n].copy_(bs[n], non_blocking=True)
                    out_done.append(ev()); out_done[-1].record(s_out)
            e1.record(s_out)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / nsteps

        pipeline(3, False)  # warm-up
        e2e_ms = max_over_ranks(pipeline(max(10, min(K, 40)), True), dist, dev)
        e2e = {"value": aggregate_rate(B * T * C, ws_n, e2e_ms), "unit": "channel-tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "pipelined": "copies of adjacent steps overlap compute and each other"}

    if rank == 0:
        units = B * T * C
        hbm, peak_kind = peaks()
        fwd_ms = statistics.mean(t_fwd)
        bwd_ms = statistics.mean(t_bwd)
        sfx = "_gated" if args.gate else ""
        fb = ALG_BYTES[("fwd" + sfx, inp["dtype"])] * units
        bb = ALG_BYTES[("bwd" + sfx, inp["dtype"])] * units
        bwd_gbs = bb / (bwd_ms * 1e-3) / 1e9
        fwd_gbs = fb / (fwd_ms * 1e-3) / 1e9
        step_ms = total_ms / K
        bwd_names, bwd_launches = BWD_PLAN[args.bwd_kernel]
        fwd_names, fwd_launches = FWD_PLAN[args.fwd_kernel]
        main_bwd = bwd_names.split(" + ")[0]
        traffic = TRAFFIC.get((args.workload, main_bwd, bool(args.gate)))
        line = {
            "metric": metric_name(args.gate),
            "value": aggregate_rate(units, ws_n, step_ms), "unit": "channel-tokens/s",
            "n_gpus": ws_n, "steps": K, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": inp["dtype"], "data": "synthetic (seeded; the RWKV-4 layer shapes and value ranges)",
            "config": {"workload": args.workload, "B": B, "T": T, "C": C,
                       **({"gate": True} if args.gate else {}),
                       "parallelism": f"replicas x{ws_n}" if ws_n > 1 else "single GPU",
                       "l2": "flushed before every timed step (2x L2 write + 2x L2 read, outside events)"},
            "roofline": {"bound": "hbm",
                         "kernel": f"wkv_backward{sfx} call ({bwd_names}), timed as one call",
                         "achieved": bwd_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": bwd_gbs / hbm, "traffic": traffic,
                         "traffic_kernel": main_bwd if traffic else None,
                         "algorithmic_bytes": bb, "peak_kind": peak_kind},
            "fwd": {"kernels": fwd_names, "ms": fwd_ms, "gbs": fwd_gbs, "frac": fwd_gbs / hbm,
                    "channel_tokens_per_s": units / (fwd_ms * 1e-3)},
            "bwd": {"kernels": bwd_names, "ms": bwd_ms, "gbs": bwd_gbs, "frac": bwd_gbs / hbm},
            "fwd_bwd_gbs": (fb + bb) / (step_ms * 1e-3) / 1e9,
            "clocks": clocks, "gpu_launches": (fwd_launches + bwd_launches) * K,
            "device_status": status,
        }
        if e2e:
            line["e2e"] = e2e
        if not args.no_cpu_baseline and ws_n == 1:
            line["cpu_baseline"] = cpu_baseline(args.workload, min_seconds=args.cpu_seconds,
                                                gate=args.gate)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_token_shift(args):
    """--token-shift: the three time-mixing interpolations (n = 3) of the
    workload's layer shape, forward then backward, through the C ABI."""
    import torch
    import rwkv_linear_rnn_b200 as W
    from rwkv_linear_rnn_b200 import abi

    ws_n, rank, local = dist_env()
    dist = None
    if ws_n > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = workloads.WORKLOADS[args.workload]
    B, T, C, n = wl.B, wl.T, wl.C, 3
    dt = W.WKV_BF16 if wl.dtype == "bf16" else W.WKV_F32
    tdt = torch.bfloat16 if dt == W.WKV_BF16 else torch.float32
    es = 2 if dt == W.WKV_BF16 else 4
    gen = torch.Generator(device="cpu").manual_seed(wl.seed + 1000 * rank)
    x = torch.randn((B, T, C), generator=gen).to(dev, tdt)
    xp = torch.randn((B, C), generator=gen).to(dev, tdt)
    mu = torch.rand((n, C), generator=gen).to(dev)
    g = torch.randn((n, B, T, C), generator=gen).to(dev, tdt)
    out = torch.empty((n, B, T, C), device=dev, dtype=tdt)
    gx = torch.empty_like(x)
    gmu = torch.empty((n, C), device=dev)
    gxp = torch.empty_like(xp)
    nws = abi.wkv_token_shift_workspace_size(B, T, C, n)
    wsb = torch.empty(nws, dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_w = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(2 * l2 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    P = lambda t: t.data_ptr()

    def fwd():
        abi.check(abi.wkv_token_shift(B, T, C, dt, n, P(mu), P(x), P(xp), P(out), sp))

    def bwd():
        abi.check(abi.wkv_token_shift_backward(B, T, C, dt, n, P(mu), P(x), P(xp), P(g), P(gx), P(gmu),
                                               P(gxp), P(wsb), nws, sp))

    for _ in range(args.warmup):
        flush_w.zero_(); flush_r.sum(); fwd(); bwd()
    torch.cuda.synchronize()
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_begin = time.monotonic()
    for i in range(K):
        flush_w.zero_(); flush_r.sum()
        ev[i][0].record(stream); fwd(); ev[i][1].record(stream); bwd(); ev[i][2].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop(window=(t_begin, time.monotonic()))
    if dist:
        dist.barrier()
    t_fwd = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    t_bwd = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    total_ms = max_over_ranks(sum(t_fwd) + sum(t_bwd), dist, dev)

    e2e = None
    if not args.no_e2e:
        hx = x.cpu().pin_memory(); hg = g.cpu().pin_memory()
        hout = torch.empty_like(out, device="cpu").pin_memory(); hgx = torch.empty_like(hx).pin_memory()
        hgmu = torch.empty((n, C)).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hx, hg))
        d2h = sum(t.numel() * t.element_size() for t in (hout, hgx, hgmu))
        ee = []
        for i in range(max(3, min(K, 10)) + 1):
            e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            x.copy_(hx, non_blocking=True); g.copy_(hg, non_blocking=True)
            fwd(); bwd()
            hout.copy_(out, non_blocking=True); hgx.copy_(gx, non_blocking=True)
            hgmu.copy_(gmu, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if i > 0:
                ee.append(e0.elapsed_time(e1))
        e2e_ms = max_over_ranks(statistics.median(ee), dist, dev)
        e2e = {"value": aggregate_rate(B * T * C, ws_n, e2e_ms), "unit": "channel-tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    if rank == 0:
        units = B * T * C
        hbm, peak_kind = peaks()
        fwd_ms, bwd_ms = statistics.mean(t_fwd), statistics.mean(t_bwd)
        fb = (1 + n) * es * units           # x read, n outputs written
        bb = (2 + n) * es * units           # x, n gradients read, grad_x written
        fwd_gbs = fb / (fwd_ms * 1e-3) / 1e9
        bwd_gbs = bb / (bwd_ms * 1e-3) / 1e9
        step_ms = total_ms / K
        line = {
            "metric": "token-shift fwd+bwd channel-tokens/s (3 interpolations; HBM GB/s alongside)",
            "value": aggregate_rate(units, ws_n, step_ms), "unit": "channel-tokens/s",
            "n_gpus": ws_n, "steps": K, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
            "data": "synthetic (seeded normal x, uniform mu)",
            "config": {"workload": args.workload, "op": "token_shift", "B": B, "T": T, "C": C, "n": n,
                       "parallelism": f"replicas x{ws_n}" if ws_n > 1 else "single GPU",
                       "l2": "flushed before every timed step (2x L2 write + 2x L2 read, outside events)"},
            "roofline": {"bound": "hbm", "kernel": "wkv_token_shift_backward call, timed as one call",
                         "achieved": bwd_gbs, "peak": hbm, "unit": "GB/s", "frac": bwd_gbs / hbm,
                         "traffic": None, "algorithmic_bytes": bb, "peak_kind": peak_kind},
            "fwd": {"ms": fwd_ms, "gbs": fwd_gbs, "frac": fwd_gbs / hbm},
            "bwd": {"ms": bwd_ms, "gbs": bwd_gbs, "frac": bwd_gbs / hbm},
            "clocks": clocks, "gpu_launches": 3 * K,
        }
        if e2e:
            line["e2e"] = e2e
        if not args.no_cpu_baseline and ws_n == 1:
            line["cpu_baseline"] = token_shift_cpu_baseline(args.workload, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)  # about a second: clock samples land inside
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libwkv", choices=["libwkv", "reference"])
    ap.add_argument("--workload", default="rwkv169m")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--fwd-kernel", default="auto", choices=sorted(FWD_PLAN))
    ap.add_argument("--bwd-kernel", default="auto", choices=sorted(BWD_PLAN))
    ap.add_argument("--gate", action="store_true",
                    help="time the gated calls (o = sigmoid(r) * wkv and its gradients)")
    ap.add_argument("--token-shift", action="store_true",
                    help="time the token shift (3 interpolations) on the workload's layer shape")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # timing rule: at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    elif args.token_shift:
        run_token_shift(args)
    else:
        run_libwkv(args)


if __name__ == "__main__":
    main()
