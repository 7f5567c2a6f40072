"""Benchmark: WKV channel-tokens/s and achieved HBM GB/s on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libwkv|reference]
                [--workload rwkv1b5_bf16|rwkv169m|longctx|decode14b|tiny]
                [--gate | --token-shift]

A step is one pass of the hot path over one batch of the workload, through
the C ABI, with the inputs resident in HBM:

* fwd+bwd workloads (the default, the RWKV-4 1.5B-shaped layer B8 T4096
  C2048 with bf16 I/O; also rwkv169m, tiny): ``wkv_forward`` (writing the
  checkpoints) then ``wkv_backward``; value = channel-tokens/s of the pair;
* ``longctx`` (B1 T65536 C2560 fp32, forward only): ``wkv_forward``;
* ``decode14b`` (512 sequences x C5120 fp32): after an untimed T128 prefill,
  32 ``wkv_step`` calls, each with its own pre-staged k_t, v_t, y_t buffers
  and the state updated in place; value = channel-steps/s over the 32 steps.

L2 is flushed (a 2x-L2 buffer is written, then another read) before every
timed step, outside the timed events; every kernel call is bracketed by CUDA
events on the launching stream.  ``--gate`` times the gated calls;
``--token-shift`` the token shift (three interpolations) on the workload's
layer shape.

Multi-GPU (torchrun): every rank runs an independent replica of the workload
on its own GPU (the operator has no cross-sequence exchange; weak scaling);
ranks are timed on the device and the maximum over ranks is reported.

``--impl reference`` times the float64 CPU oracle (the only reference this
operator has) on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import re
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

CSRC = os.path.join(ROOT, "rwkv_linear_rnn_b200", "csrc")

# algorithmic bytes per channel-token (per channel-step for the decode step)
# (gated: the forward also reads r; the backward reads r and writes grad_r)
ALG_BYTES = {("fwd", "f32"): 12, ("fwd", "bf16"): 6, ("bwd", "f32"): 20, ("bwd", "bf16"): 10,
             ("fwd_gated", "f32"): 16, ("fwd_gated", "bf16"): 8, ("bwd_gated", "f32"): 28,
             ("bwd_gated", "bf16"): 14, ("step", "f32"): 36}

# Kernels each call launches on 16-byte aligned rows (every bench workload):
# (kernel name, launches per call) per kernel selector.  The gated and
# state-gradient backwards run the segment kernel.
FWD_PLAN = {"tile": ("fwd_tile_kernel", 1), "segment": ("fwd_seg_kernel", 1), "cluster": ("fwd_clu_kernel", 1),
            "chain": ("fwd_chain_kernel", 1)}
BWD_PLAN = {"tile": ("bwd_tile_kernel", 1), "segment": ("bwd_seg_kernel", 1), "chain": ("bwd_chain_kernel", 1)}


def auto_kernel(op: str, B: int, C: int, gate: bool, num_sms: int = 148) -> str:
    """The kernel the library's AUTO selector runs on 16-byte aligned rows of
    at least one tile unit (mirrors chain_pays and tile_pays in the C ABI):
    the chain kernels when the chains (batch row, 32 channels) occupy 60 %
    or more of the warp schedulers (in one wave or several); else the tile
    kernels when a chain has at most about four resident warps' units in
    flight; else the segment kernels."""
    nchains = B * ((C + 31) // 32)
    slots = 4 * num_sms
    if nchains * 5 >= slots * 3:
        return "chain"
    warps = (6 if gate else 9) if op == "fwd" else (6 if gate else 8)
    return "tile" if nchains * 4 >= warps * num_sms else "segment"
KERNEL_IDS = {"auto": 0, "segment": 6, "cluster": 7, "tile": 8, "chain": 9}

# The source files each kernel is built from: a DRAM-traffic figure measured
# by ncu is reported only while these files are unchanged since the capture.
KERNEL_SOURCES = {
    "fwd_tile_kernel": ["wkv_tile.cu", "wkv_tile.cuh", "wkv_internal.cuh", "wkv_math.cuh", "wkv_forward.cu"],
    "bwd_tile_kernel": ["wkv_tile_bwd.cu", "wkv_tile.cuh", "wkv_bwd_math.cuh", "wkv_internal.cuh",
                        "wkv_math.cuh", "wkv_forward.cu"],
    "bwd_seg_kernel": ["wkv_seg_bwd.cu", "wkv_ring.cuh", "wkv_bwd_math.cuh", "wkv_internal.cuh",
                       "wkv_math.cuh", "wkv_forward.cu"],
    "fwd_seg_kernel": ["wkv_seg.cu", "wkv_ring.cuh", "wkv_internal.cuh", "wkv_math.cuh", "wkv_forward.cu"],
    "fwd_chain_kernel": ["wkv_chain.cu", "wkv_tile.cuh", "wkv_internal.cuh", "wkv_math.cuh", "wkv_forward.cu"],
    "bwd_chain_kernel": ["wkv_chain.cu", "wkv_tile.cuh", "wkv_bwd_math.cuh", "wkv_internal.cuh", "wkv_math.cuh",
                         "wkv_forward.cu"],
    "step_kernel": ["wkv_step.cu", "wkv_internal.cuh"],
    "linattn_backward": ["linattn.cu", "wkv_forward.cu", "wkv_tile.cuh", "wkv_internal.cuh"],
    "linattn_backward_saved": ["linattn.cu", "wkv_forward.cu", "wkv_tile.cuh", "wkv_internal.cuh"],
}

# DRAM bytes (read + write) per launch of a workload's dominant kernel, from
# one ncu capture (the summaries under profiles/ give the commands), keyed by
# (workload, kernel, gated, hash of the kernel's code).  A kernel whose code changed
# since its capture has no entry: its traffic is reported as null.
TRAFFIC = {
    ("rwkv1b5_bf16", "bwd_chain_kernel", False, "dd3bb205f2bafacc"): 453_355_776 + 212_812_800,
    ("rwkv1b5_bf16", "fwd_chain_kernel", False, "f67c813868e39fed"): 268_525_056 + 131_096_576,
    ("rwkv1b5_bf16", "bwd_chain_kernel", True, "dd3bb205f2bafacc"): 587_434_752 + 345_717_504,
    ("rwkv1b5_bf16", "fwd_chain_kernel", True, "f67c813868e39fed"): 402_733_824 + 132_948_224,
    ("rwkv169m", "bwd_seg_kernel", False, "f3ee2d2581da2ffd"): 77_673_472 + 485_376,
    ("rwkv169m", "fwd_seg_kernel", False, "fbcb48b606b747e2"): 50_391_552 + 1_572_608,
    ("longctx", "fwd_seg_kernel", False, "fbcb48b606b747e2"): 1_454_121_728 + 638_856_704,
    ("decode14b", "step_kernel", False, "5da4a196be76b807"): (1_679_439_616 + 4_633_856) // 32,
    # the three launches of one linattn_backward_saved call
    ("la_cifar_b32", "linattn_backward_saved", False, "d137bd8b0b6bb8ce"): (154_165_248 + 27_663_616 + 25_963_008
                                                                           + 256_460_288 + 107_953_408),
}


def _code_only(text: str) -> str:
    """Source without comments and blank lines: what the compiler sees
    (string literals in these files hold no comment markers)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_hash(kernel: str) -> str:
    """Hash of the code (comments excluded) of the files a kernel is built from."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def workload_mode(name: str) -> str:
    ops = workloads.WORKLOADS[name].ops
    if "step" in ops:
        return "step"
    return "fwdbwd" if "bwd" in ops else "fwd"


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


# ------------------------------------------------------------- descriptions ---

def metric_name(mode: str, gate: bool) -> str:
    what = "gated WKV" if gate else "WKV"
    if mode == "fwd":
        return f"{what} fwd channel-tokens/s, long-context scan (HBM GB/s and % of roofline alongside)"
    if mode == "step":
        return "WKV decode-step channel-steps/s, RNN mode (HBM GB/s and % of roofline alongside)"
    return f"{what} fwd+bwd channel-tokens/s (HBM GB/s and % of roofline alongside)"


def units_per_step(wl) -> int:
    """Channel-tokens (channel-steps for the decode workload) of one step."""
    if workload_mode(wl.name) == "step":
        return wl.B * wl.C * wl.steps
    return wl.B * wl.T * wl.C


def make_config(args, wl, ws_n: int) -> dict:
    """The workload description both arms print."""
    mode = workload_mode(wl.name)
    cfg = {"workload": wl.name, "mode": mode, "io_dtype": wl.dtype}
    if mode == "step":
        cfg.update({"N": wl.B, "C": wl.C, "prefill_T": wl.T, "steps": wl.steps,
                    "l2": "flushed once before the 32 timed steps (outside events); the state is updated in place"})
    else:
        cfg.update({"B": wl.B, "T": wl.T, "C": wl.C,
                    "l2": "flushed before every timed step (2x L2 write + 2x L2 read, outside events)"})
    if args.gate:
        cfg["gate"] = True
    cfg["parallelism"] = f"replicas x{ws_n}" if ws_n > 1 else "single GPU"
    return cfg


# ------------------------------------------------------------- CPU baseline ---

def _time_loop(fn, min_seconds: float, min_reps: int = 3):
    times = []
    t_end = time.perf_counter() + min_seconds
    while time.perf_counter() < t_end or len(times) < min_reps:
        t0 = time.perf_counter()
        fn()
        times.append(time.perf_counter() - t0)
    return statistics.median(times), len(times)


def cpu_baseline(wl_name: str, min_seconds: float = 10.0, gate: bool = False):
    """Time the oracle (float64) on the host on a bounded sample of the
    workload: the recurrence forward (+ the reverse-time backward for the
    fwd+bwd workloads), or the decode step.  Reported on all host threads
    (OpenMP over the independent chains) and on one thread."""
    import oracle
    wl = workloads.WORKLOADS[wl_name]
    mode = workload_mode(wl_name)
    if mode == "step":
        N, C = 512, 512
        d = workloads.generate_decode_steps(wl, N=N, C=C, steps=2)
        w, u = np.asarray(d["w"], np.float64), np.asarray(d["u"], np.float64)
        _, st = oracle.fwd_recur(d["w"], d["u"], d["k"], d["v"], want_y=False)
        kt, vt = np.asarray(d["k_steps"][0], np.float64), np.asarray(d["v_steps"][0], np.float64)
        fn = lambda: oracle.step(w, u, kt, vt, st)
        units = N * C
        sample = f"decode14b slice N={N} C={C}, one step after the T128 prefill"
        unit = "channel-steps/s"
    else:
        what = "gated fwd+bwd" if gate else ("fwd+bwd" if mode == "fwdbwd" else "fwd")
        if wl_name in ("rwkv169m", "tiny"):
            inp = workloads.generate(wl, gate=gate)
            sample = f"full {wl_name} workload (B{wl.B} T{wl.T} C{wl.C}) {what}"
        else:  # a channel slice of the big workloads keeps the sample bounded
            C = 128 if mode == "fwd" else 256
            inp = workloads.generate(wl, C=C, T=min(wl.T, 65536 if mode == "fwd" else 4096),
                                     grad=mode == "fwdbwd", gate=gate)
            sample = f"{wl_name} with C={C}, T={inp['T']} {what}"
        names = ("w", "u", "k", "v", "r", "gy") if gate else ("w", "u", "k", "v", "gy")
        args = [np.asarray(inp[n], np.float64) for n in names if n in inp]
        units = inp["B"] * inp["T"] * inp["C"]
        unit = "channel-tokens/s"
        if mode == "fwd":
            fn = lambda: oracle.fwd_recur(*args[:4], want_y=True)
        elif gate:
            fn = lambda: (oracle.fwd_gated(*args[:5]), oracle.bwd_gated(*args))
        else:
            fn = lambda: (oracle.fwd_recur(*args[:4], want_y=True), oracle.bwd_recur(*args))
    cores = oracle.num_threads()
    med, reps = _time_loop(fn, min_seconds)
    oracle.set_threads(1)
    try:
        med1, reps1 = _time_loop(fn, max(1.0, min_seconds / 4), min_reps=1)
    finally:
        oracle.set_threads(cores)
    return {"value": units / med, "unit": unit, "cores": cores, "kind": "oracle",
            "sample": f"{sample}, x{reps}, median",
            "single_thread": {"value": units / med1, "unit": unit, "cores": 1,
                              "sample": f"{sample}, x{reps1}, median"}}


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
    med, reps = _time_loop(lambda: (ots.shift(x, mu, xp), ots.shift_bwd(x, mu, g, xp)), min_seconds)
    return {"value": B * T * C / med, "unit": "channel-tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{wl_name} token shift (B{B} T{T} C{C}, n=3) fwd+bwd x{reps}, median"}


def token_shift_config(args, wl, ws_n):
    return {"workload": args.workload, "op": "token_shift", "B": wl.B, "T": wl.T, "C": wl.C, "n": 3,
            "io_dtype": wl.dtype, "parallelism": f"replicas x{ws_n}" if ws_n > 1 else "single GPU",
            "l2": "flushed before every timed step (2x L2 write + 2x L2 read, outside events)"}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    wl = workloads.WORKLOADS[args.workload]
    secs = max(1.0, 2.0 * args.steps)
    if args.token_shift:
        cb = token_shift_cpu_baseline(args.workload, min_seconds=secs)
        metric = "token-shift fwd+bwd channel-tokens/s (3 interpolations; HBM GB/s alongside)"
        cfg = token_shift_config(args, wl, 1)
        units = wl.B * wl.T * wl.C
    else:
        cb = cpu_baseline(args.workload, min_seconds=secs, gate=args.gate)
        metric = metric_name(workload_mode(args.workload), args.gate)
        cfg = make_config(args, wl, 1)
        units = units_per_step(wl)
    line = {"metric": metric, "value": cb["value"], "unit": cb["unit"], "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": units / cb["value"] * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "impl": "reference", "config": cfg,
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": cb["unit"], "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_linattn_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    wl = workloads.LINATTN_WORKLOADS[args.workload]
    cb = linattn_cpu_baseline(args.workload, max(1.0, 2.0 * args.steps))
    line = {"metric": "causal linear attention fwd+bwd head-positions/s (HBM GB/s and % of roofline alongside)",
            "value": cb["value"], "unit": cb["unit"], "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": wl.BH * wl.N / cb["value"] * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "impl": "reference", "config": linattn_config(wl, 1, not args.la_recompute),
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": cb["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- GPU arm ---

def setup_device():
    import torch
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
    return ws_n, rank, dist, dev


def make_flush(dev):
    import torch
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_w = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(2 * l2 // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # write 2x L2 (evicts everything), then read another 2x L2 so the
        # lines left behind are clean: the timed kernels neither hit their
        # inputs in L2 nor pay for write-backs of the flush
        flush_w.zero_()
        flush_r.sum()
    return flush_l2


def pipeline_e2e(nsteps, timed, in_names, out_names, host_in, host_out, sets, step_on, streams):
    """Steps pipelined over three streams (PCIe is full duplex): step i+1's
    inputs are copied in while step i computes and step i's results are
    copied out; device tensors are double buffered and events order each
    buffer's reuse.  Returns ms per step (first H2D start to last D2H end)."""
    import torch
    s_in, s_cmp, s_out = streams
    ev = lambda: torch.cuda.Event(enable_timing=timed)
    in_done, cmp_done, out_done = [], [], []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(nsteps):
        bs = sets[i % 2]
        hin = host_in[i % len(host_in)]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(cmp_done[i - 2])
            for n in in_names:
                bs[n].copy_(hin[n], non_blocking=True)
            in_done.append(ev()); in_done[-1].record(s_in)
        s_cmp.wait_event(in_done[i])
        if i >= 2:
            s_cmp.wait_event(out_done[i - 2])
        step_on(bs, s_cmp.cuda_stream, i)
        cmp_done.append(ev()); cmp_done[-1].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[i])
            for n in out_names:
                host_out[n].copy_(bs[n], non_blocking=True)
            out_done.append(ev()); out_done[-1].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / nsteps


def traffic_for(workload, kernel, gated):
    return TRAFFIC.get((workload, kernel, bool(gated), kernel_hash(kernel)))


def run_libwkv(args):
    mode = workload_mode(args.workload)
    if mode == "step":
        return run_step(args)
    import torch
    import rwkv_linear_rnn_b200 as W
    from rwkv_linear_rnn_b200 import abi

    ws_n, rank, dist, dev = setup_device()
    wl = workloads.WORKLOADS[args.workload]
    with_bwd = mode == "fwdbwd"
    inp = workloads.generate(wl, seed=wl.seed + 1000 * rank, gate=args.gate, grad=with_bwd)
    B, T, C = inp["B"], inp["T"], inp["C"]
    dt = W.WKV_BF16 if inp["dtype"] == "bf16" else W.WKV_F32

    def to_dev(name):
        if dt == W.WKV_BF16 and name in ("k", "v", "gy", "r"):
            return torch.from_numpy(inp[name + "_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(inp[name]).to(dev)

    w, u, k, v = (to_dev(n) for n in ("w", "u", "k", "v"))
    del inp["k"], inp["v"]
    gy = to_dev("gy") if with_bwd else None
    r = to_dev("r") if args.gate else None
    gr = torch.empty_like(k) if args.gate and with_bwd else None
    y = torch.empty_like(k)
    gk = torch.empty_like(k) if with_bwd else None
    gv = torch.empty_like(v) if with_bwd else None
    gw = torch.empty(C, device=dev)
    gu = torch.empty(C, device=dev)
    state = torch.empty(3, B, C, device=dev)
    ckpt = torch.empty(W.wkv_ckpt_size(B, T, C) // 4, device=dev) if with_bwd else None
    nws = W.wkv_workspace_size(W.WKV_OP_BACKWARD if with_bwd else W.WKV_OP_FORWARD, B, T, C, dt)
    wsb = torch.zeros(nws, dtype=torch.uint8, device=dev)
    flush_l2 = make_flush(dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    P = lambda t: 0 if t is None else t.data_ptr()
    fopt = abi.Options(kernel=KERNEL_IDS[args.fwd_kernel])
    bopt = abi.Options(kernel=KERNEL_IDS[args.bwd_kernel])

    def fwd(bs, sp_):
        if args.gate:
            abi.check(abi.wkv_forward_gated_ex(B, T, C, dt, P(w), P(u), P(bs["k"]), P(bs["v"]), P(bs["r"]), 0,
                                               P(bs["y"]), P(bs["state"]), P(ckpt), P(wsb), nws, sp_, fopt))
        else:
            abi.check(abi.wkv_forward_ex(B, T, C, dt, P(w), P(u), P(bs["k"]), P(bs["v"]), 0, P(bs["y"]),
                                         P(bs["state"]), P(ckpt), P(wsb), nws, sp_, fopt))

    def bwd(bs, sp_):
        if args.gate:
            abi.check(abi.wkv_backward_gated_ex(B, T, C, dt, P(w), P(u), P(bs["k"]), P(bs["v"]), P(bs["r"]),
                                                P(bs["gy"]), 0, P(ckpt), P(bs["gw"]), P(bs["gu"]), P(bs["gk"]),
                                                P(bs["gv"]), P(bs["gr"]), P(wsb), nws, sp_, bopt))
        else:
            abi.check(abi.wkv_backward_ex(B, T, C, dt, P(w), P(u), P(bs["k"]), P(bs["v"]), P(bs["gy"]), 0,
                                          P(ckpt), P(bs["gw"]), P(bs["gu"]), P(bs["gk"]), P(bs["gv"]), P(wsb),
                                          nws, sp_, bopt))

    resident = {"k": k, "v": v, "gy": gy, "r": r, "y": y, "gk": gk, "gv": gv, "gw": gw, "gu": gu, "gr": gr,
                "state": state}
    for _ in range(args.warmup):
        flush_l2()
        fwd(resident, sp)
        if with_bwd:
            bwd(resident, sp)
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
        fwd(resident, sp)
        ev[i][1].record(stream)
        if with_bwd:
            bwd(resident, sp)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop(window=(t_begin, time.monotonic()))
    if dist:
        dist.barrier()
    t_fwd = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    t_bwd = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    total_ms = max_over_ranks(sum(t_fwd) + sum(t_bwd), dist, dev)
    status = abi.wkv_get_status(P(wsb), sp)

    e2e = None
    if not args.no_e2e:
        in_names = ["k", "v"] + (["gy"] if with_bwd else []) + (["r"] if args.gate else [])
        out_names = (["y", "gk", "gv", "gw", "gu"] + (["gr"] if args.gate else [])) if with_bwd else ["y", "state"]
        host_in = [{n: resident[n].cpu().pin_memory() for n in in_names}]
        host_out = {n: torch.empty_like(resident[n], device="cpu").pin_memory() for n in out_names}
        sets = [{n: torch.empty_like(resident[n]) for n in in_names + out_names + (["state"] if with_bwd else [])}
                for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
        d2h = sum(t.numel() * t.element_size() for t in host_out.values())
        streams = (torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream())

        def step_on(bs, sp_, i):
            fwd(bs, sp_)
            if with_bwd:
                bwd(bs, sp_)
        pipeline_e2e(3, False, in_names, out_names, host_in, host_out, sets, step_on, streams)
        e2e_ms = max_over_ranks(pipeline_e2e(max(10, min(K, 40)), True, in_names, out_names, host_in, host_out,
                                             sets, step_on, streams), dist, dev)
        e2e = {"value": aggregate_rate(B * T * C, ws_n, e2e_ms), "unit": "channel-tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "pipelined": "copies of adjacent steps overlap compute and each other"}

    if rank == 0:
        units = B * T * C
        hbm, peak_kind = peaks()
        fwd_ms = statistics.mean(t_fwd)
        sfx = "_gated" if args.gate else ""
        io = inp["dtype"]
        fb = ALG_BYTES[("fwd" + sfx, io)] * units
        fwd_gbs = fb / (fwd_ms * 1e-3) / 1e9
        step_ms = total_ms / K
        nsm = torch.cuda.get_device_properties(dev).multi_processor_count
        fsel = auto_kernel("fwd", B, C, args.gate, nsm) if args.fwd_kernel == "auto" else args.fwd_kernel
        bsel = auto_kernel("bwd", B, C, args.gate, nsm) if args.bwd_kernel == "auto" else args.bwd_kernel
        fwd_names, fwd_launches = FWD_PLAN[fsel]
        bwd_names, bwd_launches = BWD_PLAN[bsel]
        line = {
            "metric": metric_name(mode, args.gate),
            "value": aggregate_rate(units, ws_n, step_ms), "unit": "channel-tokens/s",
            "n_gpus": ws_n, "steps": K, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic (seeded; the RWKV-4 layer shapes and value ranges)",
            "config": make_config(args, wl, ws_n),
            "fwd": {"kernels": fwd_names, "ms": fwd_ms, "gbs": fwd_gbs, "frac": fwd_gbs / hbm,
                    "channel_tokens_per_s": units / (fwd_ms * 1e-3), "algorithmic_bytes": fb,
                    "traffic": traffic_for(args.workload, fwd_names, args.gate)},
            "clocks": clocks, "device_status": status,
            "gpu_launches": (fwd_launches + (bwd_launches if with_bwd else 0)) * K,
        }
        if with_bwd:
            bwd_ms = statistics.mean(t_bwd)
            bb = ALG_BYTES[("bwd" + sfx, io)] * units
            bwd_gbs = bb / (bwd_ms * 1e-3) / 1e9
            line["bwd"] = {"kernels": bwd_names, "ms": bwd_ms, "gbs": bwd_gbs, "frac": bwd_gbs / hbm,
                           "algorithmic_bytes": bb}
            line["fwd_bwd_gbs"] = (fb + bb) / (step_ms * 1e-3) / 1e9
            dom, dom_ms, dom_b, dom_gbs = bwd_names, bwd_ms, bb, bwd_gbs
            call = f"wkv_backward{sfx}"
        else:
            dom, dom_ms, dom_b, dom_gbs = fwd_names, fwd_ms, fb, fwd_gbs
            call = f"wkv_forward{sfx}"
        traffic = traffic_for(args.workload, dom, args.gate)
        line["roofline"] = {"bound": "hbm", "kernel": f"{call} call ({dom}), timed as one call with CUDA events",
                            "achieved": dom_gbs, "peak": hbm, "unit": "GB/s", "frac": dom_gbs / hbm,
                            "traffic": traffic, "traffic_kernel": dom if traffic else None,
                            "algorithmic_bytes": dom_b, "ms": dom_ms, "peak_kind": peak_kind}
        if e2e:
            line["e2e"] = e2e
        if not args.no_cpu_baseline and ws_n == 1:
            line["cpu_baseline"] = cpu_baseline(args.workload, min_seconds=args.cpu_seconds, gate=args.gate)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_step(args):
    """decode14b: an untimed T128 prefill sets the state of N sequences; a
    step is 32 wkv_step calls, each with its own k_t, v_t, y_t buffers."""
    import torch
    import rwkv_linear_rnn_b200 as W
    from rwkv_linear_rnn_b200 import abi

    ws_n, rank, dist, dev = setup_device()
    wl = workloads.WORKLOADS[args.workload]
    d = workloads.generate_decode_steps(wl, seed=wl.seed + 1000 * rank)
    N, T0, C, S = d["N"], d["T"], d["C"], wl.steps
    w = torch.from_numpy(d["w"]).to(dev)
    u = torch.from_numpy(d["u"]).to(dev)
    kp = torch.from_numpy(d["k"]).to(dev)
    vp = torch.from_numpy(d["v"]).to(dev)
    ks = torch.from_numpy(d["k_steps"]).to(dev)
    vs = torch.from_numpy(d["v_steps"]).to(dev)
    ys = torch.empty_like(ks)
    state0 = torch.empty(3, N, C, device=dev)
    state = torch.empty_like(state0)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    P = lambda t: t.data_ptr()
    yp = torch.empty_like(kp)
    nws = W.wkv_workspace_size(W.WKV_OP_FORWARD, N, T0, C, W.WKV_F32)
    wsb = torch.zeros(max(nws, 256), dtype=torch.uint8, device=dev)
    abi.check(abi.wkv_forward(N, T0, C, W.WKV_F32, P(w), P(u), P(kp), P(vp), 0, P(yp), P(state0), 0, P(wsb),
                              nws, sp))
    del kp, vp, yp
    flush_l2 = make_flush(dev)

    def one(i, kt, vt, yt, sp_):
        abi.check(abi.wkv_step(N, C, P(w), P(u), P(kt), P(vt), P(state), P(yt), P(state), sp_))

    for _ in range(args.warmup):
        state.copy_(state0)
        flush_l2()
        for i in range(S):
            one(i, ks[i], vs[i], ys[i], sp)
    torch.cuda.synchronize()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(S + 1)] for _ in range(K)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_begin = time.monotonic()
    for it in range(K):
        state.copy_(state0)  # every timed step decodes from the prefill state
        flush_l2()
        ev[it][0].record(stream)
        for i in range(S):
            one(i, ks[i], vs[i], ys[i], sp)
            ev[it][i + 1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop(window=(t_begin, time.monotonic()))
    if dist:
        dist.barrier()
    per_call = [ev[it][i].elapsed_time(ev[it][i + 1]) for it in range(K) for i in range(S)]
    seq = [ev[it][0].elapsed_time(ev[it][S]) for it in range(K)]
    total_ms = max_over_ranks(sum(seq), dist, dev)
    # the same step kernel with L2 flushed before every call (each call's
    # state then comes from HBM): a per-call figure free of L2 reuse
    flushed = []
    for it in range(min(K, 5)):
        state.copy_(state0)
        for i in range(S):
            flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            one(i, ks[i], vs[i], ys[i], sp)
            e1.record(stream)
            flushed.append((e0, e1))
    torch.cuda.synchronize()
    flushed_ms = statistics.mean(a.elapsed_time(b) for a, b in flushed)

    e2e = None
    if not args.no_e2e:
        # each call's k_t, v_t come from pinned host memory and its y_t goes
        # back; the state stays resident (it is the decoder's own state)
        host_in = [{"kt": ks[i].cpu().pin_memory(), "vt": vs[i].cpu().pin_memory()} for i in range(S)]
        host_out = {"yt": torch.empty_like(ys[0], device="cpu").pin_memory()}
        sets = [{"kt": torch.empty_like(ks[0]), "vt": torch.empty_like(vs[0]), "yt": torch.empty_like(ys[0])}
                for _ in range(2)]
        streams = (torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream())

        def step_on(bs, sp_, i):
            one(i, bs["kt"], bs["vt"], bs["yt"], sp_)
        state.copy_(state0)
        pipeline_e2e(3, False, ["kt", "vt"], ["yt"], host_in, host_out, sets, step_on, streams)
        state.copy_(state0)
        torch.cuda.synchronize()
        call_ms = max_over_ranks(pipeline_e2e(S, True, ["kt", "vt"], ["yt"], host_in, host_out, sets, step_on,
                                              streams), dist, dev)
        e2e = {"value": aggregate_rate(N * C, ws_n, call_ms), "unit": "channel-steps/s",
               "h2d_bytes_per_step": S * 2 * N * C * 4, "d2h_bytes_per_step": S * N * C * 4,
               "ms_per_step": call_ms * S,
               "pipelined": "each call's k_t, v_t copied in while the previous call computes; y_t copied out"}

    if rank == 0:
        hbm, peak_kind = peaks()
        step_ms = total_ms / K
        call_ms_dev = statistics.mean(per_call)
        b_call = ALG_BYTES[("step", "f32")] * N * C
        gbs = b_call / (call_ms_dev * 1e-3) / 1e9
        gbs_flushed = b_call / (flushed_ms * 1e-3) / 1e9
        traffic = traffic_for(args.workload, "step_kernel", False)
        line = {
            "metric": metric_name("step", False),
            "value": aggregate_rate(N * C * S, ws_n, step_ms), "unit": "channel-steps/s",
            "n_gpus": ws_n, "steps": K, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded; RWKV-4 14B-shaped decode batch)",
            "config": make_config(args, wl, ws_n),
            "roofline": {"bound": "hbm", "kernel": "wkv_step call (step_kernel), mean of the 32 calls of a step",
                         "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm, "traffic": traffic,
                         "traffic_kernel": "step_kernel" if traffic else None, "algorithmic_bytes": b_call,
                         "ms": call_ms_dev, "peak_kind": peak_kind,
                         "note": "the state written by one call is partly still in L2 when the next reads it"},
            "step_l2_flushed_each_call": {"ms": flushed_ms, "gbs": gbs_flushed, "frac": gbs_flushed / hbm},
            "clocks": clocks, "gpu_launches": S * K,
        }
        if e2e:
            line["e2e"] = e2e
        if not args.no_cpu_baseline and ws_n == 1:
            line["cpu_baseline"] = cpu_baseline(args.workload, min_seconds=args.cpu_seconds)
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

    ws_n, rank, dist, dev = setup_device()
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
    flush_l2 = make_flush(dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    P = lambda t: t.data_ptr()

    def fwd():
        abi.check(abi.wkv_token_shift(B, T, C, dt, n, P(mu), P(x), P(xp), P(out), sp))

    def bwd():
        abi.check(abi.wkv_token_shift_backward(B, T, C, dt, n, P(mu), P(x), P(xp), P(g), P(gx), P(gmu),
                                               P(gxp), P(wsb), nws, sp))

    for _ in range(args.warmup):
        flush_l2(); fwd(); bwd()
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
        flush_l2()
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
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded normal x, uniform mu)",
            "config": token_shift_config(args, wl, ws_n),
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


# ------------------------------------------------- causal linear attention ---

LA_FWD_BYTES = 4 * 32 * 2   # q, k, v read, out written (bf16, D = M = 32), per head-position
LA_BWD_BYTES = 7 * 32 * 2   # q, k, v, grad_out read, grad_q, grad_k, grad_v written


def linattn_config(wl, ws_n, saved=True):
    return {"workload": wl.name, "op": "causal linear attention (elu+1)", "BH": wl.BH, "N": wl.N,
            "D": wl.D, "M": wl.D, "io_dtype": "bf16", "note": wl.note,
            "backward": "from the forward's saved state" if saved else "recomputing the forward",
            "parallelism": f"replicas x{ws_n}" if ws_n > 1 else "single GPU",
            "l2": "flushed before every timed step (2x L2 write + 2x L2 read, outside events)"}


def linattn_cpu_baseline(wl_name: str, min_seconds: float):
    """The linear-attention oracle (float64 numpy, forward then backward) on a
    few heads of the workload, full length."""
    from oracle import linattn as la
    wl = workloads.LINATTN_WORKLOADS[wl_name]
    heads = 4
    inp = workloads.generate_linattn(wl, BH=heads)
    med, reps = _time_loop(lambda: la.bwd_recur(inp["q"], inp["k"], inp["v"], inp["g"]), min_seconds)
    # bwd_recur runs the forward recurrence inside it, so one call is fwd + bwd
    return {"value": heads * wl.N / med, "unit": "head-positions/s", "cores": 1, "kind": "oracle",
            "sample": f"{wl_name}: {heads} heads x N{wl.N} fwd+bwd (numpy, one thread) x{reps}, median"}


def run_linattn(args):
    """Causal linear attention forward then backward through the C ABI
    (include/linattn.h), one call each per step."""
    import torch
    import rwkv_linear_rnn_b200 as W
    from rwkv_linear_rnn_b200 import abi

    ws_n, rank, dist, dev = setup_device()
    wl = workloads.LINATTN_WORKLOADS[args.workload]
    inp = workloads.generate_linattn(wl, seed=wl.seed + 1000 * rank)
    BH, N, D = inp["BH"], inp["N"], inp["D"]
    t = {n: torch.from_numpy(inp[n + "_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
         for n in ("q", "k", "v", "g")}
    out = torch.empty_like(t["v"])
    dq, dk, dv = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
    nf = abi.linattn_workspace_size(0, BH, N, D, D)
    nb = abi.linattn_workspace_size(1, BH, N, D, D)
    wsb = torch.zeros(max(nf, nb), dtype=torch.uint8, device=dev)
    flush_l2 = make_flush(dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    P = lambda x: x.data_ptr()

    def fwd():
        abi.check(abi.linattn_forward(BH, N, D, D, P(t["q"]), P(t["k"]), P(t["v"]), P(out), None, P(wsb),
                                      wsb.numel(), sp))

    saved = not args.la_recompute

    def bwd():
        if saved:  # from the state the forward just left in the workspace
            abi.check(abi.linattn_backward_saved(BH, N, D, D, P(t["q"]), P(t["k"]), P(t["v"]), P(out), P(t["g"]),
                                                 P(dq), P(dk), P(dv), P(wsb), wsb.numel(), sp))
        else:
            abi.check(abi.linattn_backward(BH, N, D, D, P(t["q"]), P(t["k"]), P(t["v"]), P(t["g"]), P(dq), P(dk),
                                           P(dv), P(wsb), wsb.numel(), sp))

    for _ in range(args.warmup):
        flush_l2(); fwd(); bwd()
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
        flush_l2()
        ev[i][0].record(stream); fwd(); ev[i][1].record(stream); bwd(); ev[i][2].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop(window=(t_begin, time.monotonic()))
    if dist:
        dist.barrier()
    t_fwd = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    t_bwd = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    total_ms = max_over_ranks(sum(t_fwd) + sum(t_bwd), dist, dev)
    status = abi.wkv_get_status(P(wsb), sp)

    units = BH * N
    e2e = None
    if not args.no_e2e:
        hin = {n: t[n].cpu().pin_memory() for n in t}
        hout = [torch.empty_like(x, device="cpu").pin_memory() for x in (out, dq, dk, dv)]
        h2d = sum(x.numel() * x.element_size() for x in hin.values())
        d2h = sum(x.numel() * x.element_size() for x in hout)
        ee = []
        for i in range(max(3, min(K, 10)) + 1):
            e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for n in t:
                t[n].copy_(hin[n], non_blocking=True)
            fwd(); bwd()
            for h, d in zip(hout, (out, dq, dk, dv)):
                h.copy_(d, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if i > 0:
                ee.append(e0.elapsed_time(e1))
        e2e_ms = max_over_ranks(statistics.median(ee), dist, dev)
        e2e = {"value": aggregate_rate(units, ws_n, e2e_ms), "unit": "head-positions/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    if rank == 0:
        hbm, peak_kind = peaks()
        fwd_ms, bwd_ms = statistics.mean(t_fwd), statistics.mean(t_bwd)
        fb, bb = LA_FWD_BYTES * units, LA_BWD_BYTES * units
        fwd_gbs = fb / (fwd_ms * 1e-3) / 1e9
        bwd_gbs = bb / (bwd_ms * 1e-3) / 1e9
        nch = -(-N // 128)
        # tensor-core work issued per 128-position chunk (M = 128 tiles, padding included)
        mf = lambda m, n, k: 2.0 * m * n * k
        f_chunk = mf(128, 128, 32) + mf(128, 32, 128) + mf(128, 32, 32) + mf(128, 48, 128)
        b_recompute = mf(128, 48, 128) + mf(128, 128, 32) + mf(128, 48, 128) + mf(128, 48, 32)  # state, scores, A[V|1], Q[S|Z]
        b_chunk = (mf(128, 48, 128) + 2 * mf(128, 128, 32) + 3 * (mf(128, 32, 128) + mf(128, 32, 32))
                   + (0 if saved else b_recompute))
        step_ms = total_ms / K
        line = {
            "metric": "causal linear attention fwd+bwd head-positions/s (HBM GB/s and % of roofline alongside)",
            "value": aggregate_rate(units, ws_n, step_ms), "unit": "head-positions/s",
            "n_gpus": ws_n, "steps": K, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) q, k, v, grad_out rounded to bf16)",
            "config": linattn_config(wl, ws_n, saved),
            "roofline": {"bound": "hbm",
                         "kernel": ("linattn_backward_saved call (3 launches)" if saved
                                    else "linattn_backward call (5 launches)") + ", timed as one call",
                         "achieved": bwd_gbs, "peak": hbm, "unit": "GB/s", "frac": bwd_gbs / hbm,
                         "traffic": traffic_for(args.workload,
                                                "linattn_backward_saved" if saved else "linattn_backward", False),
                         "algorithmic_bytes": bb, "peak_kind": peak_kind},
            "fwd": {"ms": fwd_ms, "gbs": fwd_gbs, "frac": fwd_gbs / hbm, "launches": 3,
                    "tensor_tflops_issued": f_chunk * BH * nch / (fwd_ms * 1e-3) / 1e12},
            "bwd": {"ms": bwd_ms, "gbs": bwd_gbs, "frac": bwd_gbs / hbm, "launches": 3 if saved else 5,
                    "tensor_tflops_issued": b_chunk * BH * nch / (bwd_ms * 1e-3) / 1e12},
            "clocks": clocks, "device_status": status, "gpu_launches": (6 if saved else 8) * K,
        }
        if e2e:
            line["e2e"] = e2e
        if not args.no_cpu_baseline and ws_n == 1:
            line["cpu_baseline"] = linattn_cpu_baseline(args.workload, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libwkv", choices=["libwkv", "reference"])
    ap.add_argument("--workload", default="rwkv1b5_bf16",
                    choices=sorted(workloads.WORKLOADS) + sorted(workloads.LINATTN_WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--fwd-kernel", default="auto", choices=["auto"] + sorted(FWD_PLAN))
    ap.add_argument("--bwd-kernel", default="auto", choices=["auto"] + sorted(BWD_PLAN))
    ap.add_argument("--gate", action="store_true",
                    help="time the gated calls (o = sigmoid(r) * wkv and its gradients)")
    ap.add_argument("--la-recompute", action="store_true",
                    help="linear attention: time the backward that recomputes the forward instead of the one "
                         "from the forward's saved state")
    ap.add_argument("--token-shift", action="store_true",
                    help="time the token shift (3 interpolations) on the workload's layer shape")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # timing rule: at least 3 untimed warm-up steps
    if args.workload in workloads.LINATTN_WORKLOADS:
        if args.gate or args.token_shift:
            raise SystemExit("--gate / --token-shift apply to the WKV workloads")
        if args.impl == "reference":
            run_linattn_reference(args)
        else:
            run_linattn(args)
        return
    if args.gate and workload_mode(args.workload) == "step":
        raise SystemExit("--gate applies to the forward/backward workloads")
    if args.impl == "reference":
        run_reference(args)
    elif args.token_shift:
        run_token_shift(args)
    else:
        run_libwkv(args)


if __name__ == "__main__":
    main()
