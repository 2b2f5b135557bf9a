#!/usr/bin/env python
"""Benchmark of the exact IO-aware attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole bf16 path over one batch: fa_fwd (O, LSE)
followed by fa_bwd (preprocess, recompute kernel, dQ conversion).  The
workload is the long-context causal attention B=1, H=32, N=32768, d=128 with
Q, K, V, dO ~ N(0, 1) (seeded synthetic inputs): the largest of the attention
configurations, and it fits one GPU.  The metric is attention TFLOP/s:
  forward FLOPs F = 4 B H N^2 d (halved when causal), backward 2.5 F,
  fwd+bwd TFLOP/s = 3.5 F / (t_fwd + t_bwd).
Rank 0 prints ONE JSON line.

With --gpus N > 1 outside a torchrun environment the script re-launches itself
under torch.distributed.run with N ranks (one per GPU).  The B*H heads of the
one problem are split into contiguous slices, one per rank: heads are
independent, so there is no collective on the data path (NCCL only takes the
max of the ranks' times).  `value` is the whole problem's FLOPs divided by the
slowest rank's time: the total work is fixed as N grows (strong scaling).

`--impl reference` times the fp64 CPU oracle (the correctness reference) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import importlib.util
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(B=1, H=32, N=32768, d=128, causal=True)
WORKLOAD_NAME = "attention fwd+bwd bf16 B1 H32 N32768 d128 causal"
WORKLOAD_SEED = 1238                 # the seed of this configuration's parity test
CPU_SAMPLE_N = 4096                  # rows and keys of the CPU oracle's sample unit
METRIC = "attention TFLOP/s fwd & fwd+bwd (bf16) and % of B200 dense tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def workload_config():
    """The `config` of both arms' lines: the workload, its shape and its seed."""
    return {"workload": WORKLOAD_NAME, **WORKLOAD, "seed": WORKLOAD_SEED, "global_batch": WORKLOAD["B"],
            "seq_len": WORKLOAD["N"]}


def fwd_flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    return f / 2.0 if causal else f


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and clock-event reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        loaded = [x for x in sm if smax and x > 0.3 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# -------------------------------------------------------------- our arm
def apply_shape(args):
    """--shape/--causal/--noncausal select another workload (profiling runs);
    the default is the bench workload."""
    global WORKLOAD_NAME
    if args.shape:
        B, H, N, d = (int(x) for x in args.shape.split(","))
        WORKLOAD.update(B=B, H=H, N=N, d=d)
    if args.causal:
        WORKLOAD["causal"] = True
    if args.noncausal:
        WORKLOAD["causal"] = False
    if args.shape or args.causal or args.noncausal:
        WORKLOAD_NAME = (f"attention fwd+bwd bf16 B{WORKLOAD['B']} H{WORKLOAD['H']} N{WORKLOAD['N']} "
                         f"d{WORKLOAD['d']} {'causal' if WORKLOAD['causal'] else 'non-causal'}")


def spawn_ranks(args) -> int:
    """Re-launch this script under torch.distributed.run with one rank per GPU."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def rank_heads(B, H, ws, rank):
    """This rank's contiguous slice [h0, h1) of the flattened B*H heads."""
    from exact_io_aware_55_b200.dist import head_range
    return head_range(B * H, ws, rank)


def head_slice(bits, B, H, h0, h1):
    """Heads [h0, h1) of a [B, H, N, d] array as a contiguous [1, h1-h0, N, d]
    array (a [B, H, N, d] tensor is B*H consecutive heads)."""
    N, d = bits.shape[2], bits.shape[3]
    return np.ascontiguousarray(bits.reshape(B * H, N, d)[h0:h1]).reshape(1, h1 - h0, N, d)


def run_ours(args):
    import torch

    import exact_io_aware_55_b200 as fa
    import synth
    from exact_io_aware_55_b200.dist import max_over_ranks

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    B, H, N, d, causal = (WORKLOAD[k] for k in ("B", "H", "N", "d", "causal"))
    h0, h1 = rank_heads(B, H, ws, rank)
    nh = h1 - h0
    scale = 1.0 / math.sqrt(d)
    inp = synth.attention_inputs(B, H, N, d, seed=WORKLOAD_SEED, want_f64=False)
    host_in = {n: head_slice(inp[n + "_bits"], B, H, h0, h1) for n in ("q", "k", "v", "do")}
    del inp

    def to_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v, do = (to_dev(host_in[n]) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((1, nh, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    work = torch.empty(max(16, fa.fa_bwd_workspace_size(1, nh, N, d)), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.fa_fwd(q, k, v, o, lse, scale, causal, stream)
        fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, scale, causal, work, stream)

    F_all = fwd_flops(B, H, N, d, causal)          # the whole problem, all ranks
    F_rank = fwd_flops(1, nh, N, d, causal)        # this rank's slice

    def timed(K, W, sampler_window_s=args.clock_window):
        for _ in range(W):
            flush.fill_(1.0)
            step()
        torch.cuda.synchronize()
        # keep the GPU busy for a clock window so the sampler sees the loaded clock
        sampler = ClockSampler(local)
        sampler.start()
        t_end = time.time() + sampler_window_s
        while time.time() < t_end:
            for _ in range(5):
                flush.fill_(1.0)
                step()
            torch.cuda.synchronize()
        # per step: [start, fwd done = bwd start, main kernel start, main kernel end, bwd end]
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(K):
            flush.fill_(1.0)                     # L2 flush, outside the events
            ev[i][0].record(stream)
            fa.fa_fwd(q, k, v, o, lse, scale, causal, stream)
            if nh > 0:
                fa.fa_bwd_events(q, k, v, o, do, lse, dq, dk, dv, scale, causal, work, ev[i][1:], stream)
            else:                                # more ranks than heads: this rank has nothing to do
                for e in ev[i][1:]:
                    e.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        clocks = sampler.stop()
        mean = lambda a, b: sum(e[a].elapsed_time(e[b]) for e in ev) / K  # noqa: E731
        return {"fwd": mean(0, 1), "bwd": mean(1, 4), "pre": mean(1, 2), "main": mean(2, 3),
                "fin": mean(3, 4)}, clocks

    t, clocks = timed(args.steps, args.warmup)
    # Re-measure once if any rank saw a throttle reason; the decision is taken
    # together so that every rank runs the same collectives.
    bad = any(r in clocks["reasons"] for r in BAD_REASONS)
    if dist is not None:
        flag = torch.tensor([1.0 if bad else 0.0], device=dev)
        dist.all_reduce(flag, op=dist.ReduceOp.MAX)
        bad = flag.item() > 0.0
    if bad:
        t, clocks = timed(args.steps, args.warmup)
        clocks["remeasured"] = True
    st, where = fa.fa_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} (wait site {where}) during the bench")

    t_step, t_fwd, t_bwd, t_main, t_pre, t_fin = max_over_ranks(
        dist, [t["fwd"] + t["bwd"], t["fwd"], t["bwd"], t["main"], t["pre"], t["fin"]], dev)
    value = 3.5 * F_all / (t_step * 1e-3) / 1e12
    fwd_tflops = F_all / (t_fwd * 1e-3) / 1e12
    bwd_tflops = 2.5 * F_all / (t_bwd * 1e-3) / 1e12

    # ---------------- e2e through the public API with pinned host buffers
    # Every step copies its inputs host -> device, runs fa_fwd + fa_bwd and
    # copies O, LSE, dQ, dK, dV back.  Three streams (H2D, compute, D2H) and
    # two device buffer sets let step i's upload and step i-1's download
    # overlap with the kernels; events order each buffer's reuse.
    host = {n: torch.from_numpy(host_in[n].view(np.int16)).view(torch.bfloat16).pin_memory()
            for n in ("q", "k", "v", "do")}
    out_names = ("o", "lse", "dq", "dk", "dv")
    shapes = {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
    host_out = [{n: torch.empty(shapes[n].shape, dtype=shapes[n].dtype, pin_memory=True) for n in out_names}
                for _ in range(2)]
    dev_in = [{n: torch.empty_like(host[n], device=dev) for n in host} for _ in range(2)]
    dev_out = [{n: torch.empty_like(shapes[n]) for n in out_names} for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    mk = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, comp_done, out_done = [mk(), mk()], [mk(), mk()], [mk(), mk()]
    started = [False, False]

    def e2e_step(i):
        b = i & 1
        if started[b]:
            s_in.wait_event(comp_done[b])                 # compute of step i-2 no longer reads dev_in[b]
        with torch.cuda.stream(s_in):
            for n in host:
                dev_in[b][n].copy_(host[n], non_blocking=True)
            in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        if started[b]:
            stream.wait_event(out_done[b])                # download of step i-2 has read dev_out[b]
        di, do_ = dev_in[b], dev_out[b]
        fa.fa_fwd(di["q"], di["k"], di["v"], do_["o"], do_["lse"], scale, causal, stream)
        fa.fa_bwd(di["q"], di["k"], di["v"], do_["o"], di["do"], do_["lse"], do_["dq"], do_["dk"], do_["dv"],
                  scale, causal, work, stream)
        comp_done[b].record(stream)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            for n in out_names:
                host_out[b][n].copy_(do_[n], non_blocking=True)
            out_done[b].record(s_out)
        started[b] = True

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    K2 = max(5, min(args.steps, 30))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(K2):
        e2e_step(i)
    s_out.wait_event(out_done[(K2 - 1) & 1])
    s_out.wait_event(comp_done[(K2 - 1) & 1])
    e1.record(s_out)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(dist, [e0.elapsed_time(e1) / K2], dev)[0]
    h2d = sum(x.numel() * x.element_size() for x in host.values())
    d2h = sum(x.numel() * x.element_size() for x in host_out[0].values())
    del host, host_out, dev_in, dev_out

    # ---------------- extra measurements (rank 0 of a 1-GPU run, not part of `value`)
    extra = {}
    if rank == 0 and ws == 1 and not args.no_extra:
        del q, k, v, do, o, lse, dq, dk, dv, work
        torch.cuda.empty_cache()
        extra = extra_measurements(fa, torch, dev, stream, flush)

    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    peak_sus = float(peaks.get("bf16_tflops_sustained", peak))
    # The dominant kernel: the backward's recompute kernel, 2.5 F of this rank's
    # slice per launch.  It is timed inside a long step (K steps of fwd + bwd
    # back to back, seconds under the 1 kW power cap), so its denominator is the
    # sustained bf16 figure; the burst one is reported beside it.
    main_tflops = 2.5 * F_rank / (t_main * 1e-3) / 1e12 if nh else 0.0
    call_tflops = 2.5 * F_rank / (t_bwd * 1e-3) / 1e12 if nh else 0.0
    roof = {"bound": "tensor", "kernel": "bwd_kernel<128, causal> (the backward's recompute kernel)",
            "achieved": round(main_tflops, 2), "peak": peak_sus, "unit": "TFLOP/s",
            "frac": round(main_tflops / peak_sus, 4),
            "traffic": committed_traffic("bwd_kernel", WORKLOAD_NAME) if ws == 1 else None,
            "algorithmic_flops_per_launch": 2.5 * F_rank,
            "ms_per_launch": round(t_main, 5),
            "peak_source": f"{peak_src} bf16_tflops_sustained (the kernel runs inside a seconds-long loaded "
                           f"region; see clocks)",
            "peak_burst": peak, "frac_of_burst_peak": round(main_tflops / peak, 4),
            "fa_bwd_call": {"achieved": round(call_tflops, 2), "frac": round(call_tflops / peak_sus, 4),
                            "frac_of_burst_peak": round(call_tflops / peak, 4),
                            "ms": round(t_bwd, 5), "ms_preprocess": round(t_pre, 5),
                            "ms_dq_convert": round(t_fin, 5)}}

    if rank == 0:
        cpu = cpu_baseline(args) if (ws == 1 and not args.no_cpu_baseline) else None
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(t_step, 5), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) Philox, rounded to bf16)",
            "config": workload_config(),
            "parallelism": f"heads split over {ws} GPU(s), {nh} on rank 0, no data-path collective",
            "l2": "inputs (4 x 256 MiB at one GPU) exceed L2; plus a 256 MiB flush write between steps, "
                  "outside the per-step CUDA events",
            "fwd_tflops": round(fwd_tflops, 2), "bwd_tflops": round(bwd_tflops, 2),
            "fwd_frac_of_peak": round(fwd_tflops / ws / peak, 4),
            "bwd_frac_of_peak": round(bwd_tflops / ws / peak, 4),
            "fwd_bwd_frac_of_peak": round(value / ws / peak, 4),
            "ms_fwd": round(t_fwd, 5), "ms_bwd": round(t_bwd, 5),
            "e2e": {"value": round(3.5 * F_all / (t_e2e * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                    "ms_per_step": round(t_e2e, 4), "h2d_bytes_per_step": h2d * ws, "d2h_bytes_per_step": d2h * ws,
                    "api": "fa_fwd + fa_bwd on pinned-host inputs copied in and results copied out every "
                           "step; copy and compute streams overlap neighbouring steps"},
            "gpu_launches": 4 * args.steps,
            "roofline": roof,
            "clocks": {k_: clocks[k_] for k_ in ("sm_mhz", "sm_max_mhz", "reasons", "samples")},
            "cpu_baseline": cpu,
            "extra": extra,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_case(args):
    """One named path on --shape, for profiling (a short JSON line, not the
    bench line): 'decode' (B,H,Nk,d with --nq queries, causal), 'standard'
    (B,H,N,d: the materialising baseline, then the fused forward, per step),
    'fp8' (B,H,N,d: the e4m3 forward) or 'det' (B,H,N,d: the backward with the
    deterministic dQ pass, after one forward)."""
    import torch

    import exact_io_aware_55_b200 as fa

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    B, H, N, d = (int(x) for x in args.shape.split(","))

    def rnd(*shape):
        return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)

    nbytes, flops = None, None
    if args.case == "decode":
        q, k, v = rnd(B, H, args.nq, d), rnd(B, H, N, d), rnd(B, H, N, d)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, args.nq), device=dev)
        work = torch.empty(max(16, fa.fa_fwd_decode_workspace_size(B, H, args.nq, N, d)), dtype=torch.uint8,
                           device=dev)

        def step():
            fa.fa_fwd_decode(q, k, v, o, lse, d ** -0.5, True, work, stream)
        nbytes = 4 * B * H * N * d
    elif args.case == "det":
        q, k, v, do = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), device=dev)
        fa.fa_fwd(q, k, v, o, lse, d ** -0.5, args.causal, stream)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        work = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)

        def step():
            fa.fa_bwd_deterministic(q, k, v, o, do, lse, dq, dk, dv, d ** -0.5, args.causal, work, stream)
        flops = 2.5 * fwd_flops(B, H, N, d, args.causal)
    elif args.case == "fp8":
        q8, k8, v8 = (torch.randn((B, H, N, d), generator=g, device=dev).mul_(100.0).clamp_(-448, 448)
                      .to(torch.float8_e4m3fn) for _ in range(3))
        o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, H, N), device=dev)

        def step():
            fa.fa_fwd_fp8(q8, k8, v8, 0.01, 0.01, 0.01, o, lse, d ** -0.5, args.causal, stream)
        flops = fwd_flops(B, H, N, d, args.causal)
    else:
        q, k, v = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), device=dev)
        work = torch.empty(fa.fa_fwd_standard_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)

        def step():
            fa.fa_fwd_standard(q, k, v, o, lse, d ** -0.5, args.causal, work, stream)
            fa.fa_fwd(q, k, v, o, lse, d ** -0.5, args.causal, stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    st, where = fa.fa_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} (wait site {where})")
    ms = e0.elapsed_time(e1) / args.steps
    line = {"case": args.case, "shape": args.shape, "causal": bool(args.causal), "ms_per_step": round(ms, 5)}
    if nbytes:
        line["nq"] = args.nq
        line["gbs"] = round(nbytes / ms / 1e6, 1)
    if flops:
        line["tflops"] = round(flops / ms / 1e9, 1)
    print(json.dumps(line), flush=True)


def kernel_source_digest(files) -> str:
    """sha256 over the named library sources (paths relative to the package's
    csrc/ directory) and the build flags: the sources a kernel is built from."""
    import hashlib
    spec = importlib.util.spec_from_file_location("_fa_build", os.path.join(ROOT, "exact_io_aware_55_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    h = hashlib.sha256()
    for name in files:
        h.update(name.encode())
        h.update(open(os.path.normpath(os.path.join(build.CSRC, name)), "rb").read())
    h.update(" ".join(build.ARCH + build.FLAGS).encode())
    return h.hexdigest()


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the sources the kernel is built from now (same digest over the files the
    entry lists, and the same build flags); else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        ent = json.load(open(path)).get(kernel, {})
        files = ent.get("source_files")
        if not files or ent.get("workload") != workload:
            return None
        if ent.get("source_digest") == kernel_source_digest(files):
            return ent.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        return None
    return None


def extra_measurements(fa, torch, dev, stream, flush):
    """Single-GPU context numbers, each call timed with CUDA events on the
    launching stream with the L2 flush write between calls: the B4 H16 N2048
    d64 non-causal configuration, long-sequence non-causal bf16 (N=8192,
    d=128), the causal B2 H16 N8192 d128 configuration, the e4m3 forward at B2
    H16 N16384 d128, standard (materialising) attention against the fused
    forward, and the split-KV decode (1 and 4 queries over a 16384-key cache,
    8 x 32 heads, d=128)."""
    out = {}

    def time_call(fn, iters=10, warm=3, parts=False):
        """Mean ms per call; with parts=True fn takes four events (fa_bwd_events)
        and the result also holds the main kernel's own time."""
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(iters)]
        for i in range(warm):
            flush.fill_(1.0)
            fn(evs[0][1:]) if parts else fn()
        torch.cuda.synchronize()
        for i in range(iters):
            flush.fill_(1.0)
            evs[i][0].record(stream)
            if parts:
                fn(evs[i][1:])
            else:
                fn()
                evs[i][4].record(stream)
        torch.cuda.synchronize()
        ms = sum(e[0].elapsed_time(e[4]) for e in evs) / iters
        if not parts:
            return ms
        return ms, sum(e[2].elapsed_time(e[3]) for e in evs) / iters

    peaks, _ = load_peaks()
    pk = peaks["bf16_tflops"]
    g = torch.Generator(device=dev)
    g.manual_seed(7)

    def bf16(*shape):
        return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)

    for (B, H, N, d, causal) in ((4, 16, 2048, 64, False), (1, 32, 8192, 128, False), (2, 16, 8192, 128, True)):
        q, k, v, do = (bf16(B, H, N, d) for _ in range(4))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        work = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
        sc = 1.0 / math.sqrt(d)
        F = fwd_flops(B, H, N, d, causal)
        it = 20 if N <= 2048 else 10
        tf = time_call(lambda: fa.fa_fwd(q, k, v, o, lse, sc, causal, stream), iters=it)
        tb, tk = time_call(lambda e: fa.fa_bwd_events(q, k, v, o, do, lse, dq, dk, dv, sc, causal, work, e, stream),
                           iters=it, parts=True)
        out[f"{'causal' if causal else 'noncausal'}_b{B}_h{H}_n{N}_d{d}"] = {
            "fwd_tflops": round(F / tf / 1e9, 1), "fwd_frac": round(F / tf / 1e9 / pk, 4),
            "bwd_tflops": round(2.5 * F / tb / 1e9, 1), "bwd_frac": round(2.5 * F / tb / 1e9 / pk, 4),
            "bwd_kernel_tflops": round(2.5 * F / tk / 1e9, 1), "bwd_kernel_frac": round(2.5 * F / tk / 1e9 / pk, 4),
            "fwd_bwd_tflops": round(3.5 * F / (tf + tb) / 1e9, 1),
            "fwd_bwd_frac": round(3.5 * F / (tf + tb) / 1e9 / pk, 4),
            "inputs": "N(0,1) from torch's seeded CUDA generator (timing only)"}
        del q, k, v, do, o, dq, dk, dv, work, lse
    B, H, N, d = 2, 16, 16384, 128
    q8, k8, v8 = (torch.randn((B, H, N, d), generator=g, device=dev).mul_(100.0).clamp_(-448, 448)
                  .to(torch.float8_e4m3fn) for _ in range(3))
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), device=dev)
    F = fwd_flops(B, H, N, d, False)
    t8 = time_call(lambda: fa.fa_fwd_fp8(q8, k8, v8, 0.01, 0.01, 0.01, o, lse, 1.0 / math.sqrt(d), False, stream))
    fp8_peak = 2.0 * pk
    out["fp8_fwd_b2_h16_n16384_d128"] = {
        "tflops": round(F / t8 / 1e9, 1), "frac_of_fp8_peak": round(F / t8 / 1e9 / fp8_peak, 4),
        "fp8_peak": fp8_peak, "fp8_peak_source": "2 x measured bf16 (nominal fp8:bf16 dense ratio)"}
    # its backward: e4m3 Q, K, V widened exactly to bf16, the bf16 backward kernels
    do = bf16(B, H, N, d)
    dq, dk, dv = (torch.empty_like(do) for _ in range(3))
    work = torch.empty(fa.fa_bwd_fp8_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    tb8 = time_call(lambda: fa.fa_bwd_fp8(q8, k8, v8, 0.01, 0.01, 0.01, o, do, lse, dq, dk, dv, 1.0 / math.sqrt(d),
                                          False, work, stream))
    out["fp8_bwd_b2_h16_n16384_d128"] = {
        "tflops": round(2.5 * F / tb8 / 1e9, 1), "frac_of_bf16_peak": round(2.5 * F / tb8 / 1e9 / pk, 4),
        "fwd_bwd_tflops": round(3.5 * F / (t8 + tb8) / 1e9, 1),
        "note": "the five products run on bf16 tensor cores (exact widening of the e4m3 inputs)"}
    del q8, k8, v8, o, lse, do, dq, dk, dv, work
    # standard (materialising) attention against the fused forward on the same
    # inputs: the IO claim of the method, measured
    for (B, H, N, d) in ((4, 16, 2048, 64), (1, 32, 8192, 128)):
        q, k, v = (bf16(B, H, N, d) for _ in range(3))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), device=dev)
        work = torch.empty(fa.fa_fwd_standard_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
        sc = 1.0 / math.sqrt(d)
        ts = time_call(lambda: fa.fa_fwd_standard(q, k, v, o, lse, sc, False, work, stream))
        tf = time_call(lambda: fa.fa_fwd(q, k, v, o, lse, sc, False, stream))
        Np = -(-N // 128) * 128
        F = fwd_flops(B, H, N, d, False)
        out[f"standard_vs_fused_b{B}_h{H}_n{N}_d{d}"] = {
            "standard_ms": round(ts, 4), "fused_ms": round(tf, 4), "speedup": round(ts / tf, 2),
            "standard_tflops": round(F / ts / 1e9, 1), "fused_tflops": round(F / tf / 1e9, 1),
            "standard_hbm_bytes": B * H * (12 * N * Np + 8 * N * d),
            "fused_hbm_bytes": B * H * (8 * N * d + 4 * N)}
        del q, k, v, o, lse, work
    # split-KV decode against a 16384-key cache: HBM-bound, K and V read once
    # (2 GiB, well above L2; the flush write runs between calls as well)
    B, H, Nk, d = 8, 32, 16384, 128
    k, v = bf16(B, H, Nk, d), bf16(B, H, Nk, d)
    for Nq in (1, 4):
        q = bf16(B, H, Nq, d)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, Nq), device=dev)
        work = torch.empty(max(16, fa.fa_fwd_decode_workspace_size(B, H, Nq, Nk, d)), dtype=torch.uint8,
                           device=dev)
        td = time_call(lambda: fa.fa_fwd_decode(q, k, v, o, lse, 1.0 / math.sqrt(d), True, work, stream), iters=20)
        nbytes = 2 * B * H * Nk * d * 2 + 2 * B * H * Nq * d * 2 + B * H * Nq * 4
        out[f"decode_b8_h32_nq{Nq}_nk16384_d128_causal"] = {
            "us": round(td * 1e3, 2), "gbs": round(nbytes / td / 1e6, 1),
            "frac_of_measured_copy_bw": round(nbytes / td / 1e6 / peaks["hbm_gbs"], 4), "bytes": nbytes,
            "note": "denominator: the measured STREAM-style copy bandwidth (read + write); a read-only "
                    "stream can exceed it"}
    return out


# ------------------------------------------------------------- CPU oracle
def _oracle_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((x.get("num_threads") or 1) for x in info if x.get("user_api") == "blas")
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def oracle_sample(budget_s: float, seed: int = 4242):
    """fwd+bwd with the fp64 oracle on sample units of the bench workload until
    the time budget is spent (at least one unit).  A unit is one head of the
    workload's shape cut to its first n = min(N, CPU_SAMPLE_N) queries and
    keys: under the causal mask those rows see exactly those keys, so the
    unit's O, LSE and dQ rows are the workload's own, computed in the same
    way.  Returns (TFLOP/s, units, seconds, n) with the unit's FLOPs counted
    by the metric's formula."""
    import oracle
    import synth

    d, causal = WORKLOAD["d"], WORKLOAD["causal"]
    n = min(WORKLOAD["N"], CPU_SAMPLE_N)
    inp = synth.attention_inputs(1, 4, n, d, seed=seed, want_f64=False)
    scale = 1.0 / math.sqrt(d)
    units, t0 = 0, time.perf_counter()
    while True:
        h = units % 4
        qh, kh, vh, doh = (synth.head_f64(inp, nm, 0, h) for nm in ("q", "k", "v", "do"))
        oracle.head_backward(qh, kh, vh, doh, scale, causal)     # includes the forward
        units += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    flops = 3.5 * fwd_flops(1, 1, n, d, causal) * units
    return flops / el / 1e12, units, el, n


def cpu_baseline(args):
    tflops, units, el, n = oracle_sample(args.cpu_budget)
    return {"value": tflops, "unit": "TFLOP/s", "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"{units} unit(s) of one head cut to its first {n} queries and keys "
                      f"(fwd+bwd, fp64 numpy/OpenBLAS, {'causal' if WORKLOAD['causal'] else 'non-causal'}, "
                      f"d={WORKLOAD['d']}) in {el:.1f} s; FLOPs by the metric's formula for the unit"}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    per_step, units_total, t_total, n = [], 0, 0.0, 0
    for _ in range(args.warmup):
        oracle_sample(0.0)
    for _ in range(args.steps):
        _, units, el, n = oracle_sample(args.ref_step_budget)
        per_step.append(el)
        units_total += units
        t_total += el
    F = 3.5 * fwd_flops(1, 1, n, WORKLOAD["d"], WORKLOAD["causal"]) * units_total
    value = F / t_total / 1e12
    cores = _oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / max(1, args.steps),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) Philox, rounded to bf16, evaluated in fp64)",
        "config": workload_config(),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: units of one head cut to its first {n} queries and keys "
                                   f"(fwd+bwd) for {args.ref_step_budget:.1f} s; {units_total} units in total"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-step-budget", type=float, default=1.0)
    ap.add_argument("--shape", default="", help="B,H,N,d of another workload (default: the bench workload)")
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--noncausal", action="store_true")
    ap.add_argument("--case", choices=["decode", "standard", "fp8", "det"], default="",
                    help="profile one path on --shape instead of the bench step")
    ap.add_argument("--nq", type=int, default=1, help="queries per head for --case decode")
    ap.add_argument("--clock-window", type=float, default=1.5,
                    help="seconds of steps run under the clock sampler before the timed region")
    args = ap.parse_args()
    if args.causal and args.noncausal:
        ap.error("--causal and --noncausal exclude each other")
    if args.case:
        if not args.shape:
            ap.error("--case needs --shape")
        run_case(args)
        return
    apply_shape(args)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
