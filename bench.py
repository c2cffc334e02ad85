"""Benchmark of the Titans memory write-and-read (libtitansmem) on B200.

One step = one tm_run over a whole workload: every chunk of every stream goes
through A1..A8 (stage inputs, forward of keys and queries, residual, backward,
coefficient scan, weight-update contractions, fused state update, chunk walk).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 3]
    python bench.py --impl reference ...     # the float64 oracle on host cores

Multi-GPU (torchrun): weak scaling; every rank runs its own full copy of the
workload (its own seed) with no collective on the data path; timing is the max
over ranks.
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

from gen import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 512 * 1024 * 1024
SM_COUNT = 148


def algorithmic_counts(w: W.Workload, T: int) -> dict:
    """Work the method must do for one pass over the workload.
    FLOPs/token = 4P (forward of keys and queries) + 2(P - P1) (backward data,
    layers 2..L) + 4P (the W and S weight-update contractions) = 10P - 2P1.
    State bytes per chunk = 16P (fp32 W and S read and written once)."""
    dims = w.dims
    P = W.param_count(dims)
    P1 = dims[0] * dims[1]
    tokens = w.streams * T
    chunks = w.streams * (T // w.C)
    tok_el = 4 if w.dtype == "f32" else 2
    return {
        "tokens": tokens,
        "flops": float(10 * P - 2 * P1) * tokens,
        "state_bytes": 16.0 * P * chunks,
        "token_io_bytes": float(3 * w.d * tok_el + 12 + 4 * w.d) * tokens,
    }


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons during timing."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    from test_trained_neural_b200.replicas import max_over_ranks as _max
    return _max(x, world, device="cuda")


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_oracle_sample(w: W.Workload, budget_s: float = 15.0, streams=None, T=None) -> dict:
    """Time the float64 oracle, as it stands, on a bounded sample of the
    workload: all streams (up to the host's cores) over a token prefix sized to
    take roughly `budget_s` seconds. Returns tokens/s and what was run."""
    import oracle
    cores = os.cpu_count() or 1
    if streams is None:
        streams = list(range(min(w.streams, cores)))
    per_tok = 12.0 * w.P  # float64 flops per token, roughly
    if T is None:
        # calibrate on a short run, then size the sample to the budget
        Tc = max(w.C, min(w.T, 64 // w.C * w.C or w.C))
        sub = W.generate(w, streams=streams, T=Tc)
        t0 = time.perf_counter()
        oracle.run_workload(w, sub, threads=len(streams))
        dt = max(time.perf_counter() - t0, 1e-4)
        T = int(budget_s / dt * Tc)
        T = max(w.C, min(w.T, T // w.C * w.C))
    sub = W.generate(w, streams=streams, T=T)
    t0 = time.perf_counter()
    oracle.run_workload(w, sub, threads=len(streams))
    dt = time.perf_counter() - t0
    tokens = len(streams) * T
    return {"value": tokens / dt, "unit": "tokens/s", "cores": min(len(streams), cores),
            "kind": "oracle", "seconds": dt, "approx_flops_per_token": per_tok,
            "sample": f"{len(streams)} of {w.streams} streams x first {T} of {w.T} tokens",
            "streams": streams, "T": T}


def run_reference(args, w: W.Workload):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps = []
    sample = None
    budget = max(2.0, 60.0 / max(args.steps + args.warmup, 1))
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(w, budget_s=budget) if sample is None else \
            cpu_oracle_sample(w, streams=sample[0], T=sample[1])
        if sample is None:
            sample = (r["streams"], r["T"])
        if i >= args.warmup:
            steps.append(r)
    val = statistics.mean(s["value"] for s in steps)
    line = {"impl": "reference", "metric": "memory tokens/sec (write+read)", "value": val,
            "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.mean(s["seconds"] for s in steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "C": w.C, "dims": w.dims},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": steps[0]["cores"],
                             "kind": "oracle", "sample": steps[0]["sample"]},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def sweep_chunk(args, w: W.Workload, sizes):
    """Chunk-size trade-off: the same workload timed at several chunk sizes C
    (gradients of a chunk are taken at its start weights, so C changes the
    method's result as well as its speed; this times it, it does not compare
    results). One JSON line per size: path taken, ms per pass, tokens/s."""
    import dataclasses

    import torch
    from test_trained_neural_b200 import NeuralMemory

    dev = torch.device("cuda", 0)
    inp = W.generate(w)
    d_in = {}
    for key in ("k", "v", "q"):
        a = np.ascontiguousarray(inp[key])
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if w.dtype == "bf16" else torch.from_numpy(a)
        d_in[key] = t.reshape(w.B, w.H, w.T, w.d).to(dev)
    for key in ("theta", "eta", "alpha", "W0", "S0"):
        d_in[key] = torch.from_numpy(np.ascontiguousarray(inp[key])).reshape(w.B, w.H, *inp[key].shape[1:]).to(dev)
    y = torch.empty((w.B, w.H, w.T, w.d), dtype=torch.float32, device=dev)
    We, Se = torch.empty_like(d_in["W0"]), torch.empty_like(d_in["S0"])
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for C in sizes:
        wc = dataclasses.replace(w, C=C)
        if wc.T % C:
            continue
        mem = NeuralMemory(w.L, w.d, w.expansion, path=args.path)
        try:
            path = mem.query_path(w.B, w.H, w.T, C, d_in["k"].dtype)
        except Exception as ex:  # no kernel for this size on the forced path
            print(json.dumps({"chunk": C, "unsupported": str(ex)}), flush=True)
            continue
        ws = mem.alloc_workspace(w.B, w.H, w.T, C, d_in["k"].dtype, dev)
        stream = torch.cuda.current_stream(dev)

        def step():
            mem.run(d_in["k"], d_in["v"], d_in["q"], d_in["theta"], d_in["eta"], d_in["alpha"],
                    d_in["W0"], d_in["S0"], C, y=y, W_end=We, S_end=Se, workspace=ws, stream=stream)
        for _ in range(args.warmup):
            flush.zero_()
            step()
        torch.cuda.synchronize()
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            step()
            a1.record(stream)
            torch.cuda.synchronize()
            ms.append(a0.elapsed_time(a1))
        mem.sync(ws, stream)
        t = statistics.mean(ms)
        print(json.dumps({"metric": "memory tokens/sec (write+read)", "workload": w.name, "T": w.T,
                          "chunk": C, "path": path, "ms_per_pass": t,
                          "tokens_per_s": w.streams * w.T / (t * 1e-3),
                          "workspace_bytes": ws.numel()}), flush=True)


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) measured by ncu
# inside the dominant kernels' launches on shortened cases (summaries under
# profiles/), with the number of tokens each capture covered; a full run is
# that figure scaled by tokens.
# - long d=128 workload: the chunk walker (cluster kernel for 15 streams,
#   global-exchange kernel for the 16th) on 16 streams x 65536 tokens, whose
#   537 MB of reads y are several times L2 so their write-back is counted:
#   784.7 + 483.3 MB and 52.5 + 4.6 MB. The state stays on chip, so the
#   traffic is the token inputs and outputs and grows with the tokens.
# - deep workload: one fused forward/backward launch and one update launch of
#   a group of 8 streams for one chunk of 128 tokens: 4.01 + 0 MB and
#   18.13 + 0 MB (the update's writes stay in L2 and are written back after
#   its launch, outside the window).
# - README-shape workload (d=384, 2 streams x 1024 tokens): every launch of
#   one tm_run (token conversion, initial copy, coefficients, 16 chunks of
#   three per-phase GEMM launches and one update): 488.2 MB read, 0 written
#   inside the launches (ncu flushes the caches before each launch, so these
#   reads are cold-cache).
# - d=64 eight-head workload: the cluster walker on 32 streams x 32768 tokens
#   (y 268 MB, twice L2): 424.2 MB read, 242.1 MB written.
# - linear d=64 workload (fp32, CUDA-core kernel, 256 tokens): 0.319 MB read,
#   nothing written back inside the launch.
CAPTURED_TRAFFIC = {("tc", "mlp2-d64-h8"): (424.181e6 + 242.146e6, 32 * 32768),
                    ("simt", "linear-d64"): (0.319e6, 256),
                    ("tc", "mlp2-d128-long"): (784.695040e6 + 483.341568e6 + 52.528896e6 + 4.637184e6, 16 * 65536),
                    ("tcl", "mlp4-d128-deep"): (4.007936e6 + 18.134528e6, 8 * 128),
                    ("tcl", "mlp2-d384-readme"): (3.152e6 + 18.885e6 + 0.034e6
                                                  + 16 * (2.585e6 + 3.275e6 + 2.880e6 + 20.395e6), 2 * 1024)}


def traffic_per_launch(path: str, w: W.Workload):
    rec = CAPTURED_TRAFFIC.get((path, w.name))
    if rec is None:
        return None
    nbytes, tokens = rec
    return nbytes * (w.streams * w.T) / tokens


def bench_decode(args, w: W.Workload):
    """One-token decode steps on the workload's memory shape and streams: each
    step reads one token per stream, writes y, and updates W and S in place.
    HBM-bound: the algorithmic traffic is every parameter of W and S read and
    written once (16P bytes per stream) plus the token's inputs and y."""
    import torch
    from test_trained_neural_b200 import NeuralMemory

    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    B, H, d = w.B, w.H, w.d
    mem = NeuralMemory(w.L, w.d, w.expansion)
    k, v, q = (torch.randn((B, H, d), generator=g, device=dev).to(dt) for _ in range(3))
    k = k / k.float().norm(dim=-1, keepdim=True).to(dt)
    q = q / q.float().norm(dim=-1, keepdim=True).to(dt)
    theta = torch.full((B, H), 1e-3, device=dev)
    eta = torch.full((B, H), 0.9, device=dev)
    alpha = torch.full((B, H), 1e-3, device=dev)
    # Cold state every step without a flush (zeroing a large buffer would leave
    # L2 full of dirty lines whose write-back lands inside a step this short):
    # rotate through enough independent states that together exceed L2 three
    # times; tiny states (which L2 holds anyway) fall back to the flush.
    state_bytes = 2 * B * H * w.P * 4
    nbuf = -(-3 * L2_BYTES // state_bytes)
    use_flush = nbuf > 64
    nbuf = 1 if use_flush else max(nbuf, 2)
    states = []
    for _ in range(nbuf):
        Wst = 0.05 * torch.randn((B, H, w.P), generator=g, device=dev)
        states.append((Wst, torch.zeros_like(Wst)))
    y = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev) if use_flush else None
    for i in range(max(args.warmup, nbuf)):
        Wst, Sst = states[i % nbuf]
        mem.decode_step(k, v, q, theta, eta, alpha, Wst, Sst, y)
    torch.cuda.synchronize()
    # steps are issued back to back (as a serving loop does), BURST per
    # measurement, so the host's launch time overlaps the device's work
    BURST = 1 if use_flush else 32
    ms = []
    for i in range(args.steps):
        if use_flush:
            flush.zero_()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for b in range(BURST):
            Wst, Sst = states[(i * BURST + b) % nbuf]
            mem.decode_step(k, v, q, theta, eta, alpha, Wst, Sst, y)
        a1.record()
        torch.cuda.synchronize()
        ms.append(a0.elapsed_time(a1) / BURST)
    t = statistics.mean(ms) * 1e-3
    streams = B * H
    el = 2 if dt == torch.bfloat16 else 4
    bytes_ = streams * (16.0 * w.P + 3 * d * el + 12 + 4 * d)
    peak = measured_peaks()
    gbs = bytes_ / t / 1e9
    print(json.dumps({"metric": "decode tokens/sec", "value": streams / t, "unit": "tokens/s", "us": t * 1e6,
                      "workload": w.name, "streams": streams, "finite": bool(torch.isfinite(Wst).all()),
                      "l2": "flushed between steps" if use_flush else "%d rotating states (%.0f MB)" % (
                          nbuf, nbuf * state_bytes / 1e6),
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak["hbm_gbs"], "unit": "GB/s",
                                   "frac": gbs / peak["hbm_gbs"], "peak_source": peak["source"] + " HBM copy"}}),
          flush=True)


def bench_backward(args, w: W.Workload):
    """Gradients of the memory layer on the workload's shape: one tm_backward
    per step (forward recomputed inside with chunk-start checkpoints, then the
    reverse pass). CUDA-core fp32: the roofline is the FP32 issue rate. FLOPs
    per token, counted from the kernels' matrix products (P1 = the first
    layer's weights): 22P at depth 1, 32P - 6P1 at depth 2, 34P - 8P1 deeper
    (forward 8P - 2P1, reverse 26P - 6P1)."""
    import torch
    from test_trained_neural_b200 import NeuralMemory

    dev = torch.device("cuda", 0)
    inp = W.generate(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d_in = {}
    for key in ("k", "v", "q"):
        a = np.ascontiguousarray(inp[key])
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if dt == torch.bfloat16 else torch.from_numpy(a)
        d_in[key] = t.reshape(w.B, w.H, w.T, w.d).to(dev)
    for key in ("theta", "eta", "alpha", "W0", "S0"):
        a = np.ascontiguousarray(inp[key], dtype=np.float32)
        d_in[key] = torch.from_numpy(a).reshape(w.B, w.H, *a.shape[1:]).to(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    dy = torch.randn((w.B, w.H, w.T, w.d), generator=g, device=dev)
    dW = torch.randn(d_in["W0"].shape, generator=g, device=dev)
    dS = torch.randn(d_in["S0"].shape, generator=g, device=dev)
    mem = NeuralMemory(w.L, w.d, w.expansion)
    run = lambda: mem.backward(d_in["k"], d_in["v"], d_in["q"], d_in["theta"], d_in["eta"], d_in["alpha"],
                               d_in["W0"], d_in["S0"], dy, dW, dS, w.C)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        out = run()
    torch.cuda.synchronize()
    ms = []
    for _ in range(args.steps):
        flush.zero_()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        out = run()
        a1.record()
        torch.cuda.synchronize()
        ms.append(a0.elapsed_time(a1))
    t = statistics.mean(ms) * 1e-3
    tokens = w.streams * w.T
    P1 = w.dims[0] * w.dims[1]
    flops = (22.0 * w.P if w.L == 1 else 32.0 * w.P - 6.0 * P1 if w.L == 2 else 34.0 * w.P - 8.0 * P1) * tokens
    peaks = measured_peaks()
    tf = flops / t / 1e12
    if w.dtype == "bf16":
        # bf16 inputs: the chunk's products run on tcgen05 with TF32 operands,
        # whose dense rate is half the bf16 one
        peak = 0.5 * peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                "peak_source": peaks["source"] + " bf16 burst (cuBLAS) x 1/2 (TF32 / BF16 nominal)",
                "kernel": "backward%s_kernel<true> (tcgen05 kind::tf32 products)" % ("1" if w.L == 1 else "2" if w.L == 2 else "L")}
    else:
        peak = SM_COUNT * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                "peak_source": "fp32 FFMA: 148 SMs x 128 lanes x 2 x max clock",
                "kernel": "backward%s_kernel<false> (fp32 FFMA)" % ("1" if w.L == 1 else "2" if w.L == 2 else "L")}
    print(json.dumps({"metric": "backward tokens/sec", "value": tokens / t, "unit": "tokens/s", "ms": t * 1e3,
                      "workload": w.name, "finite": bool(all(torch.isfinite(v).all() for v in out.values())),
                      "roofline": roof}), flush=True)


def bench_prologue(args, w: W.Workload):
    """The step before the memory on the workload's k, v, q: one fused launch of
    the depthwise causal convolution (width args.conv_width) and the L2
    normalisation of keys and queries. HBM-bound: the algorithmic traffic is
    each of k, v, q read once and written once."""
    import torch
    from test_trained_neural_b200 import prologue

    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    xs = [torch.randn((w.B, w.H, w.T, w.d), generator=g, device=dev).to(dt) for _ in range(3)]
    fs = [0.5 * torch.randn((w.H, w.d, args.conv_width), generator=g, device=dev) for _ in range(3)]
    outs = tuple(torch.empty_like(x) for x in xs)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        prologue(*xs, *fs, out=outs)
    torch.cuda.synchronize()
    ms = []
    for _ in range(args.steps):
        flush.zero_()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        prologue(*xs, *fs, out=outs)
        a1.record()
        torch.cuda.synchronize()
        ms.append(a0.elapsed_time(a1))
    t = statistics.mean(ms) * 1e-3
    bytes_ = 2.0 * 3 * xs[0].numel() * xs[0].element_size()
    peak = measured_peaks()
    gbs = bytes_ / t / 1e9
    print(json.dumps({"metric": "prologue tokens/sec", "value": w.streams * w.T / t, "unit": "tokens/s",
                      "ms": t * 1e3, "workload": w.name, "width": args.conv_width,
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak["hbm_gbs"],
                                   "unit": "GB/s", "frac": gbs / peak["hbm_gbs"],
                                   "peak_source": peak["source"] + " HBM copy"}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", type=int, default=3, help="workload index 0..4")
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tc", "tcl", "tcl-phased"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--literal-gates", action="store_true",
                    help="draw the gates exactly as specified (the MLP memories overflow)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (tokens per stream), e.g. for short profiling runs")
    ap.add_argument("--chunk", type=int, default=None, help="override the chunk size C")
    ap.add_argument("--prologue", action="store_true",
                    help="time the convolution + normalisation step before the memory instead")
    ap.add_argument("--conv-width", type=int, default=4)
    ap.add_argument("--backward", action="store_true",
                    help="time the memory layer's gradients (depth-1 workloads) instead")
    ap.add_argument("--decode", action="store_true",
                    help="time one-token decode steps on the workload's memory and streams instead")
    ap.add_argument("--sweep-chunk", default=None,
                    help="comma-separated chunk sizes: time each (same workload, T as given) "
                         "and print one JSON line per size instead of the benchmark line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--segment-tokens", type=int, default=0,
                    help="tm_run_host segment length for the end-to-end leg (0 = library default)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = W.get_literal(args.workload) if args.literal_gates else W.get(args.workload)
    if args.tokens:
        import dataclasses
        w = dataclasses.replace(w, T=args.tokens)
    if args.chunk:
        import dataclasses
        w = dataclasses.replace(w, C=args.chunk)
    if args.sweep_chunk:
        return sweep_chunk(args, w, [int(x) for x in args.sweep_chunk.split(",")])
    if args.prologue:
        return bench_prologue(args, w)
    if args.decode:
        return bench_decode(args, w)
    if args.backward:
        return bench_backward(args, w)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    from test_trained_neural_b200 import NeuralMemory

    rank, world, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from test_trained_neural_b200.replicas import aggregate_throughput, replica
    inp = W.generate(replica(w, rank))
    pinned = {}
    for key in ("k", "v", "q"):
        a = np.ascontiguousarray(inp[key])
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if w.dtype == "bf16" else torch.from_numpy(a)
        pinned[key] = t.reshape(w.B, w.H, w.T, w.d).pin_memory()
    for key in ("theta", "eta", "alpha", "W0", "S0"):
        pinned[key] = torch.from_numpy(np.ascontiguousarray(inp[key])).reshape(
            w.B, w.H, *inp[key].shape[1:]).pin_memory()
    del inp
    d_in = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
    mem = NeuralMemory(w.L, w.d, w.expansion, path=args.path)
    path_used = mem.query_path(w.B, w.H, w.T, w.C, d_in["k"].dtype)
    ws = mem.alloc_workspace(w.B, w.H, w.T, w.C, d_in["k"].dtype, dev)
    y = torch.empty((w.B, w.H, w.T, w.d), dtype=torch.float32, device=dev)
    We = torch.empty_like(d_in["W0"])
    Se = torch.empty_like(d_in["S0"])
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        mem.run(d_in["k"], d_in["v"], d_in["q"], d_in["theta"], d_in["eta"], d_in["alpha"],
                d_in["W0"], d_in["S0"], w.C, y=y, W_end=We, S_end=Se, workspace=ws, stream=stream)

    with torch.cuda.nvtx.range("tm_run warm-up"):
        for _ in range(args.warmup):
            flush.zero_()
            step()
    mem.sync(ws, stream)
    torch.cuda.synchronize()
    ok = bool(torch.isfinite(y).all() and torch.isfinite(We).all())

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    with torch.cuda.nvtx.range("tm_run timed"):
        for i in range(args.steps):
            flush.zero_()  # L2 flush between steps, outside the timed events
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    t_wall = time.perf_counter() - t_wall
    clk = clocks.stop()
    mem.sync(ws, stream)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms = statistics.mean(step_ms)
    ms_max = max_over_ranks(ms, world)

    cnt = algorithmic_counts(w, w.T)
    launches_per_step = mem.launch_count(w.B, w.H, w.T, w.C, d_in["k"].dtype)
    value = aggregate_throughput(cnt["tokens"], world, ms_max * 1e-3)
    peaks = measured_peaks()
    hbm = peaks["hbm_gbs"] * 1e9
    tens = peaks["bf16_tflops_sustained"] * 1e12
    t_flop = cnt["flops"] / tens
    t_state = (cnt["state_bytes"] + cnt["token_io_bytes"]) / hbm
    chunk_roofline_s = max(t_flop, t_state)
    sec = ms * 1e-3
    if path_used in ("tc", "tcl", "tcl-phased"):
        # The kernel runs alone at the maximum SM clock, far from the power
        # cap, so the burst figure is the denominator.
        roof = {"bound": "tensor", "achieved": cnt["flops"] / sec / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "peak_source": peaks["source"] + " bf16 burst (cuBLAS)"}
    else:
        sm_mhz = clk.get("sm_mhz") or peaks["sm_max_mhz"]
        alu_peak = SM_COUNT * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": cnt["flops"] / sec / 1e12, "peak": alu_peak,
                "unit": "TFLOP/s", "peak_source": "fp32 FFMA: 148 SMs x 128 lanes x 2 x max clock",
                "sm_mhz_seen": sm_mhz}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic_per_launch(path_used, w)
    fused = all(n <= 256 for n in w.dims)
    transposed = all(w.dims[l - 1] % 128 == 0 and w.dims[l] % 64 == 0 for l in range(1, len(w.dims)))
    upd = ("tcl_update3_kernel" if transposed else "tcl_update2_kernel") if w.C <= 128 else "tcl_update_kernel"
    roof["kernel"] = {"tc": "tc_chunk_kernel (cluster and global-exchange forms)",
                      "tcl": ("tcl_fb_kernel + " if fused else "tcl_gemm_kernel + ") + upd,
                      "tcl-phased": "tcl_gemm_kernel + " + upd}.get(path_used, "simt_chunk_kernel")
    if roof["traffic"] is not None:
        roof["traffic_scope"] = ("DRAM bytes inside the kernels' launches per tm_run, from an ncu capture "
                                 "of a shortened case scaled by tokens (profiles/)")

    e2e = None
    if not args.no_e2e:
        # End to end through the public host-buffer API (tm_run_host): pinned
        # host inputs in, the reads and the final state out, every step; the
        # library copies segments of T in and out on side streams, overlapped
        # with the kernels.
        h_y = torch.empty(y.shape, dtype=torch.float32, pin_memory=True)
        h_W = torch.empty(We.shape, dtype=torch.float32, pin_memory=True)
        h_S = torch.empty(Se.shape, dtype=torch.float32, pin_memory=True)
        bi = sum(v.numel() * v.element_size() for v in pinned.values())
        bo = sum(v.numel() * v.element_size() for v in (h_y, h_W, h_S))
        seg = args.segment_tokens
        del ws
        hws = torch.empty(mem.host_workspace_size(w.B, w.H, w.T, w.C, d_in["k"].dtype, seg),
                          dtype=torch.uint8, device=dev)

        def e2e_step():
            mem.run_host(pinned["k"], pinned["v"], pinned["q"], pinned["theta"], pinned["eta"],
                         pinned["alpha"], pinned["W0"], pinned["S0"], w.C, y=h_y, W_end=h_W, S_end=h_S,
                         workspace=hws, segment_tokens=seg, stream=stream, sync=False)

        e2e_step()                       # warm-up (first use creates the copy streams)
        torch.cuda.synchronize()
        e_ms = []
        with torch.cuda.nvtx.range("tm_run end to end"):
            for i in range(max(2, min(args.steps, 3))):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                e2e_step()
                b.record(stream)
                torch.cuda.synchronize()
                e_ms.append(a.elapsed_time(b))
        mem.sync(hws, stream)
        same = bool(torch.equal(h_y, y.cpu()) and torch.equal(h_W, We.cpu()) and torch.equal(h_S, Se.cpu()))
        e_ms_max = max_over_ranks(statistics.mean(e_ms), world)
        e2e = {"value": aggregate_throughput(cnt["tokens"], world, e_ms_max * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": e_ms_max,
               "api": "tm_run_host", "segment_tokens": seg or "default (T/16 with a ramp of shorter segments at both ends)",
               "equal_to_device_run": same}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(w)
        cpu.pop("streams", None)
        cpu.pop("T", None)
    if rank == 0:
        line = {
            "metric": "memory tokens/sec (write+read)",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" and path_used in ("tc", "tcl", "tcl-phased") else
                     ("bf16-in/f32" if w.dtype == "bf16" else "f32"),
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "C": w.C, "dims": w.dims,
                       "theta_damping": w.theta_damping, "alpha_damping": w.alpha_damping,
                       "gates": ("literal" if (w.theta_damping == 1.0 and w.alpha_damping == 1.0) else
                                 f"damped: theta draws x{w.theta_damping}, alpha draws x{w.alpha_damping}"),
                       "path": path_used,
                       "l2": "flushed between steps (512 MB write)", "parallelism": f"replicas{world}"},
            "roofline": roof,
            "chunk_roofline": {"t_flop_ms": t_flop * 1e3, "t_state_io_ms": t_state * 1e3,
                               "bound": "state" if t_state > t_flop else "flop",
                               "frac": chunk_roofline_s / (ms_max * 1e-3),
                               "state_resident": "on-chip" if path_used == "tc" else "hbm/l2"},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps * launches_per_step,
            "clocks": clk, "finite": ok, "wall_s": t_wall, "step_ms": step_ms,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
