#!/usr/bin/env python
"""Attention throughput benchmark (one JSON line on rank 0).

A step is one pass of the whole hot path over one batch: the forward kernel
(O, LSE) and the three backward stages (prepare, the fused tile kernel,
finish) -> dQ, dK, dV.  Workload: B=1, H=32, N=32768, d=128, causal, dropout
p=0.1 (seed 4), bf16 inputs drawn by the seeded recipe of
``exact_io_aware_49_b200.workloads``.  Q, K, V, dO are 268 MB each, larger
than the 126 MB L2, so no flush is needed between steps.

FLOPs per step: forward 4*B*H*N^2*d/2 (causal), backward 2.5x the forward.

  value     fwd+bwd TFLOP/s over all ranks, inputs resident in HBM, timed with
            CUDA events on the launching stream (max over ranks)
  e2e       the same through the C ABI's host-buffer call fa_fwd_bwd_host:
            each step copies Q, K, V, dO host->device from pinned memory and
            O, LSE, dQ, dK, dV back, in 16 groups of heads whose copies overlap
            the kernels of the neighbouring groups on three streams
  roofline  the kernel with the largest share of the step, achieved TFLOP/s
            from its own CUDA events against the measured bf16 burst peak
  other_workloads  fa_fwd and the backward on B=4 H=16 N=4096 d=128 causal
            p=0.1 (the other dropout workload) and on the wide head dims
            (B=2 H=16 N=8192 d=192 and d=256, causal, p=0.1), each call timed
            with CUDA events (median), TFLOP/s and % of the burst peak
  cpu_baseline  the fp64 oracle on this host's cores on a bounded sample
            (a causal prefix of one head, which is itself a complete causal
            attention problem)

``--impl reference`` times that oracle instead (rank 0 only).

``--other-workloads-only`` prints just those per-call timings (a short run,
also the command the wide kernels' ncu capture profiles).

``--decode`` prints a different line instead: the paged-cache decode kernel
(fa_decode_paged) on 16 sequences x 32768 cached positions, 32 query / 8
key-value heads, d=128, one query per sequence, pages of 64 positions in
shuffled order; value = bytes of K and V read per call / call time (GB/s),
roofline against the measured HBM copy bandwidth.
Multi-GPU (torchrun): every rank runs the full workload on its own GPU -- the
(b, h) units are independent, so there is no collective on the data path;
``scaling`` is "weak" and value sums the ranks' work over the slowest rank.
"""

import argparse
import datetime
import hashlib
import json
import os
import re
import subprocess
import sys
import time

_CORES = len(os.sched_getaffinity(0))
for _var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_var, str(_CORES))

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from exact_io_aware_49_b200 import workloads as wl  # noqa: E402

METRIC = "attention TFLOP/s fwd & fwd+bwd (bf16) and % of B200 dense BF16 peak"
WORKLOAD = "causal_dropout_N32768_d128"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TILES_SOURCE = os.path.join(ROOT, "exact_io_aware_49_b200", "csrc", "fa_bwd.cu")
FWD_SOURCE = os.path.join(ROOT, "exact_io_aware_49_b200", "csrc", "fa_fwd.cu")
DECODE_SOURCE = os.path.join(ROOT, "exact_io_aware_49_b200", "csrc", "fa_decode.cu")
DECODE_WORKLOAD = "decode_paged_B16_L32768_H32_Hkv8_d128"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")
E2E_GROUPS = 16  # head groups of the host-buffer step (copies of one overlap the kernels of the next)


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return {k: float(m[k]) for k in FALLBACK}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK), "fallback"


def _sha(path):
    """Hash of a kernel source's code: comments and whitespace removed, so that
    a recorded capture stays tied to the code it measured and nothing else."""
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = " ".join(text.split())
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def _traffic(kernel, source, workload=WORKLOAD):
    """DRAM bytes per launch from the committed ncu summary, if taken on this exact source."""
    try:
        with open(TRAFFIC_FILE) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload and parts[2] == _sha(source):
                    return float(parts[3])
    except OSError:
        pass
    return None


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (200 ms) kept only inside [start, stop]."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.t0 = self.t1 = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, RuntimeError):
            self.proc = None

    def start(self):
        self.t0 = time.time()

    def stop(self):
        self.t1 = time.time()
        if not self.proc:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return self._parse(out)

    def _parse(self, out):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            if not (self.t0 - 0.25 <= ts <= self.t1 + 0.25):
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------- oracle legs

def oracle_prefix_step(q, k, v, do, w, b, h, n):
    """fp64 oracle fwd + bwd on the causal prefix [0, n) of head (b, h); returns its FLOPs."""
    from oracle import attention
    args = [x[b, h, :n].to(torch.float64).numpy() for x in (q, k, v, do)]
    kw = dict(causal=w.causal, scale=w.scale, p_drop=w.p_drop, seed=w.seed, b=b, h=h)
    attention.forward(*args[:3], **kw)
    attention.backward(*args, **kw)
    return 3.5 * 4.0 * n * n * w.d / (2 if w.causal else 1)


def cpu_baseline(q, k, v, do, w, n=4096, min_seconds=10.0):
    n = min(n, w.N)
    flops, reps = 0.0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < min_seconds or reps == 0:
        flops += oracle_prefix_step(q, k, v, do, w, 0, reps % w.H, n)
        reps += 1
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": _CORES, "kind": "oracle",
            "sample": f"fp64 NumPy oracle, fwd+bwd of the causal prefix N={n} (a complete causal attention "
                      f"problem) of {reps} head(s) of this workload, {dt:.1f} s"}


# --------------------------------------------------------------------- arms

def run_reference(args, w, world):
    if world["rank"] != 0:
        return None
    q, k, v, do = wl.draw_inputs(w)
    n = min(2048, w.N)
    for i in range(args.warmup):
        oracle_prefix_step(q, k, v, do, w, 0, i % w.H, n)
    t0 = time.perf_counter()
    flops = 0.0
    for i in range(args.steps):
        flops += oracle_prefix_step(q, k, v, do, w, 0, i % w.H, n)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world["size"],
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _CORES, "kind": "oracle",
                         "sample": f"each step: fp64 NumPy oracle fwd+bwd of the causal prefix N={n} of one head"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def _config(w):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "p_drop": w.p_drop,
            "seed": w.seed, "l2": "no flush: Q, K, V, dO are 268 MB each, larger than the 126 MB L2",
            "parallelism": "one full workload per rank (independent (b, h) units, no data-path collective)"}


def run_ours(args, w, world, device):
    from exact_io_aware_49_b200 import binding
    binding.load_library()
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    qh, kh, vh, doh = (x.pin_memory() for x in wl.draw_inputs(w))
    q, k, v, do = (x.to(device) for x in (qh, kh, vh, doh))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), device=device, dtype=torch.float32)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(binding.fa_bwd_workspace_size(w.B, w.H, w.N, w.d), device=device, dtype=torch.uint8)
    flops_fwd, flops_bwd = w.fwd_flops(), w.bwd_flops()

    ev = {}

    def step(record):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(6)] if record else None
        if record:
            e[0].record(stream)
        binding.fa_fwd(q, k, v, w.causal, w.scale, w.p_drop, w.seed, out=o, lse=lse)
        if record:
            e[1].record(stream)
        binding.fa_bwd_stages(q, k, v, o, do, lse, w.causal, w.scale, w.p_drop, w.seed, workspace=ws, dq=dq,
                              dk=dk, dv=dv, between=(lambda i: e[2 + i].record(stream)) if record else None)
        if record:
            ev.setdefault("steps", []).append(e)

    for _ in range(args.warmup):
        step(False)
    _barrier(world)
    torch.cuda.synchronize(device)
    sampler = ClockSampler(device) if world["local_rank"] == 0 or world["size"] == 1 else None
    time.sleep(0.6 if sampler else 0.0)  # let nvidia-smi produce its first sample before the region
    if sampler:
        sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step(True)
    t_end.record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop() if sampler else None
    _barrier(world)
    ms_step = t_start.elapsed_time(t_end) / args.steps
    per = np.array([[e[0].elapsed_time(e[1]), e[2].elapsed_time(e[5]), e[3].elapsed_time(e[4])]
                    for e in ev["steps"]])
    fwd_ms, bwd_ms, tiles_ms = per.mean(axis=0)
    ms_step_max = _max_over_ranks(world, ms_step, device)

    # ---- end to end through the C ABI on host buffers (fa_fwd_bwd_host): each
    # step copies Q, K, V, dO in from pinned memory and O, LSE, dQ, dK, dV out,
    # in groups of heads whose copies overlap the kernels on three streams
    oh = torch.empty_like(qh).pin_memory()
    dqh, dkh, dvh = (torch.empty_like(qh).pin_memory() for _ in range(3))
    lseh = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    groups = E2E_GROUPS
    host_ws = torch.empty(binding.fa_fwd_bwd_host_workspace_size(w.B, w.H, w.N, w.d, groups), device=device,
                          dtype=torch.uint8)
    streams = [torch.cuda.Stream(device) for _ in range(3)]

    def e2e_step():
        binding.fa_fwd_bwd_host(qh, kh, vh, doh, w.causal, w.scale, w.p_drop, w.seed, groups=groups, device=device,
                                workspace=host_ws, streams=streams, out=oh, lse=lseh, dq=dqh, dk=dkh, dv=dvh)

    e2e_steps = max(1, min(args.steps, 10))
    for _ in range(min(args.warmup, 2)):
        e2e_step()
    _barrier(world)
    torch.cuda.synchronize(device)
    a = torch.cuda.Event(enable_timing=True)
    bev = torch.cuda.Event(enable_timing=True)
    a.record(streams[2])  # each call starts after the work on its copy-out stream
    for _ in range(e2e_steps):
        e2e_step()
    bev.record(streams[2])
    torch.cuda.synchronize(device)
    e2e_ms = _max_over_ranks(world, a.elapsed_time(bev) / e2e_steps, device)
    h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh, doh))
    d2h = sum(x.numel() * x.element_size() for x in (oh, lseh, dqh, dkh, dvh))

    from exact_io_aware_49_b200 import fa_last_device_error
    if fa_last_device_error() != 0:
        raise RuntimeError("a bounded device wait timed out during the benchmark")

    peaks, peak_src = _peaks()
    n = world["size"]
    flops_step = flops_fwd + flops_bwd
    value = n * flops_step / (ms_step_max * 1e-3) / 1e12
    # dominant kernel: the larger of the forward kernel and the backward tile kernel
    if tiles_ms >= fwd_ms:
        kname, k_ms, k_flops, src = "fa_bwd_tiles", tiles_ms, flops_bwd, TILES_SOURCE
    else:
        kname, k_ms, k_flops, src = "fa_fwd", fwd_ms, flops_fwd, FWD_SOURCE
    achieved = k_flops / (k_ms * 1e-3) / 1e12
    # the dominant kernel runs ~30 ms at a time inside a sub-second timed
    # region: the burst figure is its peak; the sustained fraction is kept beside it
    peak = peaks["bf16_tflops"]
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded randn, bf16)", "config": _config(w),
        "fwd_tflops": flops_fwd / (fwd_ms * 1e-3) / 1e12,
        "bwd_tflops": flops_bwd / (bwd_ms * 1e-3) / 1e12,
        "fwd_bwd_tflops": value / n,
        "pct_of_peak": {
            "fwd_vs_measured_burst": 100 * flops_fwd / (fwd_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "bwd_vs_measured_burst": 100 * flops_bwd / (bwd_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "fwd_vs_datasheet": 100 * flops_fwd / (fwd_ms * 1e-3) / 1e12 / DATASHEET_BF16_TFLOPS,
            "bwd_vs_datasheet": 100 * flops_bwd / (bwd_ms * 1e-3) / 1e12 / DATASHEET_BF16_TFLOPS,
            "peak_source": peak_src,
        },
        "kernel_ms": {"fa_fwd": fwd_ms, "fa_bwd (3 stages)": bwd_ms, "fa_bwd_tiles": tiles_ms},
        "roofline": {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_kind": f"bf16_tflops, burst ({peak_src})",
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "traffic": _traffic(kname, src)},
        "e2e": {"value": n * flops_step / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "call": f"fa_fwd_bwd_host (C ABI, pinned host buffers, {groups} head groups, 3 streams)"},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
    }
    if w.name == WORKLOAD and not args.no_other_workloads and world["rank"] == 0:
        # after the last collective; only rank 0's line carries them
        out["other_workloads"] = time_other_workloads(device, peaks)
    return out, (qh, kh, vh, doh)


# the other d = 128 causal dropout workload the throughput target names, then
# the head dims the d <= 128 kernels cannot hold (their own kernels, seeded as
# the recipe of exact_io_aware_49_b200.workloads draws every input)
OTHER_WORKLOADS = [
    "causal_dropout_N4096_d128",
    wl.Workload("causal_dropout_N8192_d192", 2, 16, 8192, 192, True, 0.1, 21),
    wl.Workload("causal_dropout_N8192_d256", 2, 16, 8192, 256, True, 0.1, 22),
]


def time_other_workloads(device, peaks):
    out = {}
    for o in OTHER_WORKLOADS:
        w = wl.BY_NAME[o] if isinstance(o, str) else o
        out[w.name] = time_other_workload(w, device, peaks)
    return out


def time_other_workload(w, device, peaks, reps=20, warmup=3):
    """fa_fwd and the backward (three stages) on another workload's inputs,
    each call timed alone with CUDA events on the launching stream (median of
    ``reps``); reported beside the main line, not part of its value."""
    from exact_io_aware_49_b200 import binding
    stream = torch.cuda.current_stream(device)
    q, k, v, do = (x.to(device) for x in wl.draw_inputs(w))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), device=device, dtype=torch.float32)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(binding.fa_bwd_workspace_size(w.B, w.H, w.N, w.d), device=device, dtype=torch.uint8)
    # d <= 128: the three stages (prepare, tiles, finish); wider heads: fa_bwd,
    # whose dK / dV and dQ kernels write the gradients directly
    stages = binding.fa_bwd_stages if w.d <= 128 else binding.fa_bwd
    tf, tb = [], []
    for it in range(warmup + reps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        binding.fa_fwd(q, k, v, w.causal, w.scale, w.p_drop, w.seed, out=o, lse=lse)
        e[1].record(stream)
        stages(q, k, v, o, do, lse, w.causal, w.scale, w.p_drop, w.seed, workspace=ws, dq=dq, dk=dk, dv=dv)
        e[2].record(stream)
        torch.cuda.synchronize(device)
        if it >= warmup:
            tf.append(e[0].elapsed_time(e[1]))
            tb.append(e[1].elapsed_time(e[2]))
    fwd_ms, bwd_ms = float(np.median(tf)), float(np.median(tb))
    fwd_tf = w.fwd_flops() / (fwd_ms * 1e-3) / 1e12
    bwd_tf = w.bwd_flops() / (bwd_ms * 1e-3) / 1e12
    return {"B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "p_drop": w.p_drop,
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
            "fwd_pct_of_burst": 100 * fwd_tf / peaks["bf16_tflops"],
            "bwd_pct_of_burst": 100 * bwd_tf / peaks["bf16_tflops"],
            "timing": f"CUDA events per call, median of {reps} after {warmup} warm-up calls; "
                      f"inputs (Q, K, V, dO {q.numel() * 2 / 1e6:.0f} MB each) are resident, no L2 flush"}


# --------------------------------------------------------------------- decode line

DECODE = dict(B=16, H=32, H_kv=8, Nq=1, d=128, L=32768, page=64, seed=7)


def run_decode(args, device):
    """Paged-cache decode: HBM GB/s of the cached K and V per call (one GPU)."""
    from exact_io_aware_49_b200 import binding
    c = DECODE
    B, H, H_kv, Nq, d, L, page = c["B"], c["H"], c["H_kv"], c["Nq"], c["d"], c["L"], c["page"]
    gen = torch.Generator(device="cpu").manual_seed(c["seed"])
    n_pages = B * ((L + page - 1) // page)
    kc = torch.randn(n_pages, page, H_kv, d, generator=gen, dtype=torch.float32).to(torch.bfloat16).to(device)
    vc = torch.randn(n_pages, page, H_kv, d, generator=gen, dtype=torch.float32).to(torch.bfloat16).to(device)
    table = torch.randperm(n_pages, generator=gen).to(torch.int32).view(B, -1).to(device)
    lens = torch.full((B,), L, dtype=torch.int32, device=device)
    qh = torch.randn(B, H, Nq, d, generator=gen, dtype=torch.float32).to(torch.bfloat16).pin_memory()
    q = qh.to(device)
    lib = binding.load_library()
    splits = int(lib.fa_decode_num_splits(B, H_kv, H, Nq, L))
    ws = torch.empty(max(1, int(lib.fa_decode_workspace_size(B, H, Nq, d, splits))), dtype=torch.uint8,
                     device=device)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, Nq, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def call(qq):
        return binding.fa_decode_paged(qq, kc, vc, table, lens, L, True, d ** -0.5, num_splits=splits, out=o,
                                       lse=lse, workspace=ws)

    for _ in range(args.warmup):
        call(q)
    torch.cuda.synchronize(device)
    sampler = ClockSampler(device)
    time.sleep(0.6)
    sampler.start()
    evs = []
    for _ in range(args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call(q)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    kv_bytes = 2 * B * L * H_kv * d * 2
    io_bytes = kv_bytes + 2 * q.numel() * 2 + lse.numel() * 4
    # end to end through the public API: the step's query in, output and LSE out
    oh = torch.empty_like(qh).pin_memory()
    lseh = torch.empty(B, H, Nq, dtype=torch.float32).pin_memory()
    for _ in range(2):
        q.copy_(qh, non_blocking=True)
        call(q)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        q.copy_(qh, non_blocking=True)
        call(q)
        oh.copy_(o, non_blocking=True)
        lseh.copy_(lse, non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = a.elapsed_time(b) / args.steps
    if binding.fa_last_device_error() != 0:
        raise RuntimeError("a bounded device wait timed out during the decode benchmark")
    peaks, peak_src = _peaks()
    achieved = io_bytes / (ms * 1e-3) / 1e9
    # oracle on a bounded sample: one sequence, the 4 query heads of one key/value head
    from oracle import paged
    qs = qh[:1, :4].to(torch.float64).numpy()
    pages0 = table[0].long()
    kcs = kc[pages0][:, :, :1].to(torch.float64).cpu().numpy()  # sequence 0's pages, key/value head 0
    vcs = vc[pages0][:, :, :1].to(torch.float64).cpu().numpy()
    tab = np.arange(kcs.shape[0], dtype=np.int32)[None]
    t0 = time.time()
    n_rep = 0
    while time.time() - t0 < 10.0:
        paged.decode_forward(qs, kcs, vcs, tab, np.array([L]), causal=True, scale=d ** -0.5)
        n_rep += 1
    cpu_s = (time.time() - t0) / n_rep
    cpu_bytes = 2 * L * 1 * d * 2
    return {
        "metric": "paged-cache decode attention: K/V bytes read per second (bf16)", "value": kv_bytes / (ms * 1e-3) / 1e9,
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded randn, bf16; pages in shuffled order)",
        "config": {"workload": DECODE_WORKLOAD, **{k: v for k, v in c.items() if k != "seed"},
                   "causal": True, "num_splits": splits,
                   "l2": "no flush: the K/V cache is 2.1 GB, larger than the 126 MB L2"},
        "roofline": {"bound": "hbm", "kernel": "fa_decode_kernel (+ split merge)", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "peak_kind": f"hbm_gbs ({peak_src})", "algorithmic_bytes": io_bytes,
                     "traffic": _traffic("fa_decode", DECODE_SOURCE, DECODE_WORKLOAD)},
        "e2e": {"value": kv_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": qh.numel() * 2, "d2h_bytes_per_step": oh.numel() * 2 + lseh.numel() * 4},
        "gpu_launches": args.steps * (2 if splits > 1 else 1),
        "clocks": clocks,
        "cpu_baseline": {"value": cpu_bytes / cpu_s / 1e9, "unit": "GB/s", "cores": _CORES, "kind": "oracle",
                         "sample": f"fp64 NumPy paged oracle, 1 sequence x 4 query heads of one key/value head, "
                                   f"{L} positions, {n_rep} runs in {time.time() - t0:.1f} s"},
    }


# --------------------------------------------------------------------- plumbing

def _world():
    size = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return {"size": size, "rank": rank, "local_rank": local, "pg": None}


def _barrier(world):
    if world["size"] > 1:
        torch.distributed.barrier()


def _max_over_ranks(world, x, device):
    if world["size"] == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(wl.BY_NAME))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the per-call timings of the other workloads beside the main line")
    ap.add_argument("--decode", action="store_true", help="the paged-cache decode line instead (one GPU)")
    ap.add_argument("--other-workloads-only", action="store_true",
                    help="only the per-call timings of the other workloads (one GPU)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.decode:
        print(json.dumps(run_decode(args, torch.device("cuda", 0))), flush=True)
        return
    if args.other_workloads_only:
        peaks, peak_src = _peaks()
        res = {"other_workloads": time_other_workloads(torch.device("cuda", 0), peaks), "peak_source": peak_src}
        print(json.dumps(res), flush=True)
        return
    w = wl.BY_NAME[args.workload]
    world = _world()
    if world["size"] > 1:
        backend = "nccl" if args.impl == "ours" else "gloo"
        if args.impl == "ours":
            torch.cuda.set_device(world["local_rank"])
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            res = run_reference(args, w, world)
        else:
            device = torch.device("cuda", world["local_rank"])
            res, inputs = run_ours(args, w, world, device)
            if world["rank"] == 0 and world["size"] == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(*inputs, w)
            elif world["rank"] == 0:
                res["cpu_baseline"] = None
        if world["rank"] == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world["size"] > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
