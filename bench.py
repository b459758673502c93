"""Benchmark: HQQ quantisation throughput on a Llama-2-70B-shaped weight set.

Default workload (`llama2-70b`): 80 decoder layers x (q, o 8192x8192; k, v
1024x8192; gate, up 28672x8192; down 8192x28672), fp16 synthetic weights with
the Llama-2 weight statistics (0.02*N(0,1), 0.1% outliers x10), per-layer
seeds; quantised whole at nbits/group 2/16 and at 4/128, 8-bit zero, group
stop.  One step = 1120 hqq_quantize calls, 136.9 G weights.

value     = weights quantised / device time (CUDA events), every layer resident
            in HBM (drawn on the GPU before the timed region; 137 GB).
e2e       = the same weight set end to end through hqq_quantize_stream_jobs
            (C ABI) with pinned host buffers: each step copies every weight in
            and every output out (PCIe-bound).
roofline  = the group-stop solver (solve_group_onepass_kernel), bound by the MUFU pipe
            that evaluates |r|^p (two ops per element and evaluated iterate),
            timed per hqq_quantize call with CUDA events on the launching
            stream; the HBM fraction of the same calls beside it.
cpu_baseline / --impl reference = the CPU oracle on a bounded sample.

Multi-GPU (torchrun): the layers are split across ranks (strong scaling, no
data-path collective); time = max over ranks.

Other workloads: `llama2-7b-mlp-sweep` (the Llama-2-7B MLP shapes at five
settings and two stop rules), `llama2-70b-stream` and `llama2-13b-stream`
(streamed models), and `--case` lines for single kernels.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from calibration_free_weight_b200 import synth  # noqa: E402

METRIC = "HQQ quantize Gweights/s and achieved HBM GB/s (% of B200 roofline) vs CPU oracle"
UNIT = "Gweights/s"
SWEEP = [(8, 128), (4, 64), (3, 64), (2, 16), (1, 16)]
MODES = [0, 1]  # stop_mode group, tensor
MATS = [("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
SMS = 148
MUFU_PER_CLK_PER_SM = 16
KERNEL_SOURCES = ["calibration_free_weight_b200/csrc/hqq_kernels.cu", "calibration_free_weight_b200/csrc/hqq_device.cuh"]
# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernel family per hqq_quantize call (its chunk launches and its output
# launch), averaged over the sweep's tensor-stop calls: one call per setting
# on the gate shape captured launch by launch (ncu, two DRAM metrics), the
# mean of the five (every setting has three calls of the same size); valid
# while the kernel sources hash to the captured ones.
TRAFFIC = {"src_sha256": "0c7c40747e8a1b6988d047afac0ab5f97f721b67ebefdc0dfa0e3c7c0079741d",
           "bytes_per_call": 390480000, "summary": "profiles/solve_tensor_kernel_11008x4096_b4g64.md"}


# DRAM traffic of one hqq_gemm call in the profiled case (ncu, same command as
# the summary), valid while hqq_gemm.cu hashes to the profiled source.
GEMM_SOURCES = ["calibration_free_weight_b200/csrc/hqq_gemm.cu"]
GEMM_TRAFFIC = {"src_sha256": "9ad1e18a87f9cdd83180be975fcb89b1f8c7da0978ccec10b870f0a5289f7093",
                "case": "gemm,28672,8192,4,64,256", "bytes_per_call": 145337088,
                "summary": "profiles/gemm_kernel_28672x8192_b4g64_batch256.md"}


# DRAM traffic of the group-stop solver on the 70B-shaped workload, as a ratio
# to the algorithmic bytes of the captured calls (ncu, one call per setting on
# the gate shape 28672x8192; see profiles/), valid while the kernel sources
# hash to the captured ones.
TRAFFIC70 = {"src_sha256": "0c7c40747e8a1b6988d047afac0ab5f97f721b67ebefdc0dfa0e3c7c0079741d",
             "bytes_per_alg_byte": {(2, 16): 625.87 / 572.52, (4, 128): 579.53 / 592.68},
             "summary": "profiles/solve_group_onepass_kernel_28672x8192_b2g16.md, ..._b4g128.md"}


def kernel_sources_sha(files=None):
    """sha256 of kernel sources (default: the solver's) with comments and
    blank lines removed: a change of code, not of commentary, invalidates the
    stored DRAM-traffic counters."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in files or KERNEL_SOURCES:
        with open(os.path.join(ROOT, f)) as fh:
            src = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        lines = (re.sub(r"//.*", "", ln).rstrip() for ln in src.splitlines())
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()


def solver_launches(mode, iters=20, g=64, axis=1):
    """Kernel launches of one hqq_quantize call (fp16 zero), as the library
    schedules them: group and no stop on axis 1 run one launch of the one-pass
    kernel; on axis 0 group stop runs passes of 2 and 3 evaluations and then
    the rest (no stop: one pass); tensor stop runs chunks of iterations [0,2)
    and then C at a time (C = 8 for g >= 32, with a last chunk shorter than 4
    merged into the one before; C = 4 for g <= 16), and one launch that writes
    the outputs."""
    if mode == 1:
        C = 4 if g <= 16 else 8
        if iters <= 0:
            n = 0
        elif iters <= 2:
            n = 1
        else:
            n = 1 + -(-(iters - 2) // C)
            if C >= 8 and n > 2 and (iters - 2) - (n - 2) * C < C // 2:
                n -= 1
        return n + 1
    if axis == 1 or mode == 2 or iters <= 2:
        return 1
    n, done = 0, 0
    for v in (2, 3):
        if done + v >= iters:
            break
        n, done = n + 1, done + v
    return n + 1


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("sm_max_mhz", 1965.0)), "measured"
    except Exception:
        return 6650.0, 1965.0, "fallback"


def _measured_peaks():
    """The measured peak figures (empty when the file is absent; the recipe's
    fallback for the dense bf16 figure is 1590 TFLOP/s burst)."""
    try:
        with open(PEAKS_FILE) as f:
            return json.load(f)
    except Exception:
        return {"bf16_tflops": 1590.0}


def algorithmic_bytes(rows, cols, nbits, g, zero_nbits=16):
    """One read of W (2 B/weight) + packed codes + fp16 scale + zero."""
    n = rows * cols
    G = n // g
    return 2 * n + n * nbits // 8 + 2 * G + (2 if zero_nbits == 16 else 1) * G


class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons; only the samples
    taken between mark_start() and mark_end() (the timed region) count."""

    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)  # let the sampler start before the timed region
        except Exception:
            self.proc = None
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        import datetime
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if self.t0 is not None and not (self.t0 <= ts <= self.t1):
                    continue
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


def make_inputs(layer):
    return {name: synth.weight(r, c, seed=synth.seed_for(layer, name), dtype=torch.bfloat16)
            for name, r, c in MATS}


def plan():
    """The 30 calls of one step, ordered so consecutive calls use different matrices."""
    calls = []
    for nbits, g in SWEEP:
        for mode in MODES:
            for name, r, c in MATS:
                calls.append((name, r, c, nbits, g, mode))
    return calls


# ----------------------------------------------------------------- oracle ---

def oracle_pass(ins, rows, nth):
    """One pass of the CPU oracle, as it stands, over a bounded sample of the
    step's work: the first `rows` output rows of every matrix at every setting
    and mode.  Returns (weights, seconds)."""
    import oracle
    t0 = time.perf_counter()
    n = 0
    for name, r, c, nbits, g, mode in plan():
        W = ins[name][:rows if name != "down" else max(1, rows * 4096 // 11008)].contiguous()
        Wb = W.view(torch.int16).numpy().view(np.uint16)
        oracle.quantize(Wb, nbits, g, 1, 0.7, 1.0, 1.01, 20, mode, 16, dtype=oracle.BF16, nthreads=nth)
        n += W.numel()
    return n, time.perf_counter() - t0


def oracle_calibrate(ins, pass_s, nth):
    """Rows per oracle pass so that one pass takes about pass_s seconds."""
    rows = 16
    while True:
        n, dt = oracle_pass(ins, rows, nth)
        if dt >= pass_s / 4 or rows >= 4096:
            return rows, n, dt
        rows *= 4


def oracle_desc(rows, n, nthreads=0):
    par = "one thread" if nthreads == 1 else "OpenMP over groups"
    return (f"first {rows} rows of gate/up (and the same element count of down) at all 10 settings/modes, "
            f"{n / 1e6:.2f} M weights per pass, bf16, {par}")


def oracle_sample_rate(layer, budget_s=12.0, nthreads=0):
    """Weights/s of the CPU oracle on a sample of about budget_s / 4 to budget_s
    seconds.  Returns (weights/s, threads used, sample description, n, s)."""
    import oracle
    oracle.lib()
    nth = nthreads or (os.cpu_count() or 1)
    rows, n, dt = oracle_calibrate(make_inputs(layer), budget_s, nth)
    return n / dt, nth, oracle_desc(rows, n), n, dt


def oracle_model_rate(Ws, settings, weights_total, rows=64, nthreads=0):
    """The CPU oracle, as it stands, on a deterministic sample of a streamed
    model: the first `rows` rows of each of one layer's matrices (host fp16
    tensors) with that matrix's settings; the whole model's oracle time is
    extrapolated from the sample's weights/s.  Returns a cpu_baseline dict."""
    import oracle
    nth = nthreads or (os.cpu_count() or 1)
    n, t0 = 0, time.perf_counter()
    for W, st in zip(Ws, settings):
        w = W[:rows].contiguous().numpy()
        oracle.quantize(w, st["nbits"], st["group_size"], 1, 0.7, 1.0, 1.01, 20, st["stop_mode"], st["zero_nbits"],
                        dtype=oracle.F16, nthreads=nth)
        n += w.size
    dt = time.perf_counter() - t0
    rate = n / dt
    return {"value": rate / 1e9, "unit": "Gweights/s", "cores": nth, "kind": "oracle",
            "sample": f"first {rows} rows of each matrix of one layer, {n / 1e6:.2f} M weights, "
                      f"fp16, OpenMP over groups", "extrapolated_model_s": weights_total / rate}


# ------------------------------------------------------------------- main ---

def dist_setup(backend="nccl"):
    """One process per GPU from the torchrun environment (RANK, LOCAL_RANK,
    WORLD_SIZE, MASTER_ADDR/PORT).  NCCL carries only the barrier and the max
    over ranks; the gloo backend serves the CPU tests of this path."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group(backend, timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x, world):
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def throughput(world, weights_per_step, steps, ms):
    """Whole-job G weights/s: every rank quantises weights_per_step per step
    (weak scaling), ms = the max over ranks of the timed region."""
    return world * weights_per_step * steps / (ms / 1e3) / 1e9


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle timed on the host cores, one bounded
    sample (about --ref-step seconds) per step.  Rank 0 only."""
    if rank != 0:
        return
    import oracle
    oracle.lib()
    nth = os.cpu_count() or 1
    ins = make_inputs(0)
    rows, _, _ = oracle_calibrate(ins, args.ref_step, nth)
    per_step = []
    for i in range(args.warmup + args.steps):
        n, dt = oracle_pass(ins, rows, nth)
        if i >= args.warmup:
            per_step.append((n, dt))
    desc = oracle_desc(rows, per_step[0][0] if per_step else 0)
    n = sum(a for a, _ in per_step)
    t = sum(b for _, b in per_step)
    value = n / t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_dict(world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nth, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def run_reference70(args, world, rank):
    """The reference arm of the llama2-70b workload: the CPU oracle, as it
    stands, on the machine's host cores; each step is a bounded sample of the
    workload (the first rows of every matrix of one layer at both settings,
    about --ref-step seconds; layer = step index, its seeds drawn on the host
    with the CPU generator).  Rank 0 only; the other ranks exit without work."""
    if rank != 0:
        return
    import oracle
    oracle.lib()
    nth = os.cpu_count() or 1
    mats = synth.LLAMA2_70B.matrices()
    probe = [synth.weight(64, c, seed=synth.seed_for(0, n), dtype=torch.float16) for n, r, c in mats]
    rows = oracle_rows_for_budget(probe, SETTINGS70B, args.ref_step, nth, rows0=8,
                                  rows_cap=min(r for _, r, _ in mats))
    per = []
    for i in range(args.warmup + args.steps):
        Ws = [synth.weight(rows, c, seed=synth.seed_for(i % args.layers, n), dtype=torch.float16)
              for n, r, c in mats]
        n_w, dt, _ = _oracle_fixed_rows(Ws, rows, nth)
        if i >= args.warmup:
            per.append((n_w, dt))
    n_w = sum(a for a, _ in per)
    t = sum(b for _, b in per)
    value = n_w / t / 1e9
    desc = (f"first {rows} rows of each of one layer's 7 matrices (layer = step index) at both settings, "
            f"{per[0][0] / 1e6:.2f} M weight-solves per step, fp16, OpenMP over groups")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config70(world, args.layers),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nth, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def _oracle_fixed_rows(Ws, rows, nth):
    import oracle
    n, t0 = 0, time.perf_counter()
    for nb, g in SETTINGS70B:
        for W in Ws:
            w = W[:rows].contiguous().numpy()
            oracle.quantize(w, nb, g, 1, 0.7, 1.0, 1.01, 20, 0, 8, dtype=oracle.F16, nthreads=nth)
            n += w.size
    return n, time.perf_counter() - t0, rows


def config_dict(world):
    return {"workload": "llama2-7b-mlp-sweep", "model": "Llama-2-7B MLP shapes (synthetic weights)",
            "matrices": "gate 11008x4096, up 11008x4096, down 4096x11008 (out x in), bf16",
            "settings": "nbits/group 8/128 4/64 3/64 2/16 1/16, axis 1, p 0.7, beta 1, kappa 1.01, 20 iters",
            "stop_modes": ["group", "tensor"], "zero": "fp16", "calls_per_step": len(plan()),
            "weights_per_step": sum(r * c for _, r, c, _, _, _ in plan()),
            "global_batch": world, "seq_len": None, "parallelism": f"replicas{world}",
            "l2": "inputs 270 MB > 126 MB L2; consecutive calls use different matrices"}


def run_scale8_case(spec):
    """Time hqq_quantize_scale8 (8-bit scales in runs of S) on G synthetic fp16
    scales: "scale8,G[,S[,reps]]".  HBM-bound: 2 B read + 1 B written per scale
    and 8 B per run."""
    from calibration_free_weight_b200 import hqq
    v = spec.split(",")[1:]
    G = int(v[0])
    S = int(v[1]) if len(v) > 1 else 128
    reps = int(v[2]) if len(v) > 2 else 20
    torch.cuda.set_device(0)
    q = {"scale": synth.scales(G, seed=G).cuda()}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # 256 MB > L2: each call starts cold
    hqq.quantize_scale8(q, S)
    ev = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        rc = hqq.hqq_quantize_scale8(q["scale"], G, S, q["scale_q"], q["scale_meta"])
        b.record()
        if rc != hqq.HQQ_OK:
            raise RuntimeError(hqq.hqq_status_string(rc))
        ev.append((a, b))
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in ev)
    med = ms[len(ms) // 2]
    nbytes = 3 * G + 8 * (-(-G // S))
    hbm, _, kind = peaks()
    print(json.dumps({"case": spec, "ms_median": med, "ms_min": ms[0], "bytes": nbytes,
                      "gbs": nbytes / (med / 1e3) / 1e9, "hbm_peak_gbs": hbm, "peak_kind": kind,
                      "frac": nbytes / (med / 1e3) / 1e9 / hbm, "l2": "flushed before every call"}))


LLAMA70B = [("q", 8192, 8192), ("k", 1024, 8192), ("v", 1024, 8192), ("o", 8192, 8192),
            ("gate", 28672, 8192), ("up", 28672, 8192), ("down", 8192, 28672)]


def rank_layers(layers, world, rank):
    """Layers a rank streams in the multi-GPU run: every world-th layer from
    its own index (whole layers per rank, no exchange between ranks)."""
    return list(range(rank, layers, world))


def run_stream(args):
    """Llama-2-70B-shaped model (80 layers x q, k, v, o, gate, up, down; fp16)
    streamed layer by layer from pinned host memory through hqq_quantize_stream
    at b2 g16 and b4 g128, 8-bit zero, group stop.  One layer of synthetic
    weights (layer 0's seeds) is generated and pinned, and every layer streams
    those buffers: each layer's copy-in, solve and copy-out is real, only the
    values repeat (137 GB of distinct synthetic weights would take minutes to
    generate).  Reports the end-to-end wall time of the blocking call and, for
    the same matrices resident on the device, the solver's throughput.
    Under torchrun each rank streams its share of the layers (rank_layers);
    the end-to-end time is the max over ranks of the blocking call's wall time
    between barriers."""
    from calibration_free_weight_b200 import hqq
    world, rank, local = dist_setup()
    layers = args.layers
    mine = len(rank_layers(layers, world, rank))
    Ws = [synth.weight(r, c, seed=synth.seed_for(0, n), dtype=torch.float16).pin_memory() for n, r, c in LLAMA70B]
    w_layer = sum(r * c for _, r, c in LLAMA70B)
    res = []
    for nbits, g in ((2, 16), (4, 128)):
        outs = [hqq.host_outputs(r, c, nbits, g, zero_nbits=8) for _, r, c in LLAMA70B]
        buf = hqq.quantize_stream(Ws, outs, nbits, g, zero_nbits=8)  # warm-up: one layer
        barrier(world)
        t0 = time.perf_counter()
        if mine:
            hqq.quantize_stream(Ws * mine, outs * mine, nbits, g, zero_nbits=8, device_buffer=buf)
        wall = max_over_ranks(time.perf_counter() - t0, world)
        barrier(world)
        del buf
        # the same matrices resident on the device: solver time per layer (CUDA events)
        dev = [w.cuda() for w in Ws]
        q = [hqq.alloc_outputs(r, c, nbits, g, 1, 0, 8) for _, r, c in LLAMA70B]
        for _ in range(2):
            for w, o in zip(dev, q):
                hqq.quantize(w, nbits, g, zero_nbits=8, out=o)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for w, o in zip(dev, q):
            hqq.quantize(w, nbits, g, zero_nbits=8, out=o)
        b.record()
        torch.cuda.synchronize()
        layer_ms = a.elapsed_time(b)
        alg = sum(algorithmic_bytes(r, c, nbits, g, 8) for _, r, c in LLAMA70B)
        hbm, _, kind = peaks()
        h2d = 2 * w_layer * layers
        d2h = sum(o["packed"].numel() + o["scale"].numel() * 2 + o["zero"].numel() + 8 for o in outs) * layers
        cpu = None
        if rank == 0:
            sets = [dict(nbits=nbits, group_size=g, stop_mode=0, zero_nbits=8)] * len(Ws)
            cpu = oracle_model_rate(Ws, sets, w_layer * layers)
        res.append({"nbits": nbits, "group_size": g, "e2e_s": wall, "e2e_gweights_s": w_layer * layers / wall / 1e9,
                    "cpu_baseline": cpu,
                    "h2d_bytes": h2d, "d2h_bytes": d2h, "h2d_gbs_effective": h2d / wall / 1e9,
                    "device_resident": {"ms_per_layer": layer_ms, "gweights_s": w_layer / (layer_ms / 1e3) / 1e9,
                                        "algorithmic_gbs": alg / (layer_ms / 1e3) / 1e9,
                                        "hbm_frac": alg / (layer_ms / 1e3) / 1e9 / hbm, "peak_kind": kind,
                                        "solve_s_all_layers": layer_ms / 1e3 * layers}})
        del dev, q
        torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps({"workload": "llama2-70b-stream", "layers": layers, "weights": w_layer * layers,
                          "n_gpus": world, "scaling": "layers split across ranks",
                          "dtype_in": "fp16", "zero": "8-bit", "stop_mode": "group", "host": "pinned",
                          "data": "synthetic; one layer's buffers streamed for every layer", "results": res}))
    if world > 1:
        torch.distributed.destroy_process_group()


SETTINGS70B = [(2, 16), (4, 128)]


def model70_calls(layers):
    """The hqq_quantize calls of one step of the Llama-2-70B-shaped workload on
    the given layers: the whole weight set at b2 g16, then at b4 g128."""
    mats = synth.LLAMA2_70B.matrices()
    return [(l, n, r, c, nb, g) for nb, g in SETTINGS70B for l in layers for n, r, c in mats]


def host_bytes_available():
    try:
        import psutil
        return int(psutil.virtual_memory().available)
    except Exception:
        return 0


def oracle_rows_for_budget(Ws, settings, budget_s, nth, rows0=16, rows_cap=None):
    """Rows per matrix so that the oracle over the first rows of every matrix
    at every setting takes about budget_s seconds (calibrated on rows0 rows;
    at most rows_cap, default the smallest matrix's row count)."""
    import oracle
    t0 = time.perf_counter()
    for W, (nb, g) in ((W, st) for st in settings for W in Ws):
        oracle.quantize(W[:rows0].contiguous().numpy(), nb, g, 1, 0.7, 1.0, 1.01, 20, 0, 8, dtype=oracle.F16,
                        nthreads=nth)
    dt = time.perf_counter() - t0
    rows = int(rows0 * budget_s / max(dt, 1e-3))
    return max(rows0, min(rows, rows_cap or min(W.shape[0] for W in Ws)))


def oracle_70b_sample(Ws, budget_s, nth):
    """The oracle, as it stands, on the first rows of each of one layer's
    matrices (host fp16) at both settings; returns (weights, seconds, rows)."""
    rows = oracle_rows_for_budget(Ws, SETTINGS70B, budget_s, nth)
    return _oracle_fixed_rows(Ws, rows, nth)


def config70(world, layers_total):
    mats = synth.LLAMA2_70B.matrices()
    w_layer = synth.LLAMA2_70B.weights_per_layer()
    return {"workload": "llama2-70b", "model": "Llama-2-70B shapes, synthetic weights",
            "layers": layers_total,
            "matrices": ", ".join(f"{n} {r}x{c}" for n, r, c in mats) + " (out x in), fp16",
            "settings": "nbits/group 2/16 and 4/128 (the whole weight set at each), axis 1, zero 8-bit, group stop, "
                        "p 0.7, beta 1, kappa 1.01, 20 iters",
            "calls_per_step": len(mats) * layers_total * len(SETTINGS70B),
            "weights_per_step": w_layer * layers_total * len(SETTINGS70B),
            "inputs": "per-layer seeds (1000*layer + matrix index), drawn on the GPU before the timed region, all "
                      "layers resident in HBM",
            "global_batch": world, "seq_len": None, "parallelism": f"layers split over {world} GPU(s)",
            "l2": "each step reads 137 GB of distinct weights, far above the 126 MB L2"}


def run_llama70(args):
    """The default workload: a Llama-2-70B-shaped weight set (80 layers x q, o
    8192x8192; k, v 1024x8192; gate, up 28672x8192; down 8192x28672; fp16,
    per-layer seeds) quantised whole at b2 g16 and at b4 g128, 8-bit zero, group
    stop.  One step = 1120 hqq_quantize calls over 136.9 G weights.

    value = weights / device time (CUDA events on the launching stream), every
            layer resident in HBM (drawn on the GPU before the timed region).
    e2e   = the same weight set end to end through hqq_quantize_stream_jobs with
            host buffers (pinned): every step copies all weights in and all
            outputs out; timed with CUDA events around the blocking call.
    Under torchrun the layers are split across ranks (rank_layers); each rank
    holds and quantises its own layers; time = max over ranks."""
    from calibration_free_weight_b200 import hqq
    world, rank, local = dist_setup()
    total_layers = args.layers
    layers = rank_layers(total_layers, world, rank)
    mats = synth.LLAMA2_70B.matrices()
    w_layer = synth.LLAMA2_70B.weights_per_layer()
    hbm_peak, sm_max, peak_kind = peaks()
    stream = torch.cuda.current_stream()

    t0 = time.perf_counter()
    Wd = {(l, n): synth.weight_device(r, c, synth.seed_for(l, n)) for l in layers for n, r, c in mats}
    torch.cuda.synchronize()
    gen_s = time.perf_counter() - t0

    outs, ws_bytes, g_max = {}, 0, 0
    for nb, g in SETTINGS70B:
        for n, r, c in mats:
            G = r * c // g
            outs[(n, nb, g)] = dict(packed=torch.empty(r * c * nb // 8, dtype=torch.uint8, device="cuda"),
                                    scale=torch.empty(G, dtype=torch.float16, device="cuda"),
                                    zero=torch.empty(G, dtype=torch.uint8, device="cuda"),
                                    zero_meta=torch.empty(2, dtype=torch.float32, device="cuda"))
            ws_bytes = max(ws_bytes, hqq.hqq_workspace_bytes(r, c, g, 1, 0, 8))
            g_max = max(g_max, G)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    calls = model70_calls(layers)

    def call(l, n, r, c, nb, g, dbg=None):
        o = outs[(n, nb, g)]
        rc = hqq.hqq_quantize(Wd[(l, n)], r, c, hqq.HQQ_F16, nb, g, 1, 0.7, 1.0, 1.01, 20, 0, 8, o["packed"],
                              o["scale"], o["zero"], o["zero_meta"], ws, ws.numel(), dbg)
        if rc != hqq.HQQ_OK:
            raise RuntimeError(hqq.hqq_status_string(rc))

    # algorithmic element-evaluations from the kept iterates (an untimed pass):
    # the stop rule needs e_0 .. e_{k*+1}, i.e. k* + 2 evaluations, at most iters
    bi_buf = torch.empty(g_max, dtype=torch.int32, device="cuda")
    ev_dev = torch.zeros((), dtype=torch.int64, device="cuda")
    for l, n, r, c, nb, g in calls:
        G = r * c // g
        call(l, n, r, c, nb, g, bi_buf[:G])
        ev_dev += (bi_buf[:G].to(torch.int64) + 2).clamp_(max=20).sum() * g
    evals = int(ev_dev.item())
    del bi_buf

    def one_step(rec=None):
        for cl in calls:
            if rec is not None:
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
            call(*cl)
            if rec is not None:
                b.record(stream)
                rec.append((a, b))

    for _ in range(args.warmup):
        one_step()
    barrier(world)
    rec = []
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        barrier(world)
        clk.mark_start()
        ev0.record(stream)
        for _ in range(args.steps):
            one_step(rec)
        ev1.record(stream)
        barrier(world)
        clk.mark_end()
    if hqq.hqq_get_status(ws) != hqq.HQQ_OK:
        raise RuntimeError("device status")
    dev_ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    w_rank_step = w_layer * len(layers) * len(SETTINGS70B)
    value = total_layers * w_layer * len(SETTINGS70B) * args.steps / (dev_ms / 1e3) / 1e9

    call_ms = sum(a.elapsed_time(b) for a, b in rec)
    n_calls = len(rec)
    avg_ms = call_ms / max(1, n_calls)
    mufu_ops = 2.0 * evals * args.steps  # over the timed calls
    mufu_peak = SMS * MUFU_PER_CLK_PER_SM * sm_max * 1e6 / 1e9
    achieved = mufu_ops / (call_ms / 1e3) / 1e9 if call_ms > 0 else 0.0
    alg_step = sum(algorithmic_bytes(r, c, nb, g, 8) for _, _, r, c, nb, g in calls)
    gbs = alg_step * args.steps / (call_ms / 1e3) / 1e9 if call_ms > 0 else 0.0
    traffic = None
    if TRAFFIC70["src_sha256"] == kernel_sources_sha():
        # DRAM bytes per algorithmic byte of the captured gate-shape calls, per setting,
        # applied to the benched calls' algorithmic bytes
        traffic = sum(TRAFFIC70["bytes_per_alg_byte"][(nb, g)] * algorithmic_bytes(r, c, nb, g, 8)
                      for _, _, r, c, nb, g in calls) / len(calls)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dev_ms / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (Llama-2-70B shapes, weight statistics 0.02*N(0,1) with 0.1% outliers x10)",
            "config": config70(world, total_layers),
            "roofline": {"bound": "alu", "kernel": "solve_group_onepass_kernel", "achieved": achieved, "peak": mufu_peak,
                         "unit": "Gop/s (MUFU lg2+ex2)", "frac": achieved / mufu_peak, "traffic": traffic,
                         "traffic_unit": "DRAM bytes per call", "traffic_basis": TRAFFIC70["summary"] +
                         " (ratio to algorithmic bytes per setting, scaled to the benched calls)",
                         "peak_kind": "nominal",
                         "peak_basis": f"{SMS} SMs x {MUFU_PER_CLK_PER_SM} MUFU ops/clk x {sm_max:.0f} MHz "
                                       f"(16/clk/SM confirmed by a microbenchmark of independent lg2/ex2 chains; "
                                       f"not driver-measured)",
                         "achieved_basis": "2 MUFU ops x (k*+2, at most 20) evaluations x group size, summed over "
                                           "the timed calls, / the sum of their CUDA-event durations",
                         "timed_unit": "one hqq_quantize call (its solver launches and the 8-bit zero launch)",
                         "avg_call_ms": avg_ms, "evals_per_weight": evals / max(1, w_rank_step),
                         "algorithmic_bytes_per_call": alg_step / len(calls),
                         "hbm_gbs": gbs, "hbm_peak_gbs": hbm_peak, "hbm_peak_kind": peak_kind,
                         "hbm_frac": gbs / hbm_peak},
            "gpu_launches": None, "clocks": clk.summary(), "input_generation_s": gen_s}
    line["gpu_launches"] = launches_per_call70(hqq) * len(calls) * args.steps

    # end to end through the C ABI with host buffers
    line["e2e"] = e2e70(args, hqq, world, rank, Wd, layers, mats, stream)
    del Wd, outs, ws
    torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nth = os.cpu_count() or 1
        Ws = [synth.weight_device(r, c, synth.seed_for(0, n)).cpu() for n, r, c in mats]
        n, dt, rows = oracle_70b_sample(Ws, args.ref_budget, nth)
        rate = n / dt
        # the same oracle on one host thread, on a 32 times smaller sample (about the same seconds)
        n1, dt1, rows1 = _oracle_fixed_rows(Ws, max(8, rows // 32), 1)
        line["cpu_baseline"] = {
            "value": rate / 1e9, "unit": UNIT, "cores": nth, "kind": "oracle",
            "sample": f"first {rows} rows of each of layer 0's 7 matrices at both settings, {n / 1e6:.1f} M "
                      f"weight-solves, fp16, OpenMP over groups",
            "extrapolated_model_s": w_layer * total_layers * len(SETTINGS70B) / rate,
            "single_thread": {"value": n1 / dt1 / 1e9, "cores": 1,
                              "sample": f"first {rows1} rows of each of layer 0's 7 matrices at both settings, "
                                        f"{n1 / 1e6:.2f} M weight-solves"}}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


def launches_per_call70(hqq):
    """Kernel launches of one group-stop hqq_quantize call with an 8-bit zero:
    the solver's passes and the 8-bit zero quantiser."""
    return solver_launches(0, 20, 16) + 1


def host_plan70(avail, w_layer_bytes, out_layer_bytes, nlayers):
    """How the end-to-end leg holds the weight set in host memory: (ring,
    outs_per_job).  Every layer's weights get their own pinned buffers when
    they fit (ring = nlayers), else a ring of as many layers as fit (at least
    one); outputs get a buffer set per job when those fit too, else one set
    per matrix and setting."""
    if avail >= (w_layer_bytes + out_layer_bytes) * nlayers:
        return nlayers, True
    if avail >= w_layer_bytes * nlayers + out_layer_bytes:
        return nlayers, False
    ring = int((avail - out_layer_bytes) // w_layer_bytes) if avail > out_layer_bytes else 1
    return max(1, min(ring, nlayers)), False


def e2e70(args, hqq, world, rank, Wd, layers, mats, stream):
    """The weight set through hqq_quantize_stream_jobs with host buffers.  The
    device-resident weights are copied into pinned host memory (one distinct
    buffer per matrix and layer when the host has room, else a ring of as many
    layers as fit, reused in layer order); host outputs per job when they fit,
    else per matrix and setting.  One untimed warm-up call on one layer, then
    e2e_steps timed calls over the whole set (each one copies every weight in
    and every output out)."""
    nset = len(SETTINGS70B)
    w_layer = sum(r * c for _, r, c in mats)
    out_layer = {(nb, g): sum(r * c * nb // 8 + 3 * (r * c // g) + 8 for _, r, c in mats) for nb, g in SETTINGS70B}
    ring, outs_per_job = host_plan70(host_bytes_available() - (16 << 30), 2 * w_layer, sum(out_layer.values()),
                                     len(layers))
    Wh = {}
    for i, l in enumerate(layers[:ring]):
        for n, r, c in mats:
            h = torch.empty(r, c, dtype=torch.float16, pin_memory=True)
            h.copy_(Wd[(l, n)])
            Wh[(i, n)] = h
    torch.cuda.synchronize()
    host_o = {}

    def host_out(key, r, c, nb, g):
        if key not in host_o:
            host_o[key] = hqq.host_outputs(r, c, nb, g, zero_nbits=8)
        return host_o[key]

    jobs_W, jobs_set, jobs_out = [], [], []
    for i, l in enumerate(layers):
        for n, r, c in mats:
            for nb, g in SETTINGS70B:  # consecutive jobs on one matrix share its device copy
                jobs_W.append(Wh[(i % ring, n)])
                jobs_set.append(dict(nbits=nb, group_size=g, axis=1, stop_mode=0, zero_nbits=8))
                key = (l, n, nb, g) if outs_per_job else (n, nb, g)
                jobs_out.append(host_out(key, r, c, nb, g))
    k = len(mats) * nset
    buf, _ = hqq.quantize_stream_jobs(jobs_W[:k], jobs_set[:k], jobs_out[:k])  # warm-up: one layer
    steps = max(1, min(args.steps, args.e2e_steps))
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        _, done = hqq.quantize_stream_jobs(jobs_W, jobs_set, jobs_out, device_buffer=buf)
        if done != len(jobs_W):
            raise RuntimeError("streamed run incomplete")
    e1.record(stream)
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = 2 * w_layer * len(layers)  # each matrix crosses once for both settings
    d2h = sum(out_layer.values()) * len(layers)
    del buf
    return {"value": args.layers * w_layer * nset * steps / (ms / 1e3) / 1e9, "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "s_per_step": ms / 1e3 / steps, "api": "hqq_quantize_stream_jobs (C ABI), host buffers pinned, "
                                                   "the two settings of a matrix as consecutive jobs on one copy",
            "host_weights": ("one buffer per matrix and layer" if ring == len(layers) else
                             f"a ring of {ring} layers' buffers reused in layer order (host memory)"),
            "host_outputs": "one set per job" if outs_per_job else "one set per matrix and setting, reused"}


LLAMA13B_NAMES = {"q": "self_attn.q_proj", "k": "self_attn.k_proj", "v": "self_attn.v_proj",
                  "o": "self_attn.o_proj", "gate": "mlp.gate_proj", "up": "mlp.up_proj", "down": "mlp.down_proj"}
LLAMA13B_CONFIG = dict(base=dict(nbits=4, group_size=64, stop_mode=1),
                       dynamic={"attn": dict(nbits=4, group_size=64, stop_mode=1),
                                "mlp": dict(nbits=2, group_size=32, stop_mode=1)})


def run_stream_mixed(args):
    """Llama-2-13B-shaped model (40 layers x q, k, v, o 5120x5120, gate/up
    13824x5120, down 5120x13824; fp16) with per-layer-type settings
    (attention b4 g64, MLP b2 g32, tensor stop, fp16 zero) streamed layer by
    layer from pinned host memory through hqq_quantize_stream_jobs.  As in
    the 70B workload, one layer of synthetic weights is streamed for every
    layer.  Under torchrun each rank streams its share of the layers."""
    from calibration_free_weight_b200 import hqq
    world, rank, local = dist_setup()
    model = synth.LLAMA2_13B
    layers = args.layers if args.layers_given else model.layers
    mine = len(rank_layers(layers, world, rank))
    mats = model.matrices()
    Ws = [synth.weight(r, c, seed=synth.seed_for(0, n), dtype=torch.float16).pin_memory() for n, r, c in mats]
    sets = [hqq.settings_for(f"model.layers.0.{LLAMA13B_NAMES[n]}", LLAMA13B_CONFIG["base"],
                             LLAMA13B_CONFIG["dynamic"]) for n, _, _ in mats]
    outs = [hqq.host_outputs(r, c, st["nbits"], st["group_size"], st["axis"], st["zero_nbits"])
            for (_, r, c), st in zip(mats, sets)]
    w_layer = model.weights_per_layer()
    buf, _ = hqq.quantize_stream_jobs(Ws, sets, outs)  # warm-up: one layer
    barrier(world)
    t0 = time.perf_counter()
    done = 0
    if mine:
        _, done = hqq.quantize_stream_jobs(Ws * mine, sets * mine, outs * mine, device_buffer=buf)
    wall = max_over_ranks(time.perf_counter() - t0, world)
    barrier(world)
    del buf
    # the same matrices resident on the device: solver time per layer (CUDA events)
    dev = [w.cuda() for w in Ws]
    q = [hqq.alloc_outputs(r, c, st["nbits"], st["group_size"], 1, st["stop_mode"], 16)
         for (_, r, c), st in zip(mats, sets)]
    call = lambda: [hqq.quantize(w, st["nbits"], st["group_size"], stop_mode=st["stop_mode"], out=o)  # noqa: E731
                    for w, st, o in zip(dev, sets, q)]
    for _ in range(2):
        call()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    call()
    b.record()
    torch.cuda.synchronize()
    layer_ms = a.elapsed_time(b)
    h2d = 2 * w_layer * layers
    d2h = sum(o["packed"].numel() + o["scale"].numel() * 2 + o["zero"].numel() * 2 for o in outs) * layers
    if rank == 0:
        cpu = oracle_model_rate(Ws, sets, w_layer * layers)
        print(json.dumps({"workload": "llama2-13b-stream", "cpu_baseline": cpu, "layers": layers, "weights": w_layer * layers,
                          "n_gpus": world, "scaling": "layers split across ranks", "dtype_in": "fp16",
                          "settings": {"attn (q, k, v, o)": sets[0], "mlp (gate, up, down)": sets[4]},
                          "zero": "fp16", "host": "pinned", "matrices_done_rank0": done,
                          "data": "synthetic; one layer's buffers streamed for every layer",
                          "e2e_s": wall, "e2e_gweights_s": w_layer * layers / wall / 1e9, "h2d_bytes": h2d,
                          "d2h_bytes": d2h, "h2d_gbs_effective": h2d / wall / 1e9,
                          "device_resident": {"ms_per_layer": layer_ms,
                                              "gweights_s": w_layer / (layer_ms / 1e3) / 1e9,
                                              "solve_s_all_layers": layer_ms / 1e3 * layers}}))
    if world > 1:
        torch.distributed.destroy_process_group()


def run_gemv_case(spec):
    """Time hqq_gemv (fused dequantisation + matrix-vector product) on one
    quantised synthetic fp16 matrix: "gemv,rows,cols,nbits,g[,batch[,reps]]".
    HBM-bound: codes b/8 B + fp16 scale and 8-bit zero 3/g B per weight, plus
    the activations and outputs; L2 flushed before every call."""
    from calibration_free_weight_b200 import hqq
    v = [int(x) for x in spec.split(",")[1:]]
    rows, cols, nbits, g = v[:4]
    batch = v[4] if len(v) > 4 else 1
    reps = v[5] if len(v) > 5 else 20
    torch.cuda.set_device(0)
    W = synth.weight(rows, cols, seed=7, dtype=torch.float16).cuda()
    q = hqq.quantize(W, nbits, g, zero_nbits=8)
    del W
    x = (synth.weight(batch, cols, seed=8, dtype=torch.float32) * 50).to(torch.float16).cuda()
    y = torch.empty(batch, rows, dtype=torch.float32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    hqq.gemv(q, x, rows, cols, nbits, g, zero_nbits=8, out=y)
    ev = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        hqq.gemv(q, x, rows, cols, nbits, g, zero_nbits=8, out=y)
        b.record()
        ev.append((a, b))
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in ev)
    med = ms[len(ms) // 2]
    G = rows * cols // g
    nbytes = rows * cols * nbits // 8 + 2 * G + G + 8 + batch * cols * 2 + batch * rows * 4
    hbm, _, kind = peaks()
    print(json.dumps({"case": spec, "ms_median": med, "ms_min": ms[0], "bytes": nbytes,
                      "gbs": nbytes / (med / 1e3) / 1e9, "hbm_peak_gbs": hbm, "peak_kind": kind,
                      "frac": nbytes / (med / 1e3) / 1e9 / hbm,
                      "gweights_s": rows * cols / (med / 1e3) / 1e9, "l2": "flushed before every call"}))


def run_gemm_case(spec):
    """Time hqq_gemm (fused dequantisation + tcgen05 matrix product) on one
    quantised synthetic matrix with bf16 activations:
    "gemm,rows,cols,nbits,g[,batch[,reps]]".  Reports TFLOP/s (2 rows cols
    batch per call) against the measured bf16 GEMM peak, and the HBM view
    (codes b/8 B + fp16 scale and 8-bit zero 3/g B per weight, activations,
    outputs); L2 flushed before every call."""
    from calibration_free_weight_b200 import hqq
    v = [int(x) for x in spec.split(",")[1:]]
    rows, cols, nbits, g = v[:4]
    batch = v[4] if len(v) > 4 else 128
    reps = v[5] if len(v) > 5 else 20
    torch.cuda.set_device(0)
    W = synth.weight(rows, cols, seed=7, dtype=torch.bfloat16).cuda()
    q = hqq.quantize(W, nbits, g, zero_nbits=8)
    del W
    x = synth.weight(batch, cols, seed=8, dtype=torch.float32, std=1.0).to(torch.bfloat16).cuda()
    y = torch.empty(batch, rows, dtype=torch.float32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    hqq.gemm(q, x, rows, cols, nbits, g, zero_nbits=8, out=y)
    ev = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        hqq.gemm(q, x, rows, cols, nbits, g, zero_nbits=8, out=y)
        b.record()
        ev.append((a, b))
    torch.cuda.synchronize()
    st = hqq.hqq_gemm_get_status()
    if st != hqq.HQQ_OK:
        raise RuntimeError(hqq.hqq_status_string(st))
    ms = sorted(a.elapsed_time(b) for a, b in ev)
    med = ms[len(ms) // 2]
    G = rows * cols // g
    nbytes = rows * cols * nbits // 8 + 2 * G + G + 8 + batch * cols * 2 + batch * rows * 4
    flops = 2.0 * rows * cols * batch
    hbm, _, kind = peaks()
    tf = _measured_peaks().get("bf16_tflops")
    # the oracle's product (fp64, one host thread) on a sample of rows, beside the kernel
    import oracle
    qc = {k: (v.cpu().numpy() if v is not None else None) for k, v in q.items() if k in
          ("packed", "scale", "zero", "zero_meta")}
    xo = x.cpu().view(torch.int16).numpy().view(np.uint16)
    sr = 8
    t0 = time.perf_counter()
    oracle.gemm(qc["packed"][:sr * cols * nbits // 8], qc["scale"][:sr * cols // g], qc["zero"][:sr * cols // g],
                qc["zero_meta"], sr, cols, nbits, g, 8, xo, oracle.BF16)
    ot = time.perf_counter() - t0
    achieved = flops / (med / 1e3) / 1e12
    same = ",".join(spec.split(",")[:6]) == GEMM_TRAFFIC["case"] and \
        kernel_sources_sha(GEMM_SOURCES) == GEMM_TRAFFIC["src_sha256"]
    print(json.dumps({"case": spec, "ms_median": med, "ms_min": ms[0], "tflops": achieved,
                      "roofline": {"bound": "tensor", "kernel": "gemm_kernel", "achieved": achieved, "peak": tf,
                                   "unit": "TFLOP/s", "frac": achieved / tf if tf else None,
                                   "peak_basis": "measured bf16 GEMM (burst)",
                                   "traffic": GEMM_TRAFFIC["bytes_per_call"] if same else None,
                                   "traffic_unit": "bytes per call", "algorithmic_bytes_per_call": nbytes},
                      "cpu_baseline": {"value": 2.0 * sr * cols * batch / ot / 1e12, "unit": "TFLOP/s", "cores": 1,
                                       "kind": "oracle", "sample": f"first {sr} rows, all columns, batch {batch}"},
                      "bf16_peak_tflops": tf, "tensor_frac": (flops / (med / 1e3) / 1e12 / tf) if tf else None,
                      "bytes": nbytes, "gbs": nbytes / (med / 1e3) / 1e9, "hbm_peak_gbs": hbm, "peak_kind": kind,
                      "hbm_frac": nbytes / (med / 1e3) / 1e9 / hbm, "l2": "flushed before every call"}))


def run_half_case(spec):
    """Time the half-precision solver variant beside hqq_quantize on one
    synthetic fp16 matrix: "half,rows,cols,nbits,g[,reps]" (group stop, 8-bit
    zero); L2 holds none of a large matrix between calls."""
    from calibration_free_weight_b200 import hqq
    v = [int(x) for x in spec.split(",")[1:]]
    rows, cols, nbits, g = v[:4]
    reps = v[4] if len(v) > 4 else 5
    torch.cuda.set_device(0)
    W = synth.weight(rows, cols, seed=4, dtype=torch.float16).cuda()
    res = {}
    for name, fn in (("fp32", hqq.quantize), ("half", hqq.quantize_half)):
        out = fn(W, nbits, g, zero_nbits=8)
        ev = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn(W, nbits, g, zero_nbits=8, out=out)
            b.record()
            ev.append((a, b))
        torch.cuda.synchronize()
        ms = min(a.elapsed_time(b) for a, b in ev)
        res[name] = {"ms": ms, "gweights_s": rows * cols / (ms / 1e3) / 1e9}
    print(json.dumps({"case": spec, **res, "half_over_fp32": res["fp32"]["ms"] / res["half"]["ms"]}))


def run_tensor_case(spec):
    """Tensor stop on one synthetic matrix, the resident launch (wherever it
    fits) beside the chunked launches:
    "tensor,rows,cols,nbits,g[,reps[,f16|bf16[,zero_nbits]]]" (seed-4 weights,
    20 iterations); "default_path" is the library's own choice.  Reports each path's best call time and
    its MUFU rate counted on the algorithmic evaluations (k* + 2 per group, at
    most 20; k* from a debug call) against the nominal MUFU peak."""
    from calibration_free_weight_b200 import hqq
    f = spec.split(",")[1:]
    rows, cols, nbits, g = (int(x) for x in f[:4])
    reps = int(f[4]) if len(f) > 4 else 5
    dtype = torch.float16 if len(f) > 5 and f[5] == "f16" else torch.bfloat16
    zb = int(f[6]) if len(f) > 6 else 16
    torch.cuda.set_device(0)
    W = synth.weight(rows, cols, seed=4, dtype=dtype).cuda()
    dbg = hqq.quantize(W, nbits, g, stop_mode=1, zero_nbits=zb, debug=True)
    kb = int(dbg["best_iter"][0].item())
    evals = min(kb + 2, 20)
    _, sm_max, _ = peaks()
    mufu_peak = SMS * MUFU_PER_CLK_PER_SM * sm_max * 1e6 / 1e9
    res = {}
    default = hqq.hqq_tensor_resident(rows, cols, 0 if dtype == torch.float16 else 1, g, 1, 20) == 1
    for name, on in (("resident", 2), ("chunked", 0)):
        prev = hqq.hqq_set_tensor_resident(on)
        try:
            used = hqq.hqq_tensor_resident(rows, cols, 0 if dtype == torch.float16 else 1, g, 1, 20) == 1
            out = hqq.quantize(W, nbits, g, stop_mode=1, zero_nbits=zb)
            ev = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                hqq.quantize(W, nbits, g, stop_mode=1, zero_nbits=zb, out=out)
                b.record()
                ev.append((a, b))
            torch.cuda.synchronize()
            st = hqq.hqq_get_status(out["workspace"])
            if st != hqq.HQQ_OK:
                raise RuntimeError(hqq.hqq_status_string(st))
        finally:
            hqq.hqq_set_tensor_resident(prev)
        ms = min(a.elapsed_time(b) for a, b in ev)
        gops = 2.0 * rows * cols * evals / (ms / 1e3) / 1e9
        res[name] = {"path": "resident" if used else "chunked", "ms": ms,
                     "gweights_s": rows * cols / (ms / 1e3) / 1e9, "mufu_gops": gops, "mufu_frac": gops / mufu_peak}
    print(json.dumps({"case": spec, "kept_iterate": kb, "evals_per_weight": evals, "mufu_peak_gops": mufu_peak,
                      "default_path": "resident" if default else "chunked",
                      **res, "chunked_over_resident": res["chunked"]["ms"] / res["resident"]["ms"]}))


def run_case(spec):
    """Time hqq_quantize on one synthetic matrix (used for kernel profiles)."""
    if spec.startswith("scale8"):
        run_scale8_case(spec)
        return
    if spec.startswith("gemv"):
        run_gemv_case(spec)
        return
    if spec.startswith("gemm"):
        run_gemm_case(spec)
        return
    if spec.startswith("half"):
        run_half_case(spec)
        return
    if spec.startswith("tensor"):
        run_tensor_case(spec)
        return
    from calibration_free_weight_b200 import hqq
    f = spec.split(",")
    mode, rows, cols, nbits, g = (int(x) for x in f[:5])
    reps = int(f[5]) if len(f) > 5 else 3
    dtype = torch.float16 if len(f) > 6 and f[6] == "f16" else torch.bfloat16
    zb = int(f[7]) if len(f) > 7 else 16
    torch.cuda.set_device(0)
    W = synth.weight(rows, cols, seed=4, dtype=dtype).cuda()
    out = hqq.alloc_outputs(rows, cols, nbits, g, 1, mode, zb)
    ev = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        hqq.quantize(W, nbits, g, stop_mode=mode, zero_nbits=zb, out=out)
        b.record()
        ev.append((a, b))
    torch.cuda.synchronize()
    st = hqq.hqq_get_status(out["workspace"])
    if st != hqq.HQQ_OK:
        raise RuntimeError(hqq.hqq_status_string(st))
    ms = [a.elapsed_time(b) for a, b in ev]
    print(json.dumps({"case": spec, "ms_per_call": ms, "gweights_s_last": rows * cols / (ms[-1] / 1e3) / 1e9}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--ref-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-step", type=float, default=1.0, help="seconds of oracle work per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None,
                    help="single-matrix timing: stop_mode,rows,cols,nbits,group_size[,reps[,f16|bf16[,zero_nbits]]] "
                         "(seed-4 synthetic weights, bf16 and fp16 zero by default); "
                         "or scale8,G[,S[,reps]] for the 8-bit scale quantiser, "
                         "or gemv,rows,cols,nbits,g[,batch[,reps]] for the fused dequantise + matrix-vector product, "
                         "or half,rows,cols,nbits,g[,reps] for the half-precision solver variant beside the fp32 one, "
                         "or tensor,rows,cols,nbits,g[,reps[,f16|bf16[,zero_nbits]]] for tensor stop on its "
                         "resident launch beside its chunked launches")
    ap.add_argument("--workload", default="llama2-70b",
                    choices=["llama2-70b", "llama2-7b-mlp-sweep", "llama2-70b-stream", "llama2-13b-stream"])
    ap.add_argument("--layers", type=int, default=None,
                    help="layers of a model workload (default: the model's, 80 or 40)")
    ap.add_argument("--e2e-steps", type=int, default=2,
                    help="timed steps of the end-to-end leg of the llama2-70b workload (at most --steps)")
    args = ap.parse_args()
    args.layers_given = args.layers is not None
    if args.workload == "llama2-70b" and not args.case:
        if not args.layers_given:
            args.layers = 80
        if args.impl == "reference":
            run_reference70(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        else:
            run_llama70(args)
        return
    if args.workload == "llama2-70b-stream":
        if not args.layers_given:
            args.layers = 80
        run_stream(args)
        return
    if args.workload == "llama2-13b-stream":
        run_stream_mixed(args)
        return
    if args.case:
        run_case(args.case)
        return

    if args.impl == "reference":
        # CPU oracle only: rank 0 times it, other ranks exit without work
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup()

    from calibration_free_weight_b200 import hqq
    hbm_peak, sm_max, peak_kind = peaks()
    layer = rank
    ins_cpu = make_inputs(layer)
    ins = {k: v.cuda() for k, v in ins_cpu.items()}
    calls = plan()
    stream = torch.cuda.current_stream()
    outs = {}
    for name, r, c, nbits, g, mode in calls:
        outs[(name, nbits, g, mode)] = hqq.alloc_outputs(r, c, nbits, g, 1, mode, 16)

    # algorithmic work per call: element-evaluations from the kept iterates (untimed pass)
    evals = {}
    for name, r, c, nbits, g, mode in calls:
        q = hqq.quantize(ins[name], nbits, g, stop_mode=mode, debug=True)
        bi = q["best_iter"].to(torch.int64)
        e = torch.where(bi >= 19, torch.full_like(bi, 20), bi + 2) if mode == 0 else \
            torch.full_like(bi, min(int(bi[0]) + 2, 20))
        evals[(name, nbits, g, mode)] = int(e.sum().item()) * g
        del q
    torch.cuda.synchronize()

    def one_step(record=None):
        for name, r, c, nbits, g, mode in calls:
            o = outs[(name, nbits, g, mode)]
            if record is not None:
                record.append((mode, torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                               (name, nbits, g, mode)))
                record[-1][1].record(stream)
            rc = hqq.hqq_quantize(ins[name], r, c, hqq.HQQ_BF16, nbits, g, 1, 0.7, 1.0, 1.01, 20, mode, 16,
                                  o["packed"], o["scale"], o["zero"], None, o["workspace"], o["workspace"].numel())
            if rc != hqq.HQQ_OK:
                raise RuntimeError(hqq.hqq_status_string(rc))
            if record is not None:
                record[-1][2].record(stream)

    for _ in range(args.warmup):
        one_step()
    barrier(world)
    rec = []
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        barrier(world)
        clk.mark_start()
        torch.cuda.nvtx.range_push("timed steps")
        ev0.record(stream)
        for _ in range(args.steps):
            one_step(rec)
        ev1.record(stream)
        torch.cuda.nvtx.range_pop()
        barrier(world)
        clk.mark_end()
    for o in outs.values():
        st = hqq.hqq_get_status(o["workspace"])
        if st != hqq.HQQ_OK:
            raise RuntimeError(hqq.hqq_status_string(st))
    dev_ms = ev0.elapsed_time(ev1)
    dev_ms = max_over_ranks(dev_ms, world)
    w_step = sum(r * c for _, r, c, _, _, _ in calls)
    value = throughput(world, w_step, args.steps, dev_ms)

    # per-launch durations by kernel family
    fam = {0: [], 1: []}
    for mode, a, b, key in rec:
        fam[mode].append((a.elapsed_time(b), key))
    tot = {m: sum(t for t, _ in v) for m, v in fam.items()}
    dom = max(tot, key=tot.get)
    dom_name = "solve_tensor_kernel" if dom == 1 else "solve_group_onepass_kernel"
    n_l = len(fam[dom])
    avg_ms = tot[dom] / n_l
    mufu_ops = sum(2 * evals[key] for _, key in fam[dom]) / n_l  # per call
    mufu_peak = SMS * MUFU_PER_CLK_PER_SM * sm_max * 1e6 / 1e9  # Gop/s
    achieved = mufu_ops / (avg_ms / 1e3) / 1e9
    # HBM view of the same launches (the metric's second half)
    bytes_dom = sum(algorithmic_bytes(*[(r, c) for n_, r, c in MATS if n_ == key[0]][0], key[1], key[2])
                    for _, key in fam[dom]) / n_l
    gb_dom = bytes_dom / (avg_ms / 1e3) / 1e9
    bytes_step = sum(algorithmic_bytes(r, c, nb, g) for _, r, c, nb, g, _ in calls)
    hbm_step = bytes_step * args.steps / (dev_ms / 1e3) / 1e9 * world
    grp = fam[0]
    g_ms = sum(t for t, _ in grp) / max(1, len(grp))
    g_bytes = sum(algorithmic_bytes(*[(r, c) for n_, r, c in MATS if n_ == key[0]][0], key[1], key[2])
                  for _, key in grp) / max(1, len(grp))
    g_w = sum([(r * c) for _, key in grp for n_, r, c in MATS if n_ == key[0]]) / max(1, len(grp))

    traffic = TRAFFIC["bytes_per_call"] if TRAFFIC["src_sha256"] == kernel_sources_sha() else None

    # end to end through the C ABI with host buffers
    pinned = {k: v.pin_memory() for k, v in ins_cpu.items()}
    host_out = {key: {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in o.items()
                      if k in ("packed", "scale", "zero")} for key, o in outs.items()}
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for o in host_out.values() for v in o.values())

    def e2e_step():
        for k, v in pinned.items():
            ins[k].copy_(v, non_blocking=True)
        one_step()
        for key, o in outs.items():
            for k, v in host_out[key].items():
                v.copy_(o[k], non_blocking=True)

    e2e_step()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = throughput(world, w_step, args.steps, e2e_ms)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dev_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config_dict(world),
            "roofline": {"bound": "alu", "kernel": dom_name, "achieved": achieved, "peak": mufu_peak,
                         "unit": "Gop/s (MUFU lg2+ex2)", "frac": achieved / mufu_peak, "traffic": traffic,
                         "traffic_unit": "bytes per call", "algorithmic_bytes_per_call": bytes_dom,
                         "peak_basis": f"{SMS} SMs x {MUFU_PER_CLK_PER_SM} MUFU/clk x {sm_max:.0f} MHz",
                         "timed_unit": f"one hqq_quantize call = {solver_launches(dom, 20, 64) - 1} (g >= 32) or "
                                       f"{solver_launches(dom, 20, 16) - 1} (g <= 16) chunk launches of {dom_name} "
                                       f"and one tensor_output_kernel",
                         "avg_launch_ms": avg_ms, "hbm_gbs": gb_dom, "hbm_frac": gb_dom / hbm_peak},
            "hbm": {"achieved_gbs_step": hbm_step, "peak_gbs": hbm_peak, "peak_kind": peak_kind,
                    "frac_step": hbm_step / hbm_peak,
                    "group_mode": {"avg_launch_ms": g_ms, "gbs": g_bytes / (g_ms / 1e3) / 1e9,
                                   "frac": g_bytes / (g_ms / 1e3) / 1e9 / hbm_peak,
                                   "gweights_s": g_w / (g_ms / 1e3) / 1e9}},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": sum(solver_launches(mode, 20, g) for _, _, _, _, g, mode in calls) * args.steps,
            "clocks": clk.summary()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, nth, desc, _, _ = oracle_sample_rate(0, budget_s=args.ref_budget)
        # the same sample on one host thread
        n1, t1 = oracle_pass(make_inputs(0), 16, 1)
        line["cpu_baseline"] = {"value": rate / 1e9, "unit": UNIT, "cores": nth, "kind": "oracle", "sample": desc,
                                "single_thread": {"value": n1 / t1 / 1e9, "cores": 1,
                                                  "sample": oracle_desc(16, n1, 1)}}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
