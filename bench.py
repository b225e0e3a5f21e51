#!/usr/bin/env python3
"""Benchmark of the HQQ quantize + dequantize path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole path over the workload's weight set: HQQ
quantize (fused solver + packing) of every matrix, then dequantize of every
matrix.  Inputs are generated on the device before timing and stay resident in
HBM (the default workload holds ~137 GB of fp16 weights, far above the 126 MB
L2, so no L2 flush is needed between steps).  Under torchrun every rank
quantizes its own full weight set (weak scaling, no collective on the data
path); the step time is the max over ranks.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the plain CPU
oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Gparams/s quantized & achieved HBM GB/s vs B200 peak; Llama-2-70B-shaped wall time"

# Algorithmic binary32 operations per weight of the canonical solver, counted
# by hand from its steps (reported beside the measured instruction count, not
# used for the roofline): initialisation (convert, min, max), one error
# evaluation (code: fma, 2 clamps, round; residual: sub, fma; |.|; table power:
# 4 bit-field ops, sub, mul, 3 fma, 2 mul; accumulate), one accepted update
# with W_e == 0 (threshold test, fma, accumulate), final code and packing
# (fma, 2 clamps, round, shift, or).
OPS_INIT, OPS_EVAL, OPS_UPDATE, OPS_FINAL = 3, 19, 3, 6
ALU_LANES_PER_SM = 128
# Each SM has four warp schedulers, each issuing at most one warp instruction
# per cycle: the issue peak the quantize kernel's instruction count is held to.
ISSUE_PER_SM_CLK = 4


# ------------------------------------------------------------------ workloads
def workload(name: str, rank: int = 0, layers: int | None = None):
    """List of (label, (rows, cols), nbits, group, seed, stream)."""
    import synth
    out = []
    if name in ("llama2-70b", "llama2-7b"):
        big = name == "llama2-70b"
        shapes = synth.llama2_70b_shapes() if big else synth.llama2_7b_shapes()
        n_layers, seed, nbits = (80, 5, 3) if big else (32, 2, 4)
        if layers is not None:
            n_layers = min(n_layers, layers)
        for layer in range(rank * n_layers, (rank + 1) * n_layers):
            for m in synth.MATRIX_ORDER:
                out.append((f"L{layer}.{m}", shapes[m], nbits, 64, seed,
                            synth.stream_id(layer, m)))
    elif name == "matrix-4096":
        out.append(("4096x4096 4b g64", (4096, 4096), 4, 64, 1, rank))
        out.append(("4096x4096 2b g32", (4096, 4096), 2, 32, 1, rank))
    elif name == "gate-70b":
        out.append(("L0.gate 28672x8192 3b g64", (28672, 8192), 3, 64, 5, rank * 7 + 4))
    elif name == "matrix-1024":
        out.append(("1024x1024 4b g64", (1024, 1024), 4, 64, 0, rank))
    elif name == "70b-pair":
        for g in (32, 128):
            out.append((f"8192x8192 2b g{g}", (8192, 8192), 2, g, 3, 2 * rank))
            out.append((f"28672x8192 2b g{g}", (28672, 8192), 2, g, 3, 2 * rank + 1))
    else:
        raise SystemExit(f"unknown workload {name}")
    return out


def max_over_ranks(values, pg, device=None):
    """Element-wise max of a list of floats over all ranks (identity at N = 1)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if pg is not None:
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def meta_bytes(rows, cols, group):
    return 2 * 2 * rows * (cols // group)


def algorithmic_bytes(mats):
    """One pass: read fp16 W, write packed codes + fp16 scale and zero."""
    import weight_only_quantization_b200 as hqq
    tot = 0
    for _, (r, c), nb, g, _, _ in mats:
        tot += 2 * r * c + hqq.hqq_packed_bytes(r, c, nb) + meta_bytes(r, c, g)
    return tot


# ------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------- helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def tensor_peak():
    """Dense fp16/bf16 tensor-core peak in TFLOP/s: the measured cuBLAS bf16 burst
    figure (fp16 runs at the same rate), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        return 1590.0


def profiled_counters(kernel: str, fmt: str):
    """Per-weight counters of `kernel` from the committed ncu summary whose
    source hash matches the current sources: DRAM bytes per weight and warp
    instructions per weight (each None when absent), and the summary's path;
    all None when the kernel's sources changed since the counters were taken."""
    import glob
    import hashlib
    srcs = {"quantize_kernel": ["hqq_quantize.cuh", "hqq_common.cuh"],
            "dequantize_kernel": ["hqq_dequantize.cu", "hqq_common.cuh"]}[kernel]
    m = hashlib.sha256()
    for f in srcs:
        with open(os.path.join(ROOT, "weight_only_quantization_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    cur = m.hexdigest()[:16]
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", f"{kernel}_*{fmt}*.txt"))):
        kv = {}
        with open(path) as fh:
            for line in fh:
                if ":" in line and not line.startswith("#"):
                    k, _, v = line.partition(":")
                    kv[k.strip()] = v.strip()
        if kv.get("source_sha256_16") == cur:
            get = lambda k: float(kv[k]) if k in kv else None
            return {"traffic_bytes_per_param": get("traffic_bytes_per_param"),
                    "warp_inst_per_param": get("warp_inst_per_param"),
                    "source": os.path.relpath(path, ROOT)}
    return {"traffic_bytes_per_param": None, "warp_inst_per_param": None, "source": None}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample(mats, W_source, target_s: float):
    """Bounded sample of the workload for the CPU oracle: the first rows of every
    distinct (shape, format) in the list, sized to ~target_s seconds of oracle
    work on this host's cores.  W_source(label, shape, rows) -> fp16 numpy."""
    import numpy as np
    import oracle
    seen, picks = set(), []
    for lab, shape, nb, g, seed, stream in mats:
        key = (shape, nb, g)
        if key not in seen:
            seen.add(key)
            picks.append((lab, shape, nb, g, seed, stream))
    cores = cpu_cores()
    # probe the rate on 16 rows of the first pick
    lab, shape, nb, g, seed, stream = picks[0]
    probe = W_source(lab, shape, 16, seed, stream)
    t0 = time.perf_counter()
    oracle.quantize(probe, nb, g, threads=cores)
    rate = probe.size / max(time.perf_counter() - t0, 1e-6)
    budget = rate * target_s
    total_cols = sum(s[1] for _, s, *_ in picks)
    rows = max(8, min(min(s[0] for _, s, *_ in picks), int(budget / total_cols)))
    sample = [(lab, W_source(lab, shape, rows, seed, stream), nb, g)
              for lab, shape, nb, g, seed, stream in picks]
    desc = "quantize + dequantize of the first %d rows of each distinct matrix: " % rows + \
        ", ".join(f"{lab.split('.')[-1]} {shape[0]}x{shape[1]}" for lab, shape, *_ in picks)
    return sample, desc, cores


def run_oracle_sample(sample, cores):
    """The step on the sample: quantize every sampled matrix, then dequantize
    its codes (the oracle's quantize is threaded over groups, its dequantize
    runs on one core)."""
    import oracle
    n = 0
    t0 = time.perf_counter()
    for _, W, nb, g in sample:
        r = oracle.quantize(W, nb, g, threads=cores)
        oracle.dequantize(r["codes"], r["scale"], r["zero"], g)
        n += W.size
    return n, time.perf_counter() - t0


def config_dict(name, mats, n_gpus):
    params = sum(r * c for _, (r, c), *_ in mats)
    fmts = sorted({f"{m[2]}b g{m[3]}" for m in mats})
    return {"workload": name, "matrices_per_gpu": len(mats), "params_per_gpu": params,
            "formats": fmts, "solver": {"p": 0.7, "beta": 1.0, "kappa": 1.01, "iters": 20,
                                        "early_stop": "per group"},
            "step": "quantize + dequantize of every matrix",
            "l2": "inputs larger than L2 (no flush needed)" if params * 2 > 4 * 126e6
            else "L2 flushed between steps (256 MiB written, outside the step events)",
            "parallelism": f"replicas x{n_gpus} (weak)"}


# ------------------------------------------------------------ reference arm
def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np
    import synth
    mats = workload(args.workload, 0, args.layers)

    use_dev = False
    try:
        import torch
        use_dev = torch.cuda.is_available()
    except ImportError:
        pass

    def W_source(lab, shape, rows, seed, stream):
        # input generation only (the device generator is much faster than numpy's)
        if use_dev:
            return synth.student_t_device((rows, shape[1]), seed=seed, stream=stream).cpu().numpy()
        return synth.student_t_host((rows, shape[1]), seed=seed, stream=stream)

    sample, desc, cores = oracle_sample(mats, W_source, target_s=args.ref_step_s)
    for _ in range(args.warmup):
        run_oracle_sample(sample, cores)
    times, n = [], 0
    for _ in range(args.steps):
        n, dt = run_oracle_sample(sample, cores)
        times.append(dt)
    total = sum(times)
    value = n * len(times) / total / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "Gparam/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_dict(args.workload, mats, args.gpus),
            "cpu_baseline": {"value": value, "unit": "Gparam/s", "cores": cores,
                             "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": desc + f"; {n} params per step"},
            "e2e": {"value": value, "unit": "Gparam/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ main arm
def run_gpu(args):
    import numpy as np
    import torch

    import synth
    import weight_only_quantization_b200 as hqq

    ws, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
        pg = dist

    # ---- the other workloads first (their memory is released before the main
    # set is allocated): quantize and dequantize GB/s per matrix (single
    # matrices and the 70B pair) or per set (the 7B-shaped set), each pass
    # replayed as a CUDA graph with L2 flushed before every repetition
    configs = None
    if not args.no_configs:
        configs = run_configs(hqq, dev, measured_peaks()[0], pg, rank)
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    mats = workload(args.workload, rank, args.layers)
    params = sum(r * c for _, (r, c), *_ in mats)

    # ---- resident buffers: weights, packed codes, scale/zero, dequant output
    offs_w, offs_p, offs_m = [], [], []
    nw = npk = nm = 0
    for _, (r, c), nb, g, _, _ in mats:
        offs_w.append(nw); nw += r * c
        offs_p.append(npk); npk += (hqq.hqq_packed_bytes(r, c, nb) + 15) // 16 * 16
        offs_m.append(nm); nm += (r * (c // g) + 7) // 8 * 8
    maxn = max(r * c for _, (r, c), *_ in mats)
    need = 2 * nw + npk + 4 * nm + 2 * maxn * 3 + (1 << 30)
    free_b, _ = torch.cuda.mem_get_info(dev)
    if need > free_b:
        raise SystemExit(f"workload {args.workload} needs {need / 1e9:.1f} GB of device memory, "
                         f"{free_b / 1e9:.1f} GB free")
    Wbuf = torch.empty(nw, dtype=torch.float16, device=dev)
    Pbuf = torch.empty(npk, dtype=torch.uint8, device=dev)
    Sbuf = torch.empty(nm, dtype=torch.float16, device=dev)
    Zbuf = torch.empty(nm, dtype=torch.float16, device=dev)
    Obuf = torch.empty(maxn, dtype=torch.float16, device=dev)

    views = []
    for k, (lab, (r, c), nb, g, seed, stream) in enumerate(mats):
        W = Wbuf[offs_w[k]:offs_w[k] + r * c].view(r, c)
        synth.fill_student_t_(W, seed=seed, stream=stream)
        pb = hqq.hqq_packed_bytes(r, c, nb)
        P = Pbuf[offs_p[k]:offs_p[k] + pb]
        mg = r * (c // g)
        S = Sbuf[offs_m[k]:offs_m[k] + mg].view(r, c // g)
        Z = Zbuf[offs_m[k]:offs_m[k] + mg].view(r, c // g)
        q = hqq.QuantizedMatrix(P, S, Z, r, c, nb, g)
        views.append((W, q, Obuf[:r * c].view(r, c)))
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()

    def quantize_all():
        for W, q, O in views:
            hqq.hqq_quantize(W, q.nbits, q.group, packed=q.packed, scale=q.scale,
                             zero=q.zero)

    def dequantize_all():
        for W, q, O in views:
            hqq.hqq_dequantize(q, out=O)

    # one pass = every matrix quantized, then every matrix dequantized; the two
    # loops of library calls are captured once in CUDA graphs (host launch cost
    # out of the way of small matrices) unless --no-graph
    quantize_all()
    dequantize_all()
    torch.cuda.synchronize()
    if not args.no_graph:
        gq, gd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gq):
            quantize_all()
        with torch.cuda.graph(gd):
            dequantize_all()
        run_q, run_d = gq.replay, gd.replay
    else:
        run_q, run_d = quantize_all, dequantize_all

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        run_q()
        if ev is not None:
            ev[1].record(stream)
        run_d()

    def barrier():
        if pg is not None:
            pg.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # small workloads: overwrite a buffer twice the size of L2 before every step,
    # outside the step's own events (the step time is the sum of those)
    flush = None
    if params * 2 <= 4 * 126e6:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start.record(stream)
    for s in range(args.steps):
        if flush is not None:
            flush.fill_(s & 0xFF)
        step(evs[s])
        evs[s][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = sum(evs[s][0].elapsed_time(evs[s][2]) for s in range(args.steps))
    q_ms = [evs[s][0].elapsed_time(evs[s][1]) for s in range(args.steps)]
    ms_max, qsum_max = max_over_ranks([ms, sum(q_ms)], pg, dev)
    ms_step = ms_max / args.steps
    value = ws * params * args.steps / (ms_max / 1e3) / 1e9

    # ---- per-kernel figures (rank 0's launches)
    q_launch_ms = sum(q_ms) / args.steps / len(views)
    dq_ms_step = ms_step - sum(q_ms) / args.steps
    hbm_peak, peak_kind = measured_peaks()
    qbytes = algorithmic_bytes(mats)
    q_step_s = sum(q_ms) / args.steps / 1e3
    quant_gbs = qbytes / q_step_s / 1e9
    dq_gbs = qbytes / max(dq_ms_step / 1e3, 1e-9) / 1e9

    # ---- algorithmic ALU work of the solver from the per-group iteration counts
    acc_hist = np.zeros(256, np.int64)
    max_groups = max(q.scale.numel() for _, q, _ in views)
    zf_buf = torch.empty(max_groups, dtype=torch.float32, device=dev)
    it_buf = torch.empty(max_groups, dtype=torch.uint8, device=dev)
    for W, q, _ in views:
        ng = q.scale.numel()
        qq = hqq.hqq_quantize_ex(W, q.nbits, q.group, packed=q.packed, scale=q.scale,
                                 zero=q.zero, zero_f32=zf_buf[:ng].view(q.scale.shape),
                                 iters_out=it_buf[:ng].view(q.scale.shape))
        acc_hist += torch.bincount(qq.iters.view(-1).long(), minlength=256).cpu().numpy()[:256]
    torch.cuda.synchronize()
    del zf_buf, it_buf
    acc = np.arange(256)
    evals = np.where(acc < 20, acc + 1, acc)
    n_groups_hist = acc_hist.sum()
    mean_acc = float((acc_hist * acc).sum() / n_groups_hist)
    mean_eval = float((acc_hist * evals).sum() / n_groups_hist)
    ops_per_weight = OPS_INIT + OPS_FINAL + mean_eval * OPS_EVAL + mean_acc * OPS_UPDATE
    props = torch.cuda.get_device_properties(dev)
    sm_mhz = (clk or {}).get("sm_mhz") or 1965.0

    # ---- roofline of the dominant kernel (quantize_kernel): the issue rate of
    # its warp instructions (counted by ncu on the committed profile of the
    # same sources, per weight) against 4 warp instructions per SM per cycle at
    # the SM clock sampled during the timed region; HBM fraction beside it
    fmts = sorted({f"{m[2]}b_g{m[3]}" for m in mats})
    ctr = profiled_counters("quantize_kernel", fmts[0]) if len(fmts) == 1 else \
        {"traffic_bytes_per_param": None, "warp_inst_per_param": None, "source": None}
    w_per_launch = params / len(views)
    traffic = (ctr["traffic_bytes_per_param"] * w_per_launch
               if ctr["traffic_bytes_per_param"] is not None else None)
    issue_peak = props.multi_processor_count * ISSUE_PER_SM_CLK * sm_mhz * 1e6 / 1e12  # T inst/s
    ipw = ctr["warp_inst_per_param"]
    issue_achieved = ipw * params / q_step_s / 1e12 if ipw is not None else None
    alu_peak = props.multi_processor_count * ALU_LANES_PER_SM * sm_mhz * 1e6 / 1e12  # Tops/s
    roof = {"kernel": "quantize_kernel", "bound": "alu",
            "achieved": issue_achieved, "peak": issue_peak, "unit": "T warp-inst/s",
            "frac": issue_achieved / issue_peak if issue_achieved is not None else None,
            "traffic": traffic, "traffic_unit": "bytes per launch",
            "counter_source": ctr["source"],
            "peak_source": f"{props.multi_processor_count} SMs x {ISSUE_PER_SM_CLK} warp "
                           f"instructions per cycle x {sm_mhz:.0f} MHz (sampled)",
            "warp_inst_per_weight_measured": ipw,
            "ops_per_weight_algorithmic": ops_per_weight,
            "algorithmic_ops_frac_of_fp32_lanes":
                ops_per_weight * params / q_step_s / 1e12 / alu_peak,
            "hbm": {"achieved_gbs": quant_gbs, "peak_gbs": hbm_peak,
                    "frac": quant_gbs / hbm_peak, "peak_kind": peak_kind,
                    "algorithmic_bytes_per_weight": qbytes / params}}

    line = {"metric": METRIC, "value": value, "unit": "Gparam/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic (Philox Student-t(4), std 0.02, 0.1% x20 outliers, fp16)",
            "config": config_dict(args.workload, mats, ws),
            "wall_time_s_per_pass": ms_step / 1e3,
            "quantize": {"gparam_s": params / q_step_s / 1e9, "gbs": quant_gbs,
                         "hbm_frac": quant_gbs / hbm_peak, "ms_per_pass": q_step_s * 1e3,
                         "mean_accepted_iters": mean_acc, "mean_evaluations": mean_eval},
            "dequantize": {"gbs": dq_gbs, "hbm_frac": dq_gbs / hbm_peak,
                           "ms_per_pass": dq_ms_step},
            "roofline": roof,
            "gpu_launches": 2 * len(views) * args.steps,
            "clocks": clk}

    # ---- weight-only linear layer on the quantized matrices
    if not args.no_linear:
        line["linear"] = run_linear(args, views, hqq, dev, hbm_peak, tensor_peak(), pg)

    # ---- 8-bit meta data (zero points: one group; scales: groups of 128)
    if not args.no_meta:
        line["meta8"] = run_meta8(args, views, hqq, dev, hbm_peak, pg)

    # ---- low-rank residual of the quantization error (before the RTN pass,
    # which overwrites the HQQ codes)
    if not args.no_lowrank:
        line["lowrank"] = run_lowrank(views, hqq, dev, alu_peak, pg)

    # ---- the half-precision solver over the same set (overwrites the codes;
    # runs after the sections above, which use the single-precision ones)
    line["quantize_fp16"] = run_quantize_half(views, hqq, dev, hbm_peak, qbytes, pg)

    # ---- memory-side calibration: round-to-nearest quantize pass (HBM-bound;
    # runs after the sections above, which use the HQQ codes)
    line["rtn"] = run_rtn(views, hqq, dev, hbm_peak, qbytes, pg)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    if ws == 1 and not args.no_cpu_baseline:
        def W_source(lab, shape, rows, seed, stream_):
            k = [m[0] for m in mats].index(lab)
            return views[k][0][:rows].cpu().numpy()
        sample, desc, cores = oracle_sample(mats, W_source, target_s=args.cpu_s)
        n = dt = 0.0
        reps = 0
        while dt < args.cpu_s and reps < 100:
            n1, dt1 = run_oracle_sample(sample, cores)
            n, dt, reps = n + n1, dt + dt1, reps + 1
        desc += f"; repeated {reps}x"
        line["cpu_baseline"] = {"value": n / dt / 1e9, "unit": "Gparam/s", "cores": cores,
                                "kind": "oracle", "cpu_model": cpu_model(),
                                "sample": desc + f"; {n} params, {dt:.1f} s"}

    # ---- model-shaped sets: one streamed pass, each layer's weights generated
    # on the device into one reused buffer and then quantized (wall time)
    if args.workload in ("llama2-70b", "llama2-7b") and not args.no_stream:
        line["stream_pass"] = run_stream_pass(mats, hqq, dev, views)

    # ---- end to end through the public API with host buffers
    if not args.no_e2e:
        line["e2e"] = run_e2e(args, mats, views, hqq, dev, pg, ws)

    if configs is not None:
        line["configs"] = configs
    del views, Wbuf, Pbuf, Sbuf, Zbuf, Obuf
    if rank == 0:
        print(json.dumps(line))
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def run_configs(hqq, dev, hbm_peak, pg, rank):
    """Quantize and dequantize GB/s of every other workload, on device-resident
    inputs: the 1024x1024 matrix (4-bit g64), the 4096x4096 matrix at 4-bit g64
    and 2-bit g32, the 8192x8192 and 28672x8192 pair at 2-bit g32 and g128 (per
    matrix), and the 7B-shaped set at 4-bit g64 (the whole set per pass).  Each
    pass is a CUDA graph of the library calls, repeated with a 256 MiB buffer
    written before every repetition (outside its events), so no repetition
    starts with its inputs in the 126 MB L2."""
    import torch
    import synth
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn, reps):
        g = torch.cuda.CUDAGraph()
        fn()
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            flush.fill_(1)
            g.replay()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        torch.cuda.synchronize()
        for r in range(reps):
            flush.fill_(r & 0xFF)
            evs[r][0].record(stream)
            g.replay()
            evs[r][1].record(stream)
        torch.cuda.synchronize()
        ms = statistics.median(a.elapsed_time(b) for a, b in evs)
        del g
        return max_over_ranks([ms], pg, dev)[0]

    def record(mats, ms_q, ms_d):
        params = sum(r * c for _, (r, c), *_ in mats)
        nbytes = algorithmic_bytes(mats)
        out = {}
        for name, ms in (("quantize", ms_q), ("dequantize", ms_d)):
            gbs = nbytes / (ms / 1e3) / 1e9
            out[name] = {"ms": ms, "gparam_s": params / (ms / 1e3) / 1e9, "gbs": gbs,
                         "hbm_frac": gbs / hbm_peak}
        return out

    def prepare(mats):
        res = []
        for lab, (r, c), nb, g, seed, st in mats:
            W = torch.empty((r, c), dtype=torch.float16, device=dev)
            synth.fill_student_t_(W, seed=seed, stream=st)
            q = hqq.hqq_quantize(W, nb, g)
            res.append((lab, W, q, torch.empty((r, c), dtype=torch.float16, device=dev)))
        return res

    out = {"method": "median of the repetitions; CUDA graph per pass; 256 MiB written "
                     "between repetitions (L2 flush); algorithmic bytes 2 + packed + 4/group "
                     "per weight in both directions"}
    for name in ("matrix-1024", "matrix-4096", "70b-pair"):
        mats = workload(name, rank)
        rows = []
        for (lab, W, q, O), m in zip(prepare(mats), mats):
            ms_q = timed(lambda: hqq.hqq_quantize(W, q.nbits, q.group, packed=q.packed,
                                                  scale=q.scale, zero=q.zero), 20)
            ms_d = timed(lambda: hqq.hqq_dequantize(q, out=O), 20)
            rows.append({"matrix": lab, **record([m], ms_q, ms_d)})
        out[name] = rows
        torch.cuda.empty_cache()
    mats = workload("llama2-7b", rank)
    set7 = prepare(mats)

    def q_all():
        for lab, W, q, O in set7:
            hqq.hqq_quantize(W, q.nbits, q.group, packed=q.packed, scale=q.scale, zero=q.zero)

    def d_all():
        for lab, W, q, O in set7:
            hqq.hqq_dequantize(q, out=O)
    out["llama2-7b"] = {"matrices": len(mats), **record(mats, timed(q_all, 5), timed(d_all, 5))}
    del set7
    torch.cuda.empty_cache()
    return out


def run_meta8(args, views, hqq, dev, hbm_peak, pg):
    """Times, over the whole workload, the 8-bit storage of every matrix's zero
    points (one group per matrix) and scales (groups of 128), and the one-pass
    weight dequantization from that 8-bit form (CUDA events, summed per kernel
    kind; inputs resident)."""
    import torch
    stream = torch.cuda.current_stream()
    metas = []
    for W, q, O in views:
        mg = q.scale.numel()
        zq = hqq.Meta8(torch.empty(mg, dtype=torch.uint8, device=dev),
                       torch.empty(1, dtype=torch.float16, device=dev),
                       torch.empty(1, dtype=torch.float16, device=dev), 0)
        ng = hqq.hqq_meta_groups(mg, 128)
        sq = hqq.Meta8(torch.empty(mg, dtype=torch.uint8, device=dev),
                       torch.empty(ng, dtype=torch.float16, device=dev),
                       torch.empty(ng, dtype=torch.float16, device=dev), 128)
        metas.append((zq, sq))

    # every matrix's zero points (one group) and scales (groups of 128): one
    # batched call per pass
    tensors = [(q.zero.view(-1), 0) for _, q, _ in views] + \
        [(q.scale.view(-1), 128) for _, q, _ in views]
    outs = [zq for zq, _ in metas] + [sq for _, sq in metas]

    def meta_all():
        hqq.hqq_meta_quantize_batch(tensors, outputs=outs)

    def dq_all():
        for k, (W, q, O) in enumerate(views):
            zq, sq = metas[k]
            hqq.hqq_dequantize_meta(q.packed, zq, q.rows, q.cols, q.nbits, q.group, scale_q=sq,
                                    out=O)

    meta_all()
    dq_all()
    torch.cuda.synchronize()
    if not args.no_graph:
        gm, gd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gm):
            meta_all()
        with torch.cuda.graph(gd):
            dq_all()
        run_m, run_d = gm.replay, gd.replay
    else:
        run_m, run_d = meta_all, dq_all
    reps = 3
    for _ in range(3):
        run_m()
        run_d()
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(reps)]
    torch.cuda.synchronize()
    for r in range(reps):
        evs[r][0].record(stream)
        run_m()
        evs[r][1].record(stream)
        run_d()
        evs[r][2].record(stream)
    torch.cuda.synchronize()
    mq_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / reps
    dq_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / reps
    mq_ms, dq_ms = max_over_ranks([mq_ms, dq_ms], pg, dev)
    mq_bytes = dq_bytes = 0
    for W, q, O in views:
        mg = q.scale.numel()
        ng = hqq.hqq_meta_groups(mg, 128)
        mq_bytes += 2 * (2 * mg + mg) + 2 * 2 + 2 * 2 * ng      # read fp16, write codes + s,z
        dq_bytes += (q.packed.numel() + 2 * mg + 2 * 2 + 2 * 2 * ng
                     + 2 * q.rows * q.cols)
    mq_gbs = mq_bytes / (mq_ms / 1e3) / 1e9
    dq_gbs = dq_bytes / (dq_ms / 1e3) / 1e9
    params = sum(q.rows * q.cols for _, q, _ in views)
    return {"what": "zero points 8-bit (one group per matrix), scales 8-bit (groups of 128); "
                    "weights dequantized in one pass from that form",
            "meta_quantize": {"ms_per_pass": mq_ms, "gbs": mq_gbs, "hbm_frac": mq_gbs / hbm_peak,
                              "tensors_per_pass": 2 * len(views),
                              "launches_per_pass": 2 * -(-len(views) // 128),
                              "api": "hqq_meta_quantize_batch (all tensors in one call)"},
            "dequantize_meta": {"ms_per_pass": dq_ms, "gbs": dq_gbs,
                                "hbm_frac": dq_gbs / hbm_peak,
                                "gparam_s": params / (dq_ms / 1e3) / 1e9,
                                "bytes_per_param": dq_bytes / params}}


def run_quantize_half(views, hqq, dev, hbm_peak, qbytes, pg):
    """The quantize pass with the half-precision solver (hqq_quantize_half: the
    page's fp16 solve) over every matrix, replayed as a CUDA graph; with the
    mean accepted iterations and the share of groups solved in fp16."""
    import torch
    stream = torch.cuda.current_stream()

    def half_all():
        for W, q, _ in views:
            hqq.hqq_quantize(W, q.nbits, q.group, packed=q.packed, scale=q.scale, zero=q.zero,
                             precision="fp16")

    half_all()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        half_all()
    for _ in range(2):
        g.replay()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    reps = 3
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(reps):
        g.replay()
    ev[1].record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks([ev[0].elapsed_time(ev[1]) / reps], pg, dev)[0]
    del g
    acc = n_half = n_groups = 0
    for W, q, _ in views[:7]:
        qq = hqq.hqq_quantize_ex(W, q.nbits, q.group, precision="fp16")
        acc += int(qq.iters.long().sum())
        n_half += int(qq.half.long().sum())
        n_groups += qq.iters.numel()
        del qq
    params = sum(q.rows * q.cols for _, q, _ in views)
    gbs = qbytes / (ms / 1e3) / 1e9
    return {"what": "quantize pass with the half-precision solver (each element-wise step "
                    "rounded to fp16, error and z as fp16 group means)",
            "ms_per_pass": ms, "gparam_s": params / (ms / 1e3) / 1e9, "gbs": gbs,
            "hbm_frac": gbs / hbm_peak,
            "mean_accepted_iters_first7": acc / max(n_groups, 1),
            "half_precision_group_frac_first7": n_half / max(n_groups, 1)}


def run_rtn(views, hqq, dev, hbm_peak, qbytes, pg):
    """The memory-side calibration point: the same quantize pass with zero
    solver iterations (min-max round-to-nearest + packing), HBM-bound."""
    import torch
    stream = torch.cuda.current_stream()

    def rtn_all():
        for W, q, _ in views:
            hqq.hqq_quantize(W, q.nbits, q.group, iters=0, packed=q.packed, scale=q.scale,
                             zero=q.zero)

    rtn_all()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        rtn_all()
    for _ in range(3):
        g.replay()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    reps = 3
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(reps):
        g.replay()
    ev[1].record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks([ev[0].elapsed_time(ev[1]) / reps], pg, dev)[0]
    del g
    gbs = qbytes / (ms / 1e3) / 1e9
    return {"what": "quantize pass with iters = 0 (min-max round-to-nearest + packing)",
            "ms_per_pass": ms, "gbs": gbs, "hbm_frac": gbs / hbm_peak}


def run_linear(args, views, hqq, dev, hbm_peak, tensor_peak, pg):
    """Times the weight-only linear layer Y = X W_hat^T (dequantization fused
    into the product kernels) on the workload's quantized matrices:
    decode steps (M = 1 and 16 tokens through every matrix, as CUDA graphs) and
    a prefill of M = 2048 tokens through the first seven matrices (one layer of
    the model-shaped sets).  Beside it, torch's fp16 matmul on the dequantized
    weights of those seven matrices, for context."""
    import torch
    stream = torch.cuda.current_stream()
    maxk = max(q.cols for _, q, _ in views)
    maxn = max(q.rows for _, q, _ in views)

    def timed(fn, reps=3):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(2):
            g.replay()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        torch.cuda.synchronize()
        ev[0].record(stream)
        for _ in range(reps):
            g.replay()
        ev[1].record(stream)
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / reps
        del g
        return ms

    out = {"what": "Y = X W_hat^T, W_hat dequantized inside the product kernels (warp-level MMAs "
                   "fed from registers up to 16 tokens at 3 bits, tcgen05 tiles above; fp16 X and "
                   "Y, fp32 accumulation)"}
    for M in (1, 16):
        X = torch.randn(M * maxk, device=dev).half()
        Y = torch.empty(M * maxn, dtype=torch.float16, device=dev)

        def dec():
            for _, q, _ in views:
                hqq.hqq_linear(X[:M * q.cols].view(M, q.cols), q,
                               out=Y[:M * q.rows].view(M, q.rows))
        ms = max_over_ranks([timed(dec)], pg, dev)[0]
        wbytes = sum(q.packed.numel() + 4 * q.scale.numel() for _, q, _ in views)
        iobytes = sum(2 * M * (q.cols + q.rows) for _, q, _ in views)
        gbs = (wbytes + iobytes) / (ms / 1e3) / 1e9
        flops = sum(2.0 * M * q.rows * q.cols for _, q, _ in views)
        out[f"decode_m{M}"] = {"matrices": len(views), "ms_per_pass": ms,
                               "tokens_per_s": M / (ms / 1e3),
                               "gbs": gbs, "hbm_frac": gbs / hbm_peak,
                               "tflops": flops / (ms / 1e3) / 1e12,
                               "bytes_per_pass": wbytes + iobytes}
        del X, Y
    sub = views[:7]
    M = 2048
    X = torch.randn(M * maxk, device=dev).half()
    Y = torch.empty(M * maxn, dtype=torch.float16, device=dev)

    def pre():
        for _, q, _ in sub:
            hqq.hqq_linear(X[:M * q.cols].view(M, q.cols), q, out=Y[:M * q.rows].view(M, q.rows))
    ms = max_over_ranks([timed(pre)], pg, dev)[0]
    flops = sum(2.0 * M * q.rows * q.cols for _, q, _ in sub)
    tf = flops / (ms / 1e3) / 1e12
    Wd = [hqq.hqq_dequantize(q) for _, q, _ in sub]

    def ref():
        for (_, q, _), w in zip(sub, Wd):
            torch.matmul(X[:M * q.cols].view(M, q.cols), w.t(),
                         out=Y[:M * q.rows].view(M, q.rows))
    ms_t = max_over_ranks([timed(ref)], pg, dev)[0]

    def ref1():
        for (_, q, _), w in zip(sub, Wd):
            torch.matmul(X[:q.cols].view(1, q.cols), w.t(), out=Y[:q.rows].view(1, q.rows))
    ms_t1 = max_over_ranks([timed(ref1)], pg, dev)[0]

    def dec1():
        for _, q, _ in sub:
            hqq.hqq_linear(X[:q.cols].view(1, q.cols), q, out=Y[:q.rows].view(1, q.rows))
    ms_1 = max_over_ranks([timed(dec1)], pg, dev)[0]
    out["prefill_m2048"] = {"matrices": len(sub), "ms_per_pass": ms, "tflops": tf,
                            "tensor_frac": tf / tensor_peak,
                            "torch_fp16_dequantized_ms": ms_t,
                            "torch_fp16_tflops": flops / (ms_t / 1e3) / 1e12}
    out["decode_m1_first7"] = {"ms_per_pass": ms_1, "torch_fp16_dequantized_ms": ms_t1}
    del X, Y, Wd
    return out


def run_lowrank(views, hqq, dev, fma_peak, pg):
    """Times the low-rank residual B A of the quantization error W - W_hat
    (rank 16 from a 32-column Gaussian sketch, 2 power iterations) on the first
    seven matrices (one layer of the model-shaped sets).  The products with
    Delta W, (2 * iters + 2) * rows * cols * sketch multiply-adds per matrix
    (each as three split-tf32 tensor-core products, fp32 accurate), are
    reported over the whole call's time against the fp32 FMA lane peak."""
    import torch
    sub = views[:7]
    rank, sketch, iters = 16, 32, 2
    wsb = max(hqq._lib.hqq_lowrank_workspace_bytes(q.rows, q.cols, sketch) for _, q, _ in sub)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(20)
    oms = [torch.randn(q.cols, sketch, generator=gen, device=dev) for _, q, _ in sub]

    def one():
        for (W, q, _), om in zip(sub, oms):
            hqq.hqq_lowrank(W, q, rank, om, power_iters=iters, workspace=ws)
    one()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    reps = 3
    ev[0].record()
    for _ in range(reps):
        one()
    ev[1].record()
    torch.cuda.synchronize()
    ms = max_over_ranks([ev[0].elapsed_time(ev[1]) / reps], pg, dev)[0]
    fmas = sum((2 * iters + 2) * q.rows * q.cols * sketch for _, q, _ in sub)
    return {"what": "rank-16 residual of W - W_hat by randomized subspace iteration (32-column "
                    "sketch, 2 power iterations), Delta W formed in fp32 inside the products "
                    "(split-tf32 tensor-core MMAs); rate over the whole call",
            "matrices": len(sub), "ms_per_pass": ms,
            "products_tfma_s": fmas / (ms / 1e3) / 1e12,
            "fma_frac": fmas / (ms / 1e3) / 1e12 / fma_peak,
            "fma_peak_t": fma_peak}


def run_stream_pass(mats, hqq, dev, views):
    """Generate + quantize layer by layer through one reused weight buffer
    (outputs stay resident); CUDA-event wall time of the whole pass."""
    import torch
    import synth
    maxn = max(r * c for _, (r, c), *_ in mats)
    buf = torch.empty(maxn, dtype=torch.float16, device=dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record()
    for k, (lab, (r, c), nb, g, seed, stream) in enumerate(mats):
        W = buf[:r * c].view(r, c)
        synth.fill_student_t_(W, seed=seed, stream=stream)
        q = views[k][1]
        hqq.hqq_quantize(W, nb, g, packed=q.packed, scale=q.scale, zero=q.zero)
    t1.record()
    torch.cuda.synchronize()
    s = t0.elapsed_time(t1) / 1e3
    params = sum(r * c for _, (r, c), *_ in mats)
    return {"what": "per layer: generate fp16 weights on the device, then quantize",
            "wall_s": s, "gparam_s": params / s / 1e9}


def run_e2e(args, mats, views, hqq, dev, pg, ws):
    """Same metric, through the API with pinned host buffers: every step copies
    each matrix's fp16 weights host->device, quantizes + dequantizes it, and
    copies the packed codes, scale and zero back.  Host data: one pinned buffer
    per matrix kind (the first layer's values), reused by every layer."""
    import torch
    kinds = {}
    for k, (lab, shape, nb, g, seed, stream) in enumerate(mats):
        kind = lab.split(".")[-1]
        if kind not in kinds:
            kinds[kind] = views[k][0].cpu().pin_memory()
    host_out = {}
    for k, (lab, (r, c), nb, g, *_ ) in enumerate(mats):
        kind = lab.split(".")[-1]
        if kind not in host_out:
            q = views[k][1]
            host_out[kind] = (torch.empty(q.packed.numel(), dtype=torch.uint8, pin_memory=True),
                              torch.empty(q.scale.shape, dtype=torch.float16, pin_memory=True),
                              torch.empty(q.zero.shape, dtype=torch.float16, pin_memory=True))
    maxn = max(r * c for _, (r, c), *_ in mats)
    dW = [torch.empty(maxn, dtype=torch.float16, device=dev) for _ in range(2)]
    s_copy = torch.cuda.Stream(dev)
    s_comp = torch.cuda.current_stream(dev)
    s_back = torch.cuda.Stream(dev)
    h2d = d2h = 0

    def one_step():
        nonlocal h2d, d2h
        h2d = d2h = 0
        ready = [torch.cuda.Event() for _ in range(2)]
        free = [torch.cuda.Event() for _ in range(2)]
        done = []
        for k, (lab, (r, c), nb, g, *_ ) in enumerate(mats):
            kind = lab.split(".")[-1]
            b = k % 2
            with torch.cuda.stream(s_copy):
                if k >= 2:
                    s_copy.wait_event(free[b])
                dst = dW[b][:r * c].view(r, c)
                dst.copy_(kinds[kind], non_blocking=True)
                ready[b].record(s_copy)
            h2d += 2 * r * c
            s_comp.wait_event(ready[b])
            _, q, O = views[k]
            hqq.hqq_quantize(dst, nb, g, packed=q.packed, scale=q.scale, zero=q.zero)
            free[b].record(s_comp)
            hqq.hqq_dequantize(q, out=O)
            ev = torch.cuda.Event()
            ev.record(s_comp)
            with torch.cuda.stream(s_back):
                s_back.wait_event(ev)
                hp, hs, hz = host_out[kind]
                hp.copy_(q.packed, non_blocking=True)
                hs.copy_(q.scale, non_blocking=True)
                hz.copy_(q.zero, non_blocking=True)
            d2h += q.packed.numel() + 2 * q.scale.numel() + 2 * q.zero.numel()
        s_comp.wait_stream(s_back)
        s_comp.wait_stream(s_copy)

    steps = max(1, min(args.steps, args.e2e_steps))
    one_step()
    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_comp)
    for _ in range(steps):
        one_step()
    t1.record(s_comp)
    torch.cuda.synchronize()
    ms = max_over_ranks([t0.elapsed_time(t1)], pg, dev)[0]
    params = sum(r * c for _, (r, c), *_ in mats)
    return {"value": ws * params * steps / (ms / 1e3) / 1e9, "unit": "Gparam/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "warmup": 1, "ms_per_step": ms / steps}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama2-70b",
                    choices=["llama2-70b", "llama2-7b", "matrix-4096", "matrix-1024", "70b-pair",
                             "gate-70b"])
    ap.add_argument("--layers", type=int, default=None,
                    help="first N layers only of a model-shaped set (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass")
    ap.add_argument("--no-stream", action="store_true", help="skip the streamed generate+quantize pass")
    ap.add_argument("--no-meta", action="store_true", help="skip the 8-bit meta-data timing")
    ap.add_argument("--no-linear", action="store_true", help="skip the linear-layer timing")
    ap.add_argument("--no-lowrank", action="store_true", help="skip the low-rank residual timing")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-matrix timings of the other workloads")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every library call from Python each pass instead of replaying "
                         "CUDA graphs of the passes")
    ap.add_argument("--impl", default="libhqq", choices=["libhqq", "reference"])
    ap.add_argument("--cpu-s", type=float, default=10.0, help="oracle CPU-baseline budget (s)")
    ap.add_argument("--ref-step-s", type=float, default=4.0, help="reference arm seconds per step")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl != "reference":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
