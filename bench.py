#!/usr/bin/env python
"""Benchmark: one-layer Thanos prune on the LLaMA-7B-shaped q_proj workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

A step is the whole hot path on one layer: H = 2XX^T from the layer's activations,
damping + factorisation, and the block sweep (scores, exact global-budget masks,
joint row solves, trailing updates), through the library's C ABI
(pwp_prune_layer_x).  The workload is W 4096x4096 bf16, X 16384x4096 bf16 tokens
(8 x 2048) with 0.5% outlier features x50, 50% unstructured sparsity, B = 128.

Under torchrun every rank prunes its own copy of the layer (independent layers of a
model; no data-path collective), so the job's throughput is the sum over ranks
("scaling": "weak").  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "layer prune time (ms) & weights/sec, 4096×4096 @50%; % of TC/HBM roofline"
UNIT = "weights/s"
WORKLOAD = "q_proj4096x4096"
K_HESSIAN, K_FACTOR, K_STREAM, K_SELECT, K_SOLVE, K_ROWPRUNE, K_COLNORM = 0, 1, 2, 3, 4, 5, 6
CLASS_NAMES = {K_HESSIAN: "hessian_xxt", K_FACTOR: "factor", K_STREAM: "stream_update_score",
               K_SELECT: "select", K_SOLVE: "row_solve", K_ROWPRUNE: "row_prune", K_COLNORM: "col_norm"}
CLASS_SOURCES = {K_HESSIAN: ["hessian_tc.cu", "hessian_simt.cu"], K_FACTOR: ["factor.cu"],
                 K_STREAM: ["stream_tc.cu", "prune.cu"], K_SELECT: ["select.cu"], K_SOLVE: ["solve.cu"],
                 K_ROWPRUNE: ["rowprune.cu"], K_COLNORM: ["rowprune.cu"]}
SECOND_ORDER = ("thanos", "sparsegpt")
# The only prune times the source pages give: whole models on other hardware, context only.
PAGES_CONTEXT = {
    "sparsegpt": "about 4 h to prune a 175B-parameter model to 50% unstructured on one A100 (whole model)",
    "wanda": "under 10 min for a 70B-parameter model on one GPU (whole model, no reconstruction)",
    "thanos": "no prune time reported",
}


def _load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured",
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0)}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback", "sm_max_mhz": 1965.0}


def _source_hash(names):
    h = hashlib.sha256()
    for n in names:
        p = os.path.join(ROOT, "post_weight_pruning_b200", "csrc", n)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def _traffic_record(cls):
    """Per-launch DRAM bytes of a kernel class from the committed ncu summary, or None if
    the kernel's source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    want = _source_hash(CLASS_SOURCES[cls])
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == CLASS_NAMES[cls] and f[1] == want \
                and f[2] == WORKLOAD:
            return float(f[3])
    return None


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------ algorithmic work

def algorithmic_work(cls, wl, per_launch_ms, mask=None, method="thanos"):
    """(total algorithmic units over the recorded launches, unit, bound)."""
    c, b, n, B = wl.c, wl.b, wl.n, wl.block
    nblk = (b + B - 1) // B
    if cls == K_ROWPRUNE:
        # read W (bf16), write W-hat (fp32) and the mask, read the column norms (Wanda)
        per = c * b * (2.0 + 4.0 + 1.0) + (4.0 * b if method == "wanda" else 0.0)
        return per * len(per_launch_ms), "byte", "hbm"
    if cls == K_COLNORM:
        return 2.0 * n * b * len(per_launch_ms), "byte", "hbm"   # read X (bf16) once
    if cls == K_HESSIAN:
        return float(b) * b * n * len(per_launch_ms), "flop", "tensor"
    if cls == K_STREAM:
        # per block t: read + write the fp32 active region, read B rows of U over it
        total = 0.0
        for t in range(nblk):
            j = t * B
            total += 8.0 * c * (b - j) + (4.0 * B * (b - j) if t > 0 else 0.0)
        steps = max(1, len(per_launch_ms) // nblk)
        return total * steps, "byte", "hbm"
    if cls == K_SELECT:
        total = sum(4.0 * c * (b - t * B) for t in range(nblk))
        steps = max(1, len(per_launch_ms) // nblk)
        return total * steps, "byte", "hbm"
    if cls == K_SOLVE:
        flops = solve_flops(wl, mask)
        steps = max(1, len(per_launch_ms) // nblk)
        return flops * steps, "flop", "alu"
    if cls == K_FACTOR:
        return 2.0 * b ** 3 / 3.0 * len(per_launch_ms), "flop", "alu"
    raise ValueError(cls)


def solve_flops(wl, mask):
    """Per-row solve arithmetic of one layer: sum over rows and blocks of s^3/3 + 2 s^2 (the
    Cholesky of the s x s system and its two triangular solves), s = the row's removals in
    the block."""
    c, b, B = wl.c, wl.b, wl.block
    nblk = (b + B - 1) // B
    pad = nblk * B - b
    m = np.pad(np.asarray(mask, dtype=np.uint8), ((0, 0), (0, pad))) if pad else np.asarray(mask, dtype=np.uint8)
    s = m.reshape(c, nblk, B).sum(axis=2).astype(np.float64)
    return float(np.sum(s ** 3 / 3.0 + 2.0 * s ** 2))


def block_phase_bytes(wl):
    """Algorithmic HBM bytes of the block prune phase: the fp32 active region read and
    written once per block, the block's rows of the inverse over it, and W (bf16) in plus
    W-hat (fp32) and the mask out."""
    c, b, B = wl.c, wl.b, wl.block
    act = sum(b - j for j in range(0, b, B))
    return 8.0 * c * act + 4.0 * B * sum(b - j for j in range(B, b, B)) + 7.0 * c * b


def phase_rooflines(wl, phase_ms, mask, peaks):
    """Roofline fraction of each phase from its CUDA-event time and its algorithmic work."""
    c, b, n, B = wl.c, wl.b, wl.n, wl.block
    mhz = peaks["sm_max_mhz"]
    alu = fp32_alu_peak_tflops(mhz)
    tf32 = peaks["bf16_tflops"] * 1.1 / 2.25          # nominal tf32 : bf16 dense ratio
    out = {}

    def put(name, ms, work, unit, bound, peak, note):
        if ms is None or ms <= 0:
            return
        per_s = work / (ms / 1e3)
        ach = per_s / (1e9 if unit == "GB/s" else 1e12)
        out[name] = {"ms": ms, "bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
                     "work": note}
    h = phase_ms.get("hessian_xxt")
    put("hessian_xxt", h, float(b) * b * n, "TFLOP/s", "tensor", peaks["bf16_tflops"],
        "b^2 n flops (symmetric half of 2 b^2 n), bf16 operands")
    put("factor", phase_ms.get("factor"), 2.0 * b ** 3 / 3.0, "TFLOP/s", "alu", alu, "2 b^3 / 3 flops")
    st = phase_ms.get("stream_update_score")
    upd_flops = sum(2.0 * c * min(B, b - j) * (b - j) for j in range(0, b, B))
    stream_bytes = sum(8.0 * c * (b - j) + (4.0 * B * (b - j) if j > 0 else 0.0) for j in range(0, b, B))
    put("trailing_update_tensor", st, upd_flops, "TFLOP/s", "tensor", tf32,
        "2 c B (b - j) flops per block (3xTF32 on the tensor cores; peak = measured bf16 x 1.1/2.25)")
    put("stream_update_score", st, stream_bytes, "GB/s", "hbm", peaks["hbm_gbs"],
        "8 c (b - j) + 4 B (b - j) bytes per block")
    put("row_solve", phase_ms.get("row_solve"), solve_flops(wl, mask), "TFLOP/s", "alu", alu,
        "sum of s^3/3 + 2 s^2 over rows and blocks")
    blk = sum(phase_ms.get(k, 0.0) for k in ("stream_update_score", "select", "row_solve"))
    put("block_phase", blk, block_phase_bytes(wl), "GB/s", "hbm", peaks["hbm_gbs"],
        "8 c sum(b - j) + 4 B sum(b - j) + 7 c b bytes; time = update + select + solves")
    return out


def job_throughput(local_ms, world, weights_per_step, steps, device=None):
    """Whole-job throughput (weights/s) from this rank's device time: every rank prunes
    its own layer, so the job processes world x weights_per_step x steps weights in the
    time of the slowest rank (max over ranks).  Returns (value, max_ms)."""
    import torch
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    return world * weights_per_step * steps / (max_ms / 1e3), max_ms


def fp32_alu_peak_tflops(sm_mhz):
    # 148 SMs x 128 fp32 lanes x 2 flop per FMA
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


# ------------------------------------------------------------------------------ CPU oracle

def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return int(max([i.get("num_threads", 1) for i in threadpool_info()] or [1]))
    except Exception:
        return int(os.cpu_count() or 1)


def cpu_oracle_full(wl, W_store, X_store, method="thanos"):
    """The fp64 oracle on the whole benchmarked layer, timed once: the same problem the GPU
    solves (the global budget couples every row, so no row subset is the same problem)."""
    import oracle
    import synth
    W64 = synth.to_f64(W_store, wl.dtype)
    t0 = time.perf_counter()
    X64 = synth.to_f64(X_store, wl.dtype)
    s32 = float(np.float32(wl.sparsity))
    if method in SECOND_ORDER:
        r = oracle.prune_layer(W64, Xt=X64, sparsity=s32, block=wl.block, damp=wl.damp, method=method,
                               pattern="unstructured")
        what = f"H from all {wl.n} tokens, the factor, all {(wl.b + wl.block - 1) // wl.block} blocks"
    else:
        r = oracle.prune_no_update(W64, Xt=X64, sparsity=s32, method=method)
        what = f"norms from all {wl.n} tokens" if method == "wanda" else "no activations"
    dt = time.perf_counter() - t0
    assert r["pruned"] == r.get("zstar", r.get("target"))
    return {"value": wl.c * wl.b / dt, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
            "sample": (f"fp64 numpy oracle ({method}) on the whole {wl.name} layer ({wl.c}x{wl.b} weights): "
                       f"{what}; one run, {dt:.1f} s")}


def cpu_oracle_row_sample(wl, W_store, X64, rows, method="thanos"):
    """A bounded sample of the same layer for the reference arm: the block sweep of the
    first `rows` rows (their own budget at the layer's sparsity) with the layer's H and
    factor, whose time is counted at rows/c because the whole layer shares them.  Returns
    (counted seconds, description)."""
    import oracle
    import synth
    W64 = synth.to_f64(W_store[:rows], wl.dtype)
    s32 = float(np.float32(wl.sparsity))
    if method not in SECOND_ORDER:
        t0 = time.perf_counter()
        oracle.prune_no_update(W64, Xt=X64, sparsity=s32, method=method)
        dt = time.perf_counter() - t0
        return dt, f"{rows} rows of the {wl.name} layer ({method}, norms from all {wl.n} tokens)"
    t0 = time.perf_counter()
    H = oracle.hessian(X64)
    t1 = time.perf_counter()
    Hd, _ = oracle.damp_hessian(H, wl.damp)
    oracle.inverse_cholesky_upper(Hd)
    t2 = time.perf_counter()
    oracle.prune_layer(W64, H=H, sparsity=s32, block=wl.block, damp=wl.damp, method=method, pattern="unstructured")
    t3 = time.perf_counter()
    fixed = (t1 - t0) + (t2 - t1)            # H and the factor: once per layer
    sweep = (t3 - t2) - (t2 - t1)            # prune_layer repeats the factor: take it out
    counted = fixed * rows / wl.c + max(sweep, 0.0)
    return counted, (f"{rows} of {wl.c} rows of the {wl.name} layer: the {method} sweep of those rows "
                     f"(global budget at s={wl.sparsity} on the rows) plus {rows}/{wl.c} of the layer's H "
                     f"({wl.n} tokens) and factor time")


# ------------------------------------------------------------------------------ reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    wl = synth.workload(WORKLOAD)
    W = synth.make_W(wl)
    X = synth.make_X_tokens(wl)
    X64 = synth.to_f64(X, wl.dtype)
    rows = args.cpu_rows
    for _ in range(args.warmup):
        cpu_oracle_row_sample(wl, W, X64, rows, args.method)
    counted = []
    what = ""
    for _ in range(args.steps):
        dt, what = cpu_oracle_row_sample(wl, W, X64, rows, args.method)
        counted.append(dt)
    tot = sum(counted)
    value = rows * wl.b * args.steps / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(wl, args.method),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
                         "sample": what},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(wl, method="thanos"):
    how = {"thanos": f"Thanos 50% unstructured global budget, B={wl.block}, damp={wl.damp}",
           "sparsegpt": f"SparseGPT 50% unstructured per-block quota, B={wl.block}, damp={wl.damp}",
           "wanda": "Wanda 50% per-row quota, no weight update",
           "magnitude": "magnitude 50% per-row quota, no weight update"}[method]
    return {"workload": (f"{wl.name}: W {wl.c}x{wl.b} bf16 ~N(0,0.02^2), X {wl.n}x{wl.b} bf16 tokens "
                         f"(8x2048), 0.5% outlier features x50, {how}"),
            "method": method,
            "c": wl.c, "b": wl.b, "n_tokens": wl.n, "block": wl.block, "sparsity": wl.sparsity,
            "input_dtype": "bf16", "l2": "flushed between steps (256 MiB write, untimed)",
            "parallelism": "independent layer per rank"}


# ------------------------------------------------------------------------------ GPU arm

def run_mine(args):
    import torch
    import torch.distributed as dist
    import synth
    import post_weight_pruning_b200 as pwp

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    L = pwp.lib()
    L.pwp_kernel_launches.restype = ctypes.c_int64
    L.pwp_profile_enable.argtypes = [ctypes.c_int32, ctypes.c_int32]
    L.pwp_profile_read.argtypes = [ctypes.c_void_p, ctypes.c_int32]

    wl = synth.workload(WORKLOAD)
    W_store = synth.make_W(wl)
    X_store = synth.make_X_tokens(wl)
    Wt = pwp.from_bf16_bits(W_store, dev)
    Xt = pwp.from_bf16_bits(X_store, dev)
    c, b = wl.c, wl.b
    method = args.method
    cfg_kw = dict(method=method, pattern="unstructured", sparsity=wl.sparsity, block=wl.block, damp=wl.damp)
    ws = pwp.make_workspace(pwp.config(**cfg_kw), c, b, dev)
    H = torch.empty((b, b), dtype=torch.float32, device=dev) if method in SECOND_ORDER else None
    W_out = torch.empty((c, b), dtype=torch.float32, device=dev)
    mask = torch.empty((c, b), dtype=torch.uint8, device=dev)
    stats = pwp.new_stats(dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MiB > 126 MB L2
    stream = torch.cuda.current_stream()

    def step():
        pwp.prune_layer(Wt, X=Xt, H=H, W_out=W_out, mask=mask, workspace=ws, stats=stats, check=False,
                        **cfg_kw)

    nblk = (b + wl.block - 1) // wl.block
    launches_per_class = {K_HESSIAN: 1, K_FACTOR: 1, K_STREAM: nblk, K_SELECT: nblk, K_SOLVE: nblk,
                          K_ROWPRUNE: 1, K_COLNORM: 1}
    if method in SECOND_ORDER:
        classes = (K_HESSIAN, K_FACTOR, K_STREAM, K_SELECT, K_SOLVE)
    else:
        classes = (K_COLNORM, K_ROWPRUNE) if method == "wanda" else (K_ROWPRUNE,)

    for i in range(max(args.warmup, 1)):
        flush.fill_(float(i))
        step()
    torch.cuda.synchronize()
    st = pwp.read_stats(stats)
    if st.status != 0 or st.pruned != st.target:
        raise RuntimeError(f"warm-up step failed: status {st.status} pruned {st.pruned} target {st.target}")

    # phase breakdown (untimed pass per kernel class) to pick the dominant kernel
    phase_ms = {}
    for cls in classes:
        L.pwp_profile_enable(cls, launches_per_class[cls])
        flush.fill_(0.0)
        step()
        buf = (ctypes.c_float * launches_per_class[cls])()
        n = L.pwp_profile_read(buf, launches_per_class[cls])
        phase_ms[CLASS_NAMES[cls]] = float(sum(buf[:n]))
    L.pwp_profile_enable(-1, 0)
    dom = max(classes, key=lambda k: phase_ms[CLASS_NAMES[k]])

    # timed region
    cap = launches_per_class[dom] * args.steps
    L.pwp_profile_enable(dom, cap)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = L.pwp_kernel_launches()
    for i in range(args.steps):
        flush.fill_(float(i + 1))
        ev0[i].record(stream)
        step()
        ev1[i].record(stream)
    torch.cuda.synchronize()
    launches = L.pwp_kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [ev0[i].elapsed_time(ev1[i]) for i in range(args.steps)]
    total_ms = float(sum(step_ms))
    buf = (ctypes.c_float * cap)()
    nrec = L.pwp_profile_read(buf, cap)
    L.pwp_profile_enable(-1, 0)
    dom_ms = [float(x) for x in buf[:nrec]]
    st = pwp.read_stats(stats)
    if st.status != 0 or st.pruned != st.target:
        raise RuntimeError(f"timed step failed: status {st.status}")
    mask_np = mask.cpu().numpy() if dom == K_SOLVE else None

    value, max_ms = job_throughput(total_ms, world, c * b, args.steps, dev)

    # end to end through the public API from pinned host buffers
    W_host = torch.from_numpy(W_store.view(np.int16)).view(torch.bfloat16).pin_memory()
    X_host = torch.from_numpy(X_store.view(np.int16)).view(torch.bfloat16).pin_memory()
    # the layers of a model one after another through the multi-layer host entry point: each
    # step's inputs go host -> device and its results device -> host inside the timed region,
    # overlapping the neighbouring steps' work
    e2e_steps = max(2, min(args.steps, 10))   # as many layers as the timed device steps, at most 10
    out_Ws = [torch.empty((c, b), dtype=torch.float32).pin_memory() for _ in range(e2e_steps)]
    out_ms = [torch.empty((c, b), dtype=torch.uint8).pin_memory() for _ in range(e2e_steps)]
    pwp.prune_layers_host([W_host] * 2, [X_host] * 2, out_Ws=out_Ws[:2], out_masks=out_ms[:2], device=dev,
                          **cfg_kw)
    torch.cuda.synchronize()
    flush.fill_(0.0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    _, _, e2e_stats = pwp.prune_layers_host([W_host] * e2e_steps, [X_host] * e2e_steps, out_Ws=out_Ws,
                                            out_masks=out_ms, device=dev, **cfg_kw)
    e1.record(stream)
    torch.cuda.synchronize()
    for rec in pwp.read_stats_list(e2e_stats):
        if rec.status != 0 or rec.pruned != rec.target:
            raise RuntimeError(f"end-to-end step failed: status {rec.status}")
    e2e_ms = float(e0.elapsed_time(e1))
    e2e_value, _ = job_throughput(e2e_ms, world, c * b, e2e_steps, dev)

    if rank == 0:
        peaks = _load_peaks()
        work, unit, bound = algorithmic_work(dom, wl, dom_ms, mask_np, method)
        dur_s = sum(dom_ms) / 1e3
        if unit == "byte":
            achieved = work / dur_s / 1e9
            peak, punit, psrc = peaks["hbm_gbs"], "GB/s", peaks["source"] + " hbm_gbs"
        elif bound == "tensor":
            achieved = work / dur_s / 1e12
            peak, punit, psrc = peaks["bf16_tflops"], "TFLOP/s", peaks["source"] + " bf16_tflops (burst)"
        else:
            achieved = work / dur_s / 1e12
            mhz = peaks["sm_max_mhz"]
            peak, punit, psrc = fp32_alu_peak_tflops(mhz), "TFLOP/s", f"fp32 FMA issue rate at {mhz:.0f} MHz"
        traffic = _traffic_record(dom)
        roof = {"kernel": CLASS_NAMES[dom], "bound": bound, "achieved": achieved, "peak": peak, "unit": punit,
                "frac": achieved / peak, "traffic": traffic, "peak_source": psrc,
                "launches_timed": len(dom_ms)}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": _config(wl, method),
            "roofline": roof,
            "phases_ms": phase_ms,
            "gpu_launches": int(launches),
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": int(W_host.numel() * 2 + X_host.numel() * 2),
                    "d2h_bytes_per_step": int(out_Ws[0].numel() * 4 + out_ms[0].numel())},
            "clocks": clocks,
            "context_from_pages": PAGES_CONTEXT,
        }
        if method in SECOND_ORDER:
            line["select_stats"] = {"blocks": nblk, "reread_blocks": int(st.reread_blocks),
                                    "tie_blocks": int(st.tie_blocks)}
        if method in SECOND_ORDER:
            if mask_np is None:
                mask_np = mask.cpu().numpy()
            line["phases"] = phase_rooflines(wl, phase_ms, mask_np, peaks)
        # the other workloads and the CPU baseline are reported beside the headline; a
        # failure in either is recorded in the line instead of losing it
        if world == 1 and not args.no_extra_workloads and method == "thanos":
            try:
                line["workloads"] = time_other_workloads(dev, args)
            except Exception as exc:   # noqa: BLE001
                line["workloads"] = {"error": f"{type(exc).__name__}: {exc}"}
        if world == 1 and not args.no_cpu_baseline:
            try:
                line["cpu_baseline"] = cpu_oracle_full(wl, W_store, X_store, method)
            except Exception as exc:   # noqa: BLE001
                line["cpu_baseline"] = {"error": f"{type(exc).__name__}: {exc}"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _time_calls(fn, steps, warmup=1):
    """Device time (ms) of fn() per call on the current stream, after warm-up; the L2 is
    flushed before every call (the inputs of these workloads exceed it anyway)."""
    import torch
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ms = []
    for i in range(steps):
        flush.fill_(float(i))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    del flush
    return ms


def _device_block_inputs(dev, seed=0):
    """The decoder block's activations drawn on the device (torch generator, seed 0) with the
    host generator's distributions: Gaussian with 0.5% of features x50 (attention, o and MLP
    inputs), Laplace(0, 1/sqrt 2) with 30% of entries x1e-2 (down_proj input); 128 x 2048
    tokens each.  Only the timing uses these; the parity tests draw on the host."""
    import torch
    import synth
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    acts = {}
    for inp, (b, dist, frac, scale, _) in synth.BLOCK_INPUTS.items():
        n = synth.BLOCK_TOKENS
        X = torch.empty((n, b), dtype=torch.bfloat16, device=dev)
        cols = None
        if frac > 0:
            k = int(round(frac * b))
            cols = torch.randperm(b, generator=g, device=dev)[:k]
        for r0 in range(0, n, 16384):
            r1 = min(n, r0 + 16384)
            if dist == "gaussian":
                x = torch.randn((r1 - r0, b), generator=g, device=dev)
            else:
                # u uniform on the open interval (-1/2, 1/2): rand can return 0, and
                # u = -1/2 would give log1p(-1) = -inf
                u = torch.rand((r1 - r0, b), generator=g, device=dev).clamp_(1e-7, 1.0 - 1e-7) - 0.5
                x = -torch.sign(u) * torch.log1p(-2.0 * u.abs()) / math.sqrt(2.0)
                near = torch.rand((r1 - r0, b), generator=g, device=dev) < 0.3
                x = torch.where(near, x * 1e-2, x)
            if cols is not None:
                x[:, cols] *= scale
            X[r0:r1] = x.to(torch.bfloat16)
        acts[inp] = X
    weights = {}
    for l, (name, inp, c) in enumerate(synth.BLOCK_LAYERS):
        b = synth.BLOCK_INPUTS[inp][0]
        weights[name] = (torch.randn((c, b), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    feeds = {name: inp for name, inp, _ in synth.BLOCK_LAYERS}
    return weights, acts, feeds


def time_other_workloads(dev, args):
    """Prune time of the other benchmark workloads on this GPU (CUDA events, L2 flushed):
    the 11008x4096 layer at 2:4 and the 4096x11008 layer at 4:8 (32768 tokens; H build +
    factor + sweep, with each phase's time) and the seven-layer decoder block (128 x 2048
    tokens; four H builds and seven prunes through prune_block)."""
    import torch
    import synth
    import post_weight_pruning_b200 as pwp
    L = pwp.lib()
    out = {}
    threads = max(1, min(32, os.cpu_count() or 1))
    for name in ("up_proj11008x4096_2of4", "down_proj4096x11008_4of8"):
        wl = synth.workload(name)
        W_store, X_store = synth.make_W(wl), synth.make_X_tokens(wl, threads=threads)
        Wt, Xt = pwp.from_bf16_bits(W_store, dev), pwp.from_bf16_bits(X_store, dev)
        del X_store
        kw = dict(method="thanos", pattern="nm", nm=wl.nm, sparsity=wl.sparsity, block=wl.block, damp=wl.damp)
        ws = pwp.make_workspace(pwp.config(**kw), wl.c, wl.b, dev)
        H = torch.empty((wl.b, wl.b), dtype=torch.float32, device=dev)
        W_out = torch.empty((wl.c, wl.b), dtype=torch.float32, device=dev)
        mask = torch.empty((wl.c, wl.b), dtype=torch.uint8, device=dev)
        stats = pwp.new_stats(dev)

        def call():
            pwp.prune_layer(Wt, X=Xt, H=H, W_out=W_out, mask=mask, workspace=ws, stats=stats, check=False, **kw)
        ms = _time_calls(call, steps=5)
        nblk = (wl.b + wl.block - 1) // wl.block
        per_class = {K_HESSIAN: 1, K_FACTOR: 1, K_STREAM: nblk, K_SELECT: nblk, K_SOLVE: nblk}
        phases = {}
        for cls, cnt in per_class.items():
            L.pwp_profile_enable(cls, cnt)
            call()
            buf = (ctypes.c_float * cnt)()
            n = L.pwp_profile_read(buf, cnt)
            phases[CLASS_NAMES[cls]] = float(sum(buf[:n]))
        L.pwp_profile_enable(-1, 0)
        st = pwp.read_stats(stats)
        if st.status != 0 or st.pruned != st.target:
            raise RuntimeError(f"{name}: status {st.status}")
        t = statistics.median(ms)
        out[name] = {"ms": t, "weights_per_s": wl.c * wl.b / (t / 1e3), "steps": len(ms),
                     "ms_calls": [round(x, 3) for x in ms],
                     "config": f"W {wl.c}x{wl.b} bf16, X {wl.n}x{wl.b} bf16 ({wl.x_dist}), Thanos "
                               f"{wl.nm[0]}:{wl.nm[1]}, B={wl.block}, damp={wl.damp}",
                     "phases_ms": phases}
        del Wt, Xt, ws, H, W_out, mask
        torch.cuda.empty_cache()

    weights, acts, feeds = _device_block_inputs(dev)
    res = {}

    def block():
        res.update(pwp.prune_block(weights, acts, feeds, method="thanos", pattern="unstructured", sparsity=0.5,
                                   block=128, damp=0.01, check=False))
    ms = _time_calls(block, steps=3)
    for layer, (_, _, st_t) in res.items():
        st = pwp.read_stats(st_t)
        if st.status != 0 or st.pruned != st.target:
            raise RuntimeError(f"decoder block {layer}: status {st.status}")
    total = sum(int(w.numel()) for w in weights.values())
    t = statistics.median(ms)
    out["decoder_block"] = {"ms": t, "weights_per_s": total / (t / 1e3), "steps": len(ms),
                            "ms_calls": [round(x, 3) for x in ms],
                            "config": ("q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008 bf16; 128x2048 "
                                       "tokens per input drawn on the device; Thanos 50% unstructured global budget "
                                       "per layer, B=128; one H per input (4 builds), 7 prunes")}
    del weights, acts, res
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=256,
                    help="rows of the reference arm's per-step sample")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="skip the timing of the 2:4, 4:8 and decoder-block workloads")
    ap.add_argument("--method", default="thanos", choices=["thanos", "sparsegpt", "wanda", "magnitude"],
                    help="pruning method timed on the q_proj workload (default: thanos, the headline)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_mine(args)


if __name__ == "__main__":
    sys.exit(main())
