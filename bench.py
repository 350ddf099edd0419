#!/usr/bin/env python
"""Benchmark of the WISE attention hot path on B200 (prints one JSON line on rank 0).

A bench "step" is one full WISE trajectory of one attention layer over T = 32
recurrent steps (Wan & Chen, "Attention Routing Stabilizes Early: Working-Set
Inference for Recurrent-Depth Language Models", section 7.4 and appendix B,
"Systems evaluation"): 12 dense exploration steps (the 4 window steps also
compute block mass and select/union), the one-time schedule build, and 20
block-sparse late steps, back to back on one stream with inputs resident in
HBM.  `value` is effective TFLOP/s over the trajectory, counting 4*d FLOPs per
admissible (query, key) pair of the dense steps and of the selected blocks of
the late steps (the mass pass recompute and masked work are not counted).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4k]
       [--block 32|64|128] [--impl wise|reference].  --block selects on
coarser blocks (appendix C.6's block-size study) and runs them as 32 x 32
subtiles.  For N > 1 launch one process per GPU with torch.distributed.run;
every rank runs its own independent trajectory (weak scaling, no collective
on the data path).
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "late-step sparse attn µs/step & eff. TFLOP/s at 4K; 32-step trajectory µs"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SRC = os.path.join(ROOT, "recurrent_depth_lm_b200", "csrc", "attn.cu")


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))


def reduce_max(x: float, device) -> float:
    """Max of a scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, device) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------ FLOP accounting

def dense_flops(cfg) -> float:
    """4*d per admissible (i, j <= i) pair, all heads."""
    n = cfg.seqlen
    return 4.0 * cfg.head_dim * cfg.bh * n * (n + 1) / 2


def sparse_flops_b16(cfg, union16) -> float:
    """4*d per admissible pair inside the kept 16-token blocks (16*16 off-diagonal,
    16*17/2 diagonal), from the [BH, n/16, W] working-set words on the host."""
    import numpy as np
    n16 = cfg.seqlen // 16
    words = union16.reshape(-1, n16, union16.shape[-1]).view(np.uint32)
    bits = np.tril(np.unpackbits(words.view(np.uint8), axis=-1,
                                 bitorder="little")[..., :n16].astype(bool))
    diag = np.trace(bits, axis1=1, axis2=2).sum()
    off = bits.sum() - diag
    return 4.0 * cfg.head_dim * (off * 256 + diag * 136)


def sparse_flops(cfg, row_offsets, col_idx) -> float:
    """4*d per admissible pair inside the scheduled blocks (32*32 off-diagonal, 32*33/2 diagonal)."""
    import numpy as np
    nq = cfg.nq
    ro = np.asarray(row_offsets, np.int64)
    ci = np.asarray(col_idx, np.int64)[: ro[-1]]
    rows = np.repeat(np.arange(len(ro) - 1) % nq, np.diff(ro))
    diag = int((ci == rows).sum())
    pairs = (len(ci) - diag) * 1024 + diag * 528
    return 4.0 * cfg.head_dim * pairs


def tile_waste(cfg, row_offsets, col_idx):
    """(issued, selected) 32x32 block units of a schedule.  A 128-row tile runs every key
    block that any of its 4 query blocks keeps, for all 4 of them, so it issues
    4 * |union of the 4 rows| block units against the rows' own counts."""
    import numpy as np
    nq = cfg.nq
    ro = np.asarray(row_offsets, np.int64)
    ci = np.asarray(col_idx, np.int64)[: ro[-1]]
    nrows = len(ro) - 1
    rows = np.repeat(np.arange(nrows), np.diff(ro))
    tiles = (rows // nq) * ((nq + 3) // 4) + (rows % nq) // 4
    pairs = np.unique(tiles * nq + ci)          # distinct (tile, key block)
    return 4 * len(pairs), len(ci)


# ------------------------------------------------------------------ measurement helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    with open(KERNEL_SRC, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha1") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.tmp.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ the WISE arm

def make_inputs(cfg, rank: int, device, workers: int):
    """All T steps of Q, K, V on the device: three [T, B, H, n, d] bf16 tensors."""
    import numpy as np
    import torch
    from wise_inputs.generator import StepPool
    T = cfg.steps
    shp = (T, cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim)
    q = torch.empty(shp, dtype=torch.bfloat16, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    host = None
    with StepPool(cfg, workers=workers, rank=rank) as pool:
        for t, qb, kb, vb in pool:
            for dst, src in ((q, qb), (k, kb), (v, vb)):
                dst[t - 1].copy_(torch.from_numpy(np.ascontiguousarray(src).view(np.int16))
                                 .view(torch.bfloat16))
    return q, k, v, host


class TrajectoryRunner:
    """Runs whole trajectories through the C ABI with per-call CUDA events."""

    def __init__(self, cfg, device, block: int = 32):
        import torch
        from recurrent_depth_lm_b200 import ops
        from recurrent_depth_lm_b200.trajectory import WiseTrajectory
        self.cfg, self.ops, self.block = cfg, ops, block
        self.traj = WiseTrajectory(cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim, t_d=cfg.t_d,
                                   window=cfg.window, eta=cfg.eta, block=block, device=device)
        self.o = torch.empty(cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim,
                             dtype=torch.bfloat16, device=device)
        self.device = device

    def launches_per_trajectory(self) -> int:
        cfg = self.cfg
        nwin = cfg.window[1] - cfg.window[0] + 1
        # dense steps: 1 kernel; window steps: attention + mass + select; schedule: 3
        # (block 16: 16-token mass + select; schedule fold + 3 + sub-masks = 5)
        sched = 5 if self.block == 16 else 3
        return (cfg.t_d - nwin) + 3 * nwin + sched + (cfg.steps - cfg.t_d)

    def run(self, q, k, v, events=None):
        """One trajectory.  If `events` is a dict, append (start, end) event pairs per call kind."""
        import torch
        cfg, ops, tr = self.cfg, self.ops, self.traj
        tr.reset()

        def ev():
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            return e

        if self.block == 16:   # the trajectory's own step calls, one event pair per step
            for t in range(1, cfg.steps + 1):
                a = ev() if events is not None else None
                tr.step(t, q[t - 1], k[t - 1], v[t - 1], o=self.o)
                if events is not None:
                    kind = ("sparse" if t > cfg.t_d else
                            "window" if tr.in_window(t) else "dense")
                    events.setdefault(kind, []).append((a, ev()))
            return self.o
        for t in range(1, cfg.steps + 1):
            qt, kt, vt = q[t - 1], k[t - 1], v[t - 1]
            if t <= cfg.t_d:
                if tr.in_window(t) and self.block == 32:
                    a = ev() if events is not None else None
                    ops.window_step(qt, kt, vt, tr.union, cfg.eta, o=self.o, lse=tr.lse,
                                    mass=tr.mass, workspace=tr.mass_ws)
                    if events is not None:
                        events.setdefault("window", []).append((a, ev()))
                elif tr.in_window(t):
                    a = ev() if events is not None else None
                    ops.full_attn_mass(qt, kt, vt, o=self.o, lse=tr.lse, mass=tr.mass,
                                       workspace=tr.mass_ws)
                    ops.select_union(tr.mass, tr.union, cfg.eta, head_dim=cfg.head_dim,
                                     block=self.block)
                    if events is not None:
                        events.setdefault("window", []).append((a, ev()))
                else:
                    a = ev() if events is not None else None
                    ops.full_attn_mass(qt, kt, vt, o=self.o)
                    if events is not None:
                        events.setdefault("dense", []).append((a, ev()))
                if t == cfg.t_d:
                    a = ev() if events is not None else None
                    tr.build_schedule()
                    if events is not None:
                        events.setdefault("schedule", []).append((a, ev()))
            else:
                a = ev() if events is not None else None
                ops.sparse_attn(qt, kt, vt, tr.row_offsets, tr.col_idx, tr.col_idx.numel(),
                                o=self.o)
                if events is not None:
                    events.setdefault("sparse", []).append((a, ev()))
        return self.o


def all_blocks_schedule(cfg, device):
    """The CSR schedule of every causal block (the matched comparison's support)."""
    import torch
    from recurrent_depth_lm_b200 import ops
    full = torch.full((cfg.batch, cfg.heads, cfg.nq, ops.words_per_row(cfg.nq)), -1,
                      dtype=torch.int32, device=device)
    ro, ci, _ = ops.build_schedule(full, head_dim=cfg.head_dim, exact_nnz=False)
    return ro, ci


def late_step_us(cfg, q, k, v, ro, ci, o, reps: int = 1):
    """Median CUDA-event time of the block-sparse kernel over the late steps' inputs."""
    import torch
    from recurrent_depth_lm_b200 import ops
    xs = []
    for _ in range(reps):
        for t in range(cfg.t_d + 1, cfg.steps + 1):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            ops.sparse_attn(q[t - 1], k[t - 1], v[t - 1], ro, ci, ci.numel(), o=o)
            b.record()
            xs.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(x.elapsed_time(y) * 1000.0 for x, y in xs)


def matched_record(cfg, q, k, v, runner, device, f_sparse):
    """The late step on the WISE schedule against the same kernel on every causal block
    (the pages' matched exact-B=32 comparison), with density and tile waste."""
    import numpy as np
    tr = runner.traj
    ro_w, ci_w = tr.row_offsets, tr.col_idx
    ro_a, ci_a = all_blocks_schedule(cfg, device)
    late_us_w = late_step_us(cfg, q, k, v, ro_w, ci_w, runner.o, reps=2)
    late_us_a = late_step_us(cfg, q, k, v, ro_a, ci_a, runner.o, reps=2)
    issued, selected = tile_waste(cfg, ro_w.cpu().numpy(), ci_w.cpu().numpy())
    density = tr.density()
    return {"late_step_us": round(late_us_w, 2),
            "all_blocks_late_step_us": round(late_us_a, 2),
            "speedup": round(late_us_a / late_us_w, 3),
            "inverse_density": round(1.0 / density, 3),
            "density": round(density, 4),
            "issued_over_selected_blocks": round(issued / selected, 4),
            "late_step_tflops": round(f_sparse / (late_us_w * 1e-6) / 1e12, 2)}


def config_record(cfg, q, k, v, device, reps: int, peak: float):
    """One workload measured on its own: per-call medians over `reps` trajectories, the
    matched all-blocks late step and the tile waste."""
    import torch
    runner = TrajectoryRunner(cfg, device)
    for _ in range(2):
        runner.run(q, k, v)
    torch.cuda.synchronize()
    events = {}
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(reps):
        runner.run(q, k, v, events=events)
    t1.record()
    torch.cuda.synchronize()
    traj_us = t0.elapsed_time(t1) * 1000.0 / reps
    med = {kind: statistics.median(a.elapsed_time(b) * 1000.0 for a, b in xs)
           for kind, xs in events.items()}
    ro = runner.traj.row_offsets.cpu().numpy()
    ci = runner.traj.col_idx.cpu().numpy()
    f_dense, f_sparse = dense_flops(cfg), sparse_flops(cfg, ro, ci)
    traj_flops = cfg.t_d * f_dense + (cfg.steps - cfg.t_d) * f_sparse
    late, dense = med.get("sparse"), med.get("dense")
    rec = {"workload": f"{cfg.name}: batch {cfg.batch}, {cfg.heads} heads, head_dim "
                       f"{cfg.head_dim}, n={cfg.seqlen}, eta={cfg.eta}",
           "trajectory_us": round(traj_us, 1),
           "trajectory_tflops": round(traj_flops / (traj_us * 1e-6) / 1e12, 2),
           "late_step_us": round(late, 2),
           "late_step_tflops": round(f_sparse / (late * 1e-6) / 1e12, 2),
           "late_step_frac": round(f_sparse / (late * 1e-6) / 1e12 / peak, 4),
           "dense_step_us": round(dense, 2) if dense else None,
           "dense_step_tflops": round(f_dense / (dense * 1e-6) / 1e12, 2) if dense else None,
           "dense_step_frac": round(f_dense / (dense * 1e-6) / 1e12 / peak, 4) if dense else None,
           "window_step_us": round(med["window"], 2),
           "window_over_dense_us": round(med["window"] - dense, 2) if dense else None,
           "schedule_us": round(med["schedule"], 2),
           "setup_inclusive_late_us": round(((cfg.steps - cfg.t_d) * late + med["schedule"])
                                            / (cfg.steps - cfg.t_d), 2),
           "trajectories_timed": reps,
           "l2": ("inputs fit in L2 (one trajectory is "
                  f"{3 * cfg.steps * cfg.bh * cfg.seqlen * cfg.head_dim * 2 / 1e6:.1f} MB)"
                  if 3 * cfg.steps * cfg.bh * cfg.seqlen * cfg.head_dim * 2 < 126e6
                  else "inputs larger than L2")}
    rec["matched"] = matched_record(cfg, q, k, v, runner, device, f_sparse)
    rec["density"] = rec["matched"]["density"]
    return rec


def run_e2e(cfg, runner, host_q, host_k, host_v, reps: int):
    """Trajectories through the public API from pinned host buffers.

    Every step copies its Q, K, V host->device (prefetched one step ahead on a
    copy stream) and copies its O device->host (on a second copy stream, so the
    two PCIe directions run at once; O is double-buffered); the clock covers
    everything.
    """
    import torch
    ops, tr = runner.ops, runner.traj
    dev = runner.device
    T = cfg.steps
    shp = (cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim)
    bufs = [[torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(3)] for _ in range(2)]
    obufs = [torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    host_o = torch.empty((T,) + shp, dtype=torch.bfloat16).pin_memory()
    copy = torch.cuda.Stream(device=dev)
    back = torch.cuda.Stream(device=dev)
    comp = torch.cuda.current_stream(dev)
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]     # step's O written
    drained = [torch.cuda.Event() for _ in range(2)]  # O buffer copied out

    def h2d(t):
        s = (t - 1) % 2
        with torch.cuda.stream(copy):
            copy.wait_event(free[s])
            for dst, src in zip(bufs[s], (host_q, host_k, host_v)):
                dst.copy_(src[t - 1], non_blocking=True)
            ready[s].record(copy)

    for s in range(2):   # once: afterwards each refers to its buffer's last copy-out
        drained[s].record(comp)

    def one():
        tr.reset()
        for s in range(2):
            free[s].record(comp)
        h2d(1)
        for t in range(1, T + 1):
            s = (t - 1) % 2
            if t < T:
                h2d(t + 1)
            comp.wait_event(ready[s])
            comp.wait_event(drained[s])
            qt, kt, vt = bufs[s]
            tr.step(t, qt, kt, vt, o=obufs[s])
            free[s].record(comp)
            done[s].record(comp)
            with torch.cuda.stream(back):
                back.wait_event(done[s])
                host_o[t - 1].copy_(obufs[s], non_blocking=True)
                drained[s].record(back)

    one()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(reps):
        one()
    torch.cuda.synchronize()
    dt = (time.perf_counter() - t0) / reps
    per = cfg.bh * cfg.seqlen * cfg.head_dim * 2
    return dt, 3 * T * per, T * per


def routing_stats(cfg, q, k, v, device, block: int = 32):
    """Untimed: block density and retained future attention mass (WISE paper appendix B,
    "Evaluation metrics") of the WISE working set and of the selection-only controls,
    each from one trajectory over the same inputs with the late-step mass tracked."""
    from recurrent_depth_lm_b200.trajectory import WiseTrajectory
    out = {}
    supports = ["wise", "static95"] + (["size_matched", "mass_matched"] if block == 32 else [])
    for support in supports:
        tr = WiseTrajectory(cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim, t_d=cfg.t_d,
                            window=cfg.window, eta=cfg.eta, block=block, support=support,
                            track_retained=True, device=device)
        for t in range(1, cfg.steps + 1):
            tr.step(t, q[t - 1], k[t - 1], v[t - 1])
        out[support] = {"density": round(tr.density(), 4),
                        "retained_future_mass": round(tr.retained_future_mass(), 4)}
        del tr
    return out


def cpu_oracle_sample(cfg, n_heads: int = 1, block: int = 32):
    """The CPU oracle, as it stands, on a bounded sample: for each sampled head one
    exploration step (dense attention + block mass + eta-selection -> schedule) and
    one late block-sparse step.  Returns (seconds, useful FLOPs, description)."""
    import numpy as np
    from oracle import wise_oracle as O
    from wise_inputs import bf16_bits_to_f64, iter_steps
    heads = [(0, h) for h in range(n_heads)]
    steps = {}
    for t, q, k, v in iter_steps(cfg, heads=heads, steps=cfg.t_d + 1):
        if t >= cfg.t_d:
            steps[t] = (q, k, v)
    flops = 0.0
    t0 = time.perf_counter()
    for i in range(len(heads)):
        q, k, v = (bf16_bits_to_f64(x[i]) for x in steps[cfg.t_d])
        O.causal_attention(q, k, v, cfg.scale)
        r = O.block_mass(q, k, cfg.scale, block=block)
        sup = O.select(r, cfg.eta)
        if block > 32:
            sup = O.expand_support(sup, block // 32)
        ro, ci = O.csr_schedule(sup)
        q, k, v = (bf16_bits_to_f64(x[i]) for x in steps[cfg.t_d + 1])
        n = cfg.seqlen
        flops += 4.0 * cfg.head_dim * n * (n + 1) / 2
        if block == 16:   # the oracle attends the 16-token support directly
            O.masked_attention(q, k, v, sup, cfg.scale, block=16)
            kept = np.tril(sup)
            diag = int(np.trace(kept))
            flops += 4.0 * cfg.head_dim * ((int(kept.sum()) - diag) * 256 + diag * 136)
        else:
            O.sparse_attention(q, k, v, ro, ci, cfg.scale)
            flops += sparse_flops(cfg.with_(batch=1, heads=1), ro, ci)
    dt = time.perf_counter() - t0
    desc = (f"{len(heads)} head(s) of {cfg.name}: one dense exploration step with block mass and "
            f"eta-selection (B={block}), plus one block-sparse late step, numpy float64")
    return dt, flops, desc


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count() or 1)
    except Exception:
        return os.cpu_count() or 1


def workload(args):
    """The named workload with the one-at-a-time overrides (eta, t_d, window) applied."""
    from wise_inputs import CONFIGS, SUPPLEMENTARY
    if args.config not in CONFIGS and args.config not in SUPPLEMENTARY:
        raise SystemExit(f"unknown workload {args.config!r}: one of "
                         f"{sorted(CONFIGS) + sorted(SUPPLEMENTARY)}")
    cfg = CONFIGS.get(args.config) or SUPPLEMENTARY[args.config]
    kw = {}
    if args.eta is not None:
        kw["eta"] = args.eta
    if args.t_d is not None:
        kw["t_d"] = args.t_d
        kw["window"] = (max(1, args.t_d - 3), args.t_d)
    if args.window is not None:
        kw["window"] = tuple(args.window)
    cfg = cfg.with_(**kw) if kw else cfg
    if not (1 <= cfg.window[0] <= cfg.window[1] <= cfg.t_d < cfg.steps):
        raise SystemExit(f"bad discovery window {cfg.window} for t_d={cfg.t_d}, T={cfg.steps}")
    return cfg


def bench_wise(args):
    import numpy as np
    import torch

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    cfg = workload(args)
    workers = args.workers or max(1, min(16, (os.cpu_count() or 2) // max(1, world)))

    q, k, v, _ = make_inputs(cfg, rank, device, workers)
    runner = TrajectoryRunner(cfg, device, block=args.block)
    ops = runner.ops

    for _ in range(args.warmup):
        runner.run(q, k, v)
    torch.cuda.synchronize()
    assert ops.device_status() == 0, "device status flagged during warm-up"
    ro = runner.traj.row_offsets.cpu().numpy()
    ci = runner.traj.col_idx.cpu().numpy()
    nnz = int(ro[-1])
    f_dense = dense_flops(cfg)
    if args.block == 16:
        f_sparse = sparse_flops_b16(cfg, runner.traj.union.cpu().numpy())
    else:
        f_sparse = sparse_flops(cfg, ro, ci)
    nwin = cfg.window[1] - cfg.window[0] + 1
    traj_flops = cfg.t_d * f_dense + (cfg.steps - cfg.t_d) * f_sparse
    density = runner.traj.density()

    sampler = ClockSampler(local).start() if args.clocks else None
    barrier()
    torch.cuda.synchronize()
    events = {}
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for _ in range(args.steps):
        runner.run(q, k, v, events=events)
    t_end.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    ms_local = t_start.elapsed_time(t_end) / args.steps
    ms = reduce_max(ms_local, device)
    status = ops.device_status()
    launches = runner.launches_per_trajectory() * args.steps

    def avg_us(kind):
        xs = [a.elapsed_time(b) * 1000.0 for a, b in events.get(kind, [])]
        return (statistics.median(xs), xs) if xs else (None, [])

    dense_us, _ = avg_us("dense")
    win_us, _ = avg_us("window")
    sched_us, _ = avg_us("schedule")
    sparse_us, sparse_all = avg_us("sparse")
    q25, q75 = (np.percentile(sparse_all, [25, 75]).tolist() if sparse_all else (None, None))

    total_flops = reduce_sum(traj_flops, device)   # all ranks' useful work per step
    value = total_flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    # dominant kernel of the trajectory: the block-sparse or the dense attention launch
    t_sparse_tot = (cfg.steps - cfg.t_d) * (sparse_us or 0.0)
    t_dense_tot = (cfg.t_d - nwin) * (dense_us or 0.0)
    if t_sparse_tot >= t_dense_tot:
        kname, k_us, k_flops = "sparse_attn", sparse_us, f_sparse
    else:
        kname, k_us, k_flops = "dense_attn", dense_us, f_dense
    # each launch is timed on its own (~0.2 ms at 4K) at full clock: the burst figure
    peak = float(peaks["bf16_tflops"])
    achieved = k_flops / (k_us * 1e-6) / 1e12
    roofline = {"bound": "tensor", "kernel": kname, "achieved": round(achieved, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} bf16_tflops (burst: dense bf16 cuBLAS GEMM, best "
                               f"of 10, at {peaks.get('sm_max_mhz', 'max')} MHz)",
                "traffic": profiled_traffic(kname, cfg.name),
                "flops_per_launch": k_flops}

    routing = (routing_stats(cfg, q, k, v, device, args.block)
               if args.routing and args.block != 16 else None)
    matched = (matched_record(cfg, q, k, v, runner, device, f_sparse)
               if args.block != 16 else None)

    e2e = None
    if args.e2e:
        shp = (cfg.steps, cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim)
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        e2e_s, h2d, d2h = run_e2e(cfg, runner, hq, hk, hv, reps=args.e2e_reps)
        e2e_s = reduce_max(e2e_s, device)
        e2e = {"value": round(total_flops / e2e_s / 1e12, 3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e2e_s * 1e3, 3)}
        del hq, hk, hv

    workloads = None
    if args.configs and (args.block == 16 or world > 1):
        workloads = {"skipped": "per-workload records are taken at block size 32 on one GPU"}
    elif args.configs:
        # every other workload (16K also at eta = 1 on the same inputs), then the
        # supplementary sparse-regime one; the headline's inputs are freed first
        from wise_inputs import CONFIGS, SUPPLEMENTARY
        del q, k, v
        runner = None
        torch.cuda.empty_cache()
        todo = [c for n, c in CONFIGS.items() if n != cfg.name] + list(SUPPLEMENTARY.values())
        workloads = {}
        for c in todo:
            xq, xk, xv, _ = make_inputs(c, 0, device, workers)
            workloads[c.name] = config_record(c, xq, xk, xv, device, args.config_reps, peak)
            if c.name == "16k":
                workloads["16k_eta1"] = config_record(c.with_(eta=1.0), xq, xk, xv, device,
                                                      args.config_reps, peak)
            del xq, xk, xv
            torch.cuda.empty_cache()
        if "4k_sparse" in workloads:
            workloads["4k_sparse"]["note"] = (
                "supplementary: the 4K workload with the hot-block bias raised from 3 to 7.5 "
                "(a working set of ~40% of causal blocks); not one of the five configs")

    cpu = None
    if rank == 0 and world == 1 and args.cpu_baseline:
        secs, fl, desc = cpu_oracle_sample(cfg, n_heads=args.cpu_heads, block=args.block)
        cpu = {"value": round(fl / secs / 1e12, 6), "unit": UNIT, "cores": blas_threads(),
               "kind": "oracle", "sample": desc, "seconds": round(secs, 2)}

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generator standing in for the pages' saved Huginn workloads)",
        "config": {"workload": f"{cfg.name}: batch {cfg.batch}, {cfg.heads} heads, head_dim "
                               f"{cfg.head_dim}, n={cfg.seqlen}, T={cfg.steps}, dense 1-{cfg.t_d}, "
                               f"union {cfg.window[0]}-{cfg.window[1]}, eta={cfg.eta}, "
                               f"B={args.block}"
                               + ({16: " (32x32 tiles with 16x16 sub-masks)", 32: ""}
                                  .get(args.block, " (run as 32x32 subtiles)")),
                   "step": "one full WISE trajectory (dense + mass/select + schedule + sparse)",
                   "seed": f"[{cfg.seed}, rank, batch, head] per head (PCG64)",
                   "l2": "inputs larger than L2: every trajectory streams "
                         f"{3 * cfg.steps * cfg.bh * cfg.seqlen * cfg.head_dim * 2 / 1e9:.2f} GB "
                         "of fresh Q/K/V",
                   "parallelism": f"dp{world} (independent trajectories per GPU)"},
        "trajectory_us": round(ms * 1000.0, 1),
        "late_step_us": round(sparse_us, 2) if sparse_us else None,
        "late_step_iqr_us": [round(q25, 2), round(q75, 2)] if q25 is not None else None,
        "late_step_tflops": round(f_sparse / (sparse_us * 1e-6) / 1e12, 2) if sparse_us else None,
        "setup_inclusive_late_us": round(((cfg.steps - cfg.t_d) * sparse_us + sched_us)
                                         / (cfg.steps - cfg.t_d), 2)
                                   if sparse_us and sched_us else None,
        "dense_step_us": round(dense_us, 2) if dense_us else None,
        "dense_step_tflops": round(f_dense / (dense_us * 1e-6) / 1e12, 2) if dense_us else None,
        # a window step: attention + block mass + selection (three launches)
        "window_step_us": round(win_us, 2) if win_us else None,
        "window_over_dense_us": round(win_us - dense_us, 2) if win_us and dense_us else None,
        "schedule_us": round(sched_us, 2) if sched_us else None,
        "density": round(density, 4), "nnz_blocks": nnz,
        "routing": routing,
        "matched": matched,
        "workloads": workloads,
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
        "gpu_launches": launches,
        "device_status": status,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


# ------------------------------------------------------------------ the reference arm (oracle)

def bench_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    cfg = workload(args)
    for _ in range(args.warmup):
        cpu_oracle_sample(cfg, n_heads=1, block=args.block)
    secs, flops = 0.0, 0.0
    desc = ""
    for _ in range(args.steps):
        s, f, desc = cpu_oracle_sample(cfg, n_heads=1, block=args.block)
        secs += s
        flops += f
    value = flops / secs / 1e12
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "impl": "reference",
        "data": "synthetic (seeded generator)",
        "config": {"workload": f"{cfg.name}, dense 1-{cfg.t_d}, union {cfg.window[0]}-"
                               f"{cfg.window[1]}, eta={cfg.eta}, B={args.block}",
                   "step": "bounded oracle sample (see cpu_baseline)"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "kind": "oracle",
                         "cores": blas_threads(), "sample": desc},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["wise", "reference"], default="wise")
    ap.add_argument("--config", default="4k")
    ap.add_argument("--block", type=int, choices=[16, 32, 64, 128], default=32,
                    help="selection block size (64 / 128 run as 32x32 subtiles, 16 as "
                         "32x32 tiles with 16x16 sub-masks)")
    ap.add_argument("--eta", type=float, default=None,
                    help="mass threshold (default: the workload's, 0.95)")
    ap.add_argument("--t-d", dest="t_d", type=int, default=None,
                    help="discovery depth: last dense step (default 12)")
    ap.add_argument("--window", type=int, nargs=2, default=None, metavar=("FIRST", "LAST"),
                    help="discovery window (default: the last four steps up to t_d)")
    ap.add_argument("--workers", type=int, default=0)
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--e2e-reps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-heads", type=int, default=16)
    ap.add_argument("--no-clocks", dest="clocks", action="store_false")
    ap.add_argument("--no-routing", dest="routing", action="store_false",
                    help="skip the untimed density / retained-future-mass pass")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the per-workload records of the other configs (measured "
                         "after the headline's timed region)")
    ap.add_argument("--config-reps", type=int, default=3,
                    help="trajectories timed per extra workload record")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_wise(args)


if __name__ == "__main__":
    main()
