"""Per-head oracle checks of a GPU trajectory (test code, not product code).

A GPU trajectory runs every head of a workload; these checks recompute one head
at a time with the fp64 oracle from the same seeded inputs and compare:

* window steps: block masses (1e-4) and the step's selection (bit-exact up to
  near-cut rows, which are counted);
* the union equals the OR of the GPU's own step selections, and the schedule is
  the CSR of that union (bit-exact);
* the steps in ``o_steps``: dense O (t <= t_d) or O masked to the GPU's schedule
  (t > t_d); with eta >= 1 the late O must also equal dense causal attention.

Heads are independent, so they are spread over a spawn-started process pool (the
parent has initialised CUDA, and a forked child of such a process can hang).
"""

from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

from oracle import wise_oracle as O
from parity_utils import (MASS_TOL, bits_to_bool, check_csr, coarse_of_fine, compare_o,
                          compare_selection)
from wise_inputs import bf16_bits_to_f64, iter_steps


def check_head(job) -> dict:
    """One head: job = (cfg, (b, h), eta, block, gpu) with gpu = {"mass": {t: [nq, nq]},
    "bits": {t: [nq, W]}, "union": [nq, W], "sched": (ro, ci), "o": {t: [n, d]}}."""
    cfg, head, eta, block, gpu = job
    f = block // 32
    nq = cfg.nq
    win = range(cfg.window[0], cfg.window[1] + 1)
    need = set(win) | set(gpu["o"])
    out = {"head": head, "exempt": 0, "o": []}
    step_sel = []
    for t, q, k, v in iter_steps(cfg, heads=[head], steps=max(need)):
        if t not in need:
            continue
        q, k, v = (bf16_bits_to_f64(x[0]) for x in (q, k, v))
        if t in win:
            r_ref = O.block_mass(q, k, cfg.scale)
            err = np.abs(np.tril(gpu["mass"][t]) - r_ref).max()
            assert err <= MASS_TOL, f"head {head} step {t}: mass error {err:.3e}"
            sel = bits_to_bool(gpu["bits"][t], nq)
            if f == 1:
                out["exempt"] += compare_selection(sel, r_ref, eta)
            else:   # block-size variant: coarse selection, run as 32 x 32 subtiles
                coarse = coarse_of_fine(sel, f)
                assert np.array_equal(sel, O.expand_support(coarse, f))
                out["exempt"] += compare_selection(coarse, O.block_mass(q, k, cfg.scale, block),
                                                   eta)
            step_sel.append(sel)
            if t == cfg.window[1]:
                union = bits_to_bool(gpu["union"], nq)
                assert np.array_equal(union, O.temporal_union(step_sel)), f"head {head}: union"
                ro, ci = gpu["sched"]
                check_csr(ro, ci, union)
                sup = O.support_from_csr(ro, ci, nq)
        if t in gpu["o"]:
            what = f"{cfg.name} head {head} step {t}"
            if t <= cfg.t_d:
                ref, _ = O.causal_attention(q, k, v, cfg.scale)
            else:
                ref, _ = O.masked_attention(q, k, v, sup, cfg.scale)
                if eta >= 1.0:   # eta = 1 reproduces dense causal attention
                    dense, _ = O.causal_attention(q, k, v, cfg.scale)
                    compare_o(gpu["o"][t], dense, "eta=1 " + what)
            out["o"].append((t,) + compare_o(gpu["o"][t], ref, what))
    return out


def _init_worker(threads: int):
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(threads)
    except ImportError:
        pass


def check_heads(jobs) -> list:
    """Run check_head over jobs in a spawn-started pool; re-raises the first failure."""
    cpus = os.cpu_count() or 2
    workers = max(1, min(len(jobs), cpus, 32))
    if workers == 1:
        return [check_head(j) for j in jobs]
    threads = max(1, cpus // workers)
    with mp.get_context("spawn").Pool(workers, initializer=_init_worker,
                                      initargs=(threads,)) as pool:
        return pool.map(check_head, jobs, chunksize=1)
