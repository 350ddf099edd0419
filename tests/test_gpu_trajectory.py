"""Full WISE trajectories on the GPU against the oracle, for every workload config.

The GPU runs every head of the config through the same calls the benchmark
times (WiseTrajectory: dense / dense+mass+select / schedule / sparse); the
oracle recomputes sampled heads from the same seeded inputs.  Checked:
dense O, block masses and per-step selections on window steps (bit-exact up to
near-cut rows), union = OR of the step selections, schedule = CSR of the union
(bit-exact), and late-step O against masked attention with the GPU's schedule.
The 16K config also runs an eta = 1.0 trajectory whose late steps must equal
dense causal attention; the 1K config also runs the 64 / 128-token block-size
variants (selection on the coarse masses, run as 32 x 32 subtiles).
"""

import os

import numpy as np
import pytest

from oracle import wise_oracle as O
from parity_utils import (MASS_TOL, O_OBSERVED, bits_to_bool, check_csr, compare_o,
                          compare_selection)
from traj_oracle import check_heads
from wise_inputs import CONFIGS, SUPPLEMENTARY, bf16_bits_to_f64, iter_steps
from wise_inputs.generator import StepPool

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def run_config(cfg, sel_heads, o_heads, o_steps, etas=(None,), block=32):
    """Run all heads of `cfg` on the GPU; return host copies for the checked heads:
    window-step masses / selections, union and schedule for `sel_heads`, and O at
    `o_steps` for `o_heads`."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from recurrent_depth_lm_b200 import WiseTrajectory, ops
    heads = sorted(set(sel_heads) | set(o_heads))
    idx = [b * cfg.heads + h for (b, h) in heads]
    oi = [heads.index(x) for x in o_heads]
    trajs = {eta: WiseTrajectory(cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim, t_d=cfg.t_d,
                                 window=cfg.window, eta=cfg.eta if eta is None else eta,
                                 block=block, keep_step_bits=True) for eta in etas}
    res = {eta: {"o": {}, "mass": {}, "bits": {}} for eta in etas}
    workers = max(1, min(16, (os.cpu_count() or 2)))
    with StepPool(cfg, workers=workers) as pool:
        for t, q, k, v in pool:
            dq, dk, dv = _dev(q), _dev(k), _dev(v)
            for eta, tr in trajs.items():
                o = tr.step(t, dq, dk, dv)
                flat = lambda x: x.reshape(cfg.bh, *x.shape[2:])[idx]
                if t in o_steps:
                    res[eta]["o"][t] = flat(o).float().cpu().numpy()
                if tr.in_window(t):
                    res[eta]["mass"][t] = flat(tr.mass).cpu().numpy()
                    res[eta]["bits"][t] = flat(tr.step_bits[t]).cpu().numpy()
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    jobs = {}
    for eta, tr in trajs.items():
        ro = tr.row_offsets.cpu().numpy()
        ci = tr.col_idx.cpu().numpy()
        nq = cfg.nq
        union = tr.union.reshape(cfg.bh, nq, -1)[idx].cpu().numpy()
        r = res[eta]
        jobs[eta] = []
        for j, (hd, i) in enumerate(zip(heads, idx)):
            gpu = {"mass": {t: m[j] for t, m in r["mass"].items()},
                   "bits": {t: bb[j] for t, bb in r["bits"].items()},
                   "union": union[j],
                   "sched": (ro[i * nq:(i + 1) * nq + 1] - ro[i * nq],
                             ci[ro[i * nq]:ro[(i + 1) * nq]]),
                   "o": {t: o[j] for t, o in r["o"].items()} if j in oi else {}}
            jobs[eta].append((cfg, hd, cfg.eta if eta is None else eta, block, gpu))
        jobs[eta] = (jobs[eta], tr.density())
    return jobs


def check_config(cfg, sel_heads, o_heads, o_steps, etas=(None,), block=32):
    """Returns {eta: {"exempt_rows", "density", "o_max", "heads"}}; prints the counts."""
    jobs = run_config(cfg, sel_heads, o_heads, o_steps, etas, block)
    report = {}
    for eta, (js, density) in jobs.items():
        out = check_heads(js)
        O_OBSERVED.extend((x[1], x[2]) for r in out for x in r["o"])   # worker comparisons
        o_max = max((x[1] for r in out for x in r["o"]), default=0.0)
        report[eta] = {"exempt_rows": sum(r["exempt"] for r in out), "density": density,
                       "o_max": o_max, "heads": len(out)}
        print(f"{cfg.name} eta={eta or cfg.eta} block={block}: {len(out)} heads checked, "
              f"{report[eta]['exempt_rows']} near-cut rows exempt, worst O max-abs "
              f"{o_max:.3e}, density {density:.4f}")
    return report


def all_heads(cfg):
    return [(b, h) for b in range(cfg.batch) for h in range(cfg.heads)]


def test_trajectory_tiny_all_heads_all_steps():
    cfg = CONFIGS["tiny"]
    rep = check_config(cfg, all_heads(cfg), all_heads(cfg), range(1, cfg.steps + 1))
    assert rep[None]["exempt_rows"] <= 1


def test_trajectory_1k():
    cfg = CONFIGS["1k"]
    rep = check_config(cfg, all_heads(cfg), [(0, 0), (0, 13), (0, 22), (0, 31)],
                       range(1, cfg.steps + 1))
    # 32 heads x 32 query blocks x 4 window steps = 4096 selection rows
    assert rep[None]["exempt_rows"] <= 8


@pytest.mark.parametrize("block", [64, 128])
def test_trajectory_1k_block_sizes(block):
    cfg = CONFIGS["1k"]
    rep = check_config(cfg, [(0, 0), (0, 31)], [(0, 0), (0, 31)], [12, 13, 32], block=block)
    assert rep[None]["exempt_rows"] <= 2


# One-at-a-time variants of the frozen configuration (WISE paper appendix C.5, Table 7,
# and C.7, Table 9): the mass threshold, the discovery depth and the union width.
VARIANTS = [
    dict(eta=0.90), dict(eta=0.98), dict(eta=0.99),
    dict(t_d=8, window=(5, 8)), dict(t_d=16, window=(13, 16)),
    dict(window=(12, 12)), dict(window=(11, 12)),
]


@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: "-".join(f"{k}{v[k]}" for k in v))
def test_trajectory_1k_hyperparameter_variants(variant):
    cfg = CONFIGS["1k"].with_(**variant)
    late = [cfg.t_d + 1, cfg.steps]
    rep = check_config(cfg, [(0, 3), (0, 30)], [(0, 3), (0, 30)], late)
    assert rep[None]["exempt_rows"] <= 2


def test_trajectory_4k():
    cfg = CONFIGS["4k"]
    # every head's window-step masses and selections (32 x 128 x 4 = 16384 rows); O on 4
    rep = check_config(cfg, all_heads(cfg), [(0, 0), (0, 11), (0, 21), (0, 31)],
                       [1, 9, 12, 13, 20, 32])
    assert rep[None]["exempt_rows"] <= 16


def test_trajectory_2k_b4_h40_d96():
    cfg = CONFIGS["2k_b4_h40_d96"]
    # every head of every batch (160 x 64 x 4 = 40960 selection rows); O on 5 heads,
    # including the last head of the last batch
    rep = check_config(cfg, all_heads(cfg), [(0, 0), (1, 20), (2, 17), (3, 0), (3, 39)],
                       [1, 12, 13, 25, 32])
    assert rep[None]["exempt_rows"] <= 40


def test_trajectory_4k_sparse_regime():
    """The supplementary 4K workload with a ~40% working set (hot-block bias 7.5)."""
    cfg = SUPPLEMENTARY["4k_sparse"]
    rep = check_config(cfg, all_heads(cfg), [(0, 0), (0, 7), (0, 21), (0, 31)],
                       [12, 13, 20, 32])
    assert rep[None]["exempt_rows"] <= 16
    assert 0.25 < rep[None]["density"] < 0.65


def test_trajectory_16k_and_eta_one():
    cfg = CONFIGS["16k"]
    # 8 heads' window-step masses and selections (8 x 512 x 4 = 16384 rows); O on 4
    sel = [(0, h) for h in (0, 5, 9, 14, 18, 23, 27, 31)]
    rep = check_config(cfg, sel, [(0, 5), (0, 14), (0, 23), (0, 31)], [12, 13, 32],
                       etas=(None, 1.0))
    assert rep[None]["exempt_rows"] <= 16
    assert rep[1.0]["exempt_rows"] == 0 and rep[1.0]["density"] == 1.0


# ------------------------------------------------------------- selection-only controls

def _size_matched_near_tie(row, k):
    """The K-th and (K+1)-th largest masses are within the mass tolerance (TopK may flip)."""
    srt = np.sort(row)[::-1]
    return 0 < k < len(srt) and srt[k - 1] - srt[k] <= MASS_TOL


@pytest.mark.parametrize("support", ["wise", "static95", "size_matched", "mass_matched"])
def test_trajectory_controls_and_retained_mass(support):
    """Late steps on a control support (appendix B "Intervention controls") with the retained
    future mass tracked.  The control is checked against the oracle's control computed from
    the oracle's step-1 masses and the GPU's own union (so a near-cut flip in the union does
    not cascade); the schedule, late O and per-row retained mass against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from recurrent_depth_lm_b200 import WiseTrajectory, ops
    cfg = CONFIGS["1k"]
    sample = [(0, 0), (0, 31)]
    idx = [b * cfg.heads + h for (b, h) in sample]
    nq = cfg.nq
    check_steps = [13, 20, 32]
    tr = WiseTrajectory(cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim, t_d=cfg.t_d,
                        window=cfg.window, eta=cfg.eta, support=support, track_retained=True)
    flat = lambda x: x.reshape(cfg.bh, *x.shape[2:])[idx]
    o_late, retained = {}, {}
    with StepPool(cfg, workers=max(1, min(16, os.cpu_count() or 2))) as pool:
        for t, q, k, v in pool:
            o = tr.step(t, _dev(q), _dev(k), _dev(v))
            if t == 1 and tr.mass1 is not None:
                mass1 = flat(tr.mass1).cpu().numpy()
            if t in check_steps:
                o_late[t] = flat(o).float().cpu().numpy()
            if t > cfg.t_d:
                retained[t] = flat(tr.retained[t]).cpu().numpy()
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    union = bits_to_bool(flat(tr.union).cpu().numpy(), nq)
    frozen = bits_to_bool(flat(tr.frozen).cpu().numpy(), nq)
    ro_all, ci_all = tr.row_offsets.cpu().numpy(), tr.col_idx.cpu().numpy()
    host = {t: (q, k, v) for t, q, k, v in iter_steps(cfg, heads=sample)}
    exempt = 0
    for si, bhi in enumerate(idx):
        ro = ro_all[bhi * nq:(bhi + 1) * nq + 1] - ro_all[bhi * nq]
        ci = ci_all[ro_all[bhi * nq]:ro_all[(bhi + 1) * nq]]
        check_csr(ro, ci, frozen[si])
        if support != "wise":
            q1, k1, _ = (bf16_bits_to_f64(x[si]) for x in host[1])
            r1 = O.block_mass(q1, k1, cfg.scale)
            assert np.abs(np.tril(mass1[si]) - r1).max() <= MASS_TOL
            if support == "static95":
                exempt += compare_selection(frozen[si], r1, cfg.eta)
            else:
                want = (O.size_matched if support == "size_matched" else O.mass_matched)(
                    r1, union[si])
                for qb in range(nq):
                    if np.array_equal(frozen[si, qb], want[qb]):
                        continue
                    row = r1[qb, : qb + 1]
                    if support == "size_matched":
                        assert frozen[si, qb].sum() == np.tril(union[si])[qb].sum()
                        assert _size_matched_near_tie(row, int(want[qb].sum())), qb
                    else:
                        m = O.retained_mass(r1, union[si])[qb]
                        d_ck, d_ck1, _ = O.cut_margins(row, m)
                        assert min(d_ck, d_ck1) <= 1e-4, qb
                    exempt += 1
        else:
            assert np.array_equal(frozen[si], union[si])
        for t in range(cfg.t_d + 1, cfg.steps + 1):
            if t not in check_steps:
                continue
            q, k, v = (bf16_bits_to_f64(x[si]) for x in host[t])
            ref, _ = O.masked_attention(q, k, v, frozen[si], cfg.scale)
            compare_o(o_late[t][si], ref, f"{support} head {sample[si]} step {t}")
            want_ret = O.retained_mass(O.block_mass(q, k, cfg.scale), frozen[si])
            assert np.abs(retained[t][si] - want_ret).max() <= MASS_TOL
    assert exempt <= 3
    rfm = tr.retained_future_mass()
    assert 0.0 < rfm <= 1.0 + 1e-6


# ------------------------------------------------------------- block size 16

def test_trajectory_1k_block16():
    """B = 16 (appendix C.6): window-step selections over 16-token masses against the
    oracle's, the union, the schedule decoded back to the union, and late O against
    masked attention at B = 16 over the GPU's union."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from recurrent_depth_lm_b200 import WiseTrajectory, ops
    cfg = CONFIGS["1k"]
    sample = [(0, 2), (0, 29)]
    idx = [b * cfg.heads + h for (b, h) in sample]
    nq, n16 = cfg.nq, cfg.seqlen // 16
    check_steps = [13, 32]
    tr = WiseTrajectory(cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim, t_d=cfg.t_d,
                        window=cfg.window, eta=cfg.eta, block=16, keep_step_bits=True)
    flat = lambda x: x.reshape(cfg.bh, *x.shape[2:])[idx]
    o_late, bits = {}, {}
    with StepPool(cfg, workers=max(1, min(16, os.cpu_count() or 2))) as pool:
        for t, q, k, v in pool:
            o = tr.step(t, _dev(q), _dev(k), _dev(v))
            if tr.in_window(t):
                bits[t] = bits_to_bool(flat(tr.step_bits[t]).cpu().numpy(), n16)
            if t in check_steps:
                o_late[t] = flat(o).float().cpu().numpy()
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    union = bits_to_bool(flat(tr.union).cpu().numpy(), n16)
    ro_all, ci_all = tr.row_offsets.cpu().numpy(), tr.col_idx.cpu().numpy()
    sub_all = tr.sub.cpu().numpy()
    host = {t: (q, k, v) for t, q, k, v in iter_steps(cfg, heads=sample)}
    exempt = 0
    for si, bhi in enumerate(idx):
        steps = []
        for t in range(cfg.window[0], cfg.window[1] + 1):
            q, k, _ = (bf16_bits_to_f64(x[si]) for x in host[t])
            exempt += compare_selection(bits[t][si], O.block_mass(q, k, cfg.scale, block=16),
                                        cfg.eta)
            steps.append(bits[t][si])
        assert np.array_equal(union[si], O.temporal_union(steps))
        lo, hi = ro_all[bhi * nq], ro_all[(bhi + 1) * nq]
        sel = np.zeros((n16, n16), bool)
        for qq in range(nq):
            for e in range(ro_all[bhi * nq + qq], ro_all[bhi * nq + qq + 1]):
                for a in range(2):
                    for c in range(2):
                        if (sub_all[e] >> (2 * a + c)) & 1:
                            sel[2 * qq + a, 2 * ci_all[e] + c] = True
        assert hi >= lo and np.array_equal(sel, np.tril(union[si]))
        for t in check_steps:
            q, k, v = (bf16_bits_to_f64(x[si]) for x in host[t])
            ref, _ = O.masked_attention(q, k, v, union[si], cfg.scale, block=16)
            compare_o(o_late[t][si], ref, f"B16 head {sample[si]} step {t}")
    assert exempt <= 2
    assert 0.0 < tr.density() <= 1.0


def test_saved_working_set_replays_late_steps(tmp_path):
    """A trajectory restored from a saved working set runs the late steps alone and gives
    bit-identical outputs (the schedule is all the late steps depend on)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from recurrent_depth_lm_b200 import WiseTrajectory
    cfg = CONFIGS["tiny"]
    mk = lambda: WiseTrajectory(cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim, t_d=cfg.t_d,
                                window=cfg.window, eta=cfg.eta)
    tr = mk()
    late = {}
    with StepPool(cfg, workers=2) as pool:
        for t, q, k, v in pool:
            x = (_dev(q), _dev(k), _dev(v))
            o = tr.step(t, *x)
            if t > cfg.t_d:
                late[t] = (x, o.clone())
    path = tmp_path / "working_set.npz"
    tr.save(path)
    tr2 = mk()
    tr2.load(path)
    for t, (x, o) in late.items():
        assert torch.equal(tr2.step(t, *x), o)
    torch.cuda.synchronize()
