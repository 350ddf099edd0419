"""Host-side logic that needs no GPU: trajectory argument checks, the 16-token density
count, bench.py's workload overrides and FLOP accounting."""

import argparse

import numpy as np
import pytest

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def traj_cls():
    from recurrent_depth_lm_b200.trajectory import WiseTrajectory
    return WiseTrajectory


def make(traj_cls, **kw):
    args = dict(batch=1, heads=2, seqlen=256, head_dim=64, device="cpu")
    args.update(kw)
    return traj_cls(args.pop("batch"), args.pop("heads"), args.pop("seqlen"),
                    args.pop("head_dim"), **args)


@pytest.mark.parametrize("kw", [
    dict(block=48),                                   # not a supported block size
    dict(block=128, seqlen=192),                      # seqlen not a multiple of the block
    dict(support="oracle"),                           # unknown support
    dict(support="size_matched", block=64),           # controls are defined at B = 32
    dict(support="mass_matched", block=16),
    dict(support="static95", block=16),               # B = 16 runs the WISE support only
    dict(block=16, track_retained=True),
])
def test_trajectory_rejects_bad_arguments(traj_cls, kw):
    with pytest.raises(ValueError):
        make(traj_cls, **kw)


def test_late_step_before_schedule_and_untracked_retained_mass(traj_cls):
    tr = make(traj_cls)
    x = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        tr.step(tr.t_d + 1, x, x, x)
    with pytest.raises(RuntimeError):
        tr.retained_future_mass()


def test_block16_density_counts_causal_16_token_blocks(traj_cls):
    tr = make(traj_cls, block=16, seqlen=320)
    n16 = 320 // 16
    rng = np.random.default_rng(0)
    sel = rng.random((2, n16, n16)) < 0.4
    words = np.zeros((2, n16, tr.union.shape[-1]), np.uint32)
    for b in range(n16):
        words[..., b // 32] |= sel[..., b].astype(np.uint32) << np.uint32(b % 32)
    tr.union.copy_(torch.from_numpy(words.view(np.int32)).reshape(tr.union.shape))
    want = np.tril(sel).sum() / (2 * n16 * (n16 + 1) / 2)
    assert abs(tr.density() - want) < 1e-12


def _args(**kw):
    base = dict(config="4k", eta=None, t_d=None, window=None)
    base.update(kw)
    return argparse.Namespace(**base)


def test_bench_workload_overrides():
    import bench
    cfg = bench.workload(_args())
    assert (cfg.eta, cfg.t_d, cfg.window) == (0.95, 12, (9, 12))
    cfg = bench.workload(_args(eta=0.9, t_d=8))
    assert (cfg.eta, cfg.t_d, cfg.window) == (0.9, 8, (5, 8))     # window follows t_d
    cfg = bench.workload(_args(window=[11, 12]))
    assert cfg.window == (11, 12) and cfg.t_d == 12
    with pytest.raises(SystemExit):
        bench.workload(_args(window=[10, 14]))                      # past t_d
    with pytest.raises(SystemExit):
        bench.workload(_args(t_d=32))                               # no late step left


def test_bench_flops_b16_counts_pairs_inside_kept_blocks():
    """4*d per admissible pair: 16*16 per kept off-diagonal 16-block, 16*17/2 per diagonal."""
    import bench
    from wise_inputs import CONFIGS
    cfg = CONFIGS["tiny"]                             # n = 256: 16 blocks of 16 tokens
    n16 = cfg.seqlen // 16
    sel = np.zeros((cfg.bh, n16, n16), bool)
    sel[0, 5, 5] = True                               # diagonal
    sel[0, 5, 2] = True                               # off-diagonal
    sel[1, 3, 7] = True                               # above the diagonal: not counted
    words = np.zeros((cfg.bh, n16, 1), np.uint32)
    for b in range(n16):
        words[..., 0] |= sel[..., b].astype(np.uint32) << np.uint32(b)
    flops = bench.sparse_flops_b16(cfg, words.view(np.int32))
    assert flops == 4.0 * cfg.head_dim * (256 + 136)


def test_bench_tile_waste_counts_the_union_of_four_query_blocks():
    """A 128-row tile issues every key block any of its 4 query blocks keeps, for all 4."""
    import bench
    from oracle import wise_oracle as O
    from wise_inputs import CONFIGS
    cfg = CONFIGS["tiny"].with_(heads=1)                # nq = 8: two tiles per head
    full = np.tril(np.ones((8, 8), bool))
    ro, ci = O.csr_schedule(full)
    issued, selected = bench.tile_waste(cfg, ro, ci)
    assert (issued, selected) == (4 * 4 + 4 * 8, 36)    # tiles run blocks 0-3 and 0-7
    own = np.zeros((8, 8), bool)
    own[4:, 0] = own[4:, 2] = True                      # rows 4-7 share one list
    own[:4, 0] = True
    own[1, 1] = True                                    # row 1 alone keeps block 1
    ro, ci = O.csr_schedule(own)
    assert bench.tile_waste(cfg, ro, ci) == (4 * 2 + 4 * 2, 4 + 1 + 8)
    two = cfg.with_(heads=2)                            # heads never share a tile
    ro2 = np.concatenate([ro, ro[1:] + ro[-1]])
    assert bench.tile_waste(two, ro2, np.concatenate([ci, ci])) == (32, 26)


def _fake_schedule(tr, rng):
    """A random causal working set and its CSR written into a CPU trajectory's buffers."""
    from oracle import wise_oracle as O
    nq = tr.nq
    words = np.zeros(tuple(tr.union.shape), np.uint32)
    ro_all, ci_all = [0], []
    for x in range(tr.b * tr.h):
        sup = np.tril(rng.random((nq, nq)) < 0.5)
        np.fill_diagonal(sup, True)
        for b in range(nq):
            words[0, x, :, b // 32] |= sup[:, b].astype(np.uint32) << np.uint32(b % 32)
        ro, ci = O.csr_schedule(sup)
        ro_all += (ro[1:] + ro_all[-1]).tolist()
        ci_all += ci.tolist()
    tr.union.copy_(torch.from_numpy(words.view(np.int32)))
    tr.row_offsets.copy_(torch.tensor(ro_all, dtype=torch.int32))
    tr.col_idx[:len(ci_all)].copy_(torch.tensor(ci_all, dtype=torch.int32))
    tr.scheduled = True
    return len(ci_all)


def test_save_and_load_round_trip(traj_cls, tmp_path):
    tr = make(traj_cls, heads=3, seqlen=320)
    with pytest.raises(RuntimeError):
        tr.state()                                     # nothing frozen yet
    nnz = _fake_schedule(tr, np.random.default_rng(5))
    path = tmp_path / "ws.npz"
    tr.save(path)
    tr2 = make(traj_cls, heads=3, seqlen=320)
    tr2.load(path)
    assert tr2.scheduled and tr2.nnz() == nnz
    assert torch.equal(tr2.union, tr.union)
    assert torch.equal(tr2.row_offsets, tr.row_offsets)
    assert torch.equal(tr2.col_idx[:nnz], tr.col_idx[:nnz])
    with pytest.raises(ValueError):
        make(traj_cls, heads=3, seqlen=256).load(path)     # another shape
    with pytest.raises(ValueError):
        make(traj_cls, heads=3, seqlen=320, block=64).load(path)   # another block size
