"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): max/sum over
ranks, barrier, per-rank seeds, and the weak-scaling throughput formula."""

import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, lr = bench.dist_env()
    bench.init_dist(w, "gloo")
    dev = torch.device("cpu")
    ms = 10.0 + 5.0 * r                       # rank 1 is slower
    mx = bench.reduce_max(ms, dev)
    tot = bench.reduce_sum(1e12, dev)         # each rank did 1 TFLOP of useful work
    bench.barrier()
    from wise_inputs import CONFIGS, iter_steps
    first = next(iter_steps(CONFIGS["tiny"], heads=[(0, 0)], rank=r))[1]
    q.put((r, mx, tot, tot / (mx * 1e-3) / 1e12, first[0, :4, :4].tobytes()))
    dist.destroy_process_group()


def test_two_rank_reductions_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, mx0, tot0, v0, d0), (r1, mx1, tot1, v1, d1) = out
    assert mx0 == mx1 == 15.0                 # max over ranks, the slowest rank decides
    assert tot0 == tot1 == 2e12               # whole-job work
    assert abs(v0 - 2e12 / 15e-3 / 1e12) < 1e-9
    assert d0 != d1                           # ranks draw disjoint synthetic data


def test_single_process_reductions_are_identity():
    import bench
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    assert bench.reduce_sum(2.0, torch.device("cpu")) == 2.0


def test_reference_arm_json_contract(capsys, monkeypatch):
    """`bench.py --impl reference` prints one JSON line with the contract's keys (the
    oracle timed on the host on a bounded sample); a non-zero rank prints nothing."""
    import json

    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    bench.main(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "3",
                "--eta", "0.9"])
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "eta=0.9" in d["config"]["workload"]
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    bench.main(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out.strip() == ""


def test_bench_rejects_fewer_than_three_warmups():
    import bench
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "2"])
