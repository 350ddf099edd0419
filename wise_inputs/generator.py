"""Seeded synthetic Q/K/V workloads for the WISE attention hot path.

This module is shared by the CPU oracle, the tests and the benchmark.  It
draws random numbers and rounds them to bf16; it holds none of the method's
arithmetic (no attention, no block mass, no selection, no schedule).

Workload recipe (stand-in for the unreleased saved Huginn/HotpotQA attention
workloads of "Attention Routing Stabilizes Early: Working-Set Inference for
Recurrent-Depth Language Models", App. B "Systems evaluation"):

* every (batch, head) pair owns an independent PCG64 stream seeded with
  ``[config.seed, rank, b, h]``, so any single head can be regenerated without
  the others and ranks of a multi-GPU run draw disjoint data;
* per head, in this order: a unit vector ``u`` (normalised N(0, I_d)); for
  configs with a hot-fraction range, the head's fraction ~ U(lo, hi); a hot
  key-block set of ``max(1, round(f * nq))`` blocks drawn without
  replacement; for configs with a diagonal/first-block bias, one unit vector
  ``v_b`` per key block; base Q, K, V ~ N(0, 1) of shape [n, d] (fp32);
* ``Q += bias * u`` on every query, ``K += bias * u`` on keys of hot blocks;
  with a diagonal/first-block bias ``c``: ``K[block 0] += c * u`` and, for
  every block b, ``Q[block b] += c * v_b`` and ``K[block b] += c * v_b``;
* recurrent drift: for t = 1..T, ``X^(t) = X^(t-1) + sigma0 * decay**t * eps``
  for X in (Q, K, V), eps ~ N(0, 1) drawn as eps_Q, eps_K, eps_V; fp32 masters
  are kept and each step is rounded to bf16 (round to nearest even).

Arrays handed out are bf16 bit patterns (``uint16``) in [B, H, n, d] order.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Iterator, Sequence

import numpy as np

BLOCK = 32


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    batch: int
    heads: int
    head_dim: int
    seqlen: int
    steps: int            # T, recurrent steps
    t_d: int              # last exploration (dense) step
    window: tuple         # (first, last) step whose selections are unioned
    hot_frac: object      # float, or (lo, hi) drawn per head
    seed: int
    bias: float = 3.0
    diag_first_bias: float = 0.0
    sigma0: float = 0.3
    decay: float = 0.8
    eta: float = 0.95

    @property
    def nq(self) -> int:
        return self.seqlen // BLOCK

    @property
    def bh(self) -> int:
        return self.batch * self.heads

    @property
    def scale(self) -> float:
        return float(1.0 / np.sqrt(self.head_dim))

    def with_(self, **kw) -> "WorkloadConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": WorkloadConfig("tiny", 1, 2, 64, 256, steps=8, t_d=4, window=(3, 4),
                           hot_frac=0.25, seed=0),
    "1k": WorkloadConfig("1k", 1, 32, 128, 1024, steps=32, t_d=12, window=(9, 12),
                         hot_frac=0.15, seed=1),
    "4k": WorkloadConfig("4k", 1, 32, 128, 4096, steps=32, t_d=12, window=(9, 12),
                         hot_frac=0.08, seed=2, diag_first_bias=2.0),
    "2k_b4_h40_d96": WorkloadConfig("2k_b4_h40_d96", 4, 40, 96, 2048, steps=32, t_d=12,
                                    window=(9, 12), hot_frac=(0.05, 0.20), seed=3,
                                    sigma0=0.4),
    "16k": WorkloadConfig("16k", 1, 32, 128, 16384, steps=32, t_d=12, window=(9, 12),
                          hot_frac=0.03, seed=4),
}

# Supplementary workload, not one of the five above: the 4K workload with the hot-block
# bias raised from 3 to 7.5, which brings the working set to ~40% of the causal blocks
# (the 4K density range the paper reports) so that late-step cost against density can
# be measured.  With bias 3 every config keeps ~94% of its causal blocks.
SUPPLEMENTARY = {
    "4k_sparse": dataclasses.replace(CONFIGS["4k"], name="4k_sparse", bias=7.5),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((b >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


class HeadStream:
    """Generator state of one (batch, head): fp32 masters plus its PCG64 stream."""

    def __init__(self, cfg: WorkloadConfig, b: int, h: int, rank: int = 0):
        self.cfg = cfg
        rng = np.random.default_rng([cfg.seed, rank, b, h])
        self.rng = rng
        n, d, nq = cfg.seqlen, cfg.head_dim, cfg.nq
        u = rng.standard_normal(d)
        u = (u / np.linalg.norm(u)).astype(np.float32)
        if isinstance(cfg.hot_frac, tuple):
            frac = float(rng.uniform(cfg.hot_frac[0], cfg.hot_frac[1]))
        else:
            frac = float(cfg.hot_frac)
        m = max(1, int(round(frac * nq)))
        self.hot_blocks = np.sort(rng.choice(nq, size=m, replace=False))
        vb = None
        if cfg.diag_first_bias:
            vb = rng.standard_normal((nq, d))
            vb = (vb / np.linalg.norm(vb, axis=1, keepdims=True)).astype(np.float32)
        q = rng.standard_normal((n, d), dtype=np.float32)
        k = rng.standard_normal((n, d), dtype=np.float32)
        v = rng.standard_normal((n, d), dtype=np.float32)
        q += np.float32(cfg.bias) * u
        hot_rows = (self.hot_blocks[:, None] * BLOCK + np.arange(BLOCK)[None, :]).ravel()
        k[hot_rows] += np.float32(cfg.bias) * u
        if vb is not None:
            c = np.float32(cfg.diag_first_bias)
            k[:BLOCK] += c * u
            per_row = np.repeat(vb, BLOCK, axis=0)
            q += c * per_row
            k += c * per_row
        self.masters = [q, k, v]
        self.t = 0

    def next_step(self):
        """Advance to the next recurrent step; returns bf16 bits (q, k, v), each [n, d]."""
        self.t += 1
        sigma = np.float32(self.cfg.sigma0 * self.cfg.decay ** self.t)
        n, d = self.cfg.seqlen, self.cfg.head_dim
        out = []
        for x in self.masters:
            x += sigma * self.rng.standard_normal((n, d), dtype=np.float32)
            out.append(f32_to_bf16_bits(x))
        return tuple(out)


def all_heads(cfg: WorkloadConfig):
    return [(b, h) for b in range(cfg.batch) for h in range(cfg.heads)]


def iter_steps(cfg: WorkloadConfig, heads: Sequence | None = None, rank: int = 0,
               steps: int | None = None) -> Iterator:
    """Yield (t, Q, K, V) for t = 1..T.

    With ``heads=None`` the arrays are [B, H, n, d]; otherwise ``heads`` is a
    list of (b, h) pairs and the arrays are [len(heads), n, d].
    """
    sel = all_heads(cfg) if heads is None else list(heads)
    streams = [HeadStream(cfg, b, h, rank) for (b, h) in sel]
    n, d = cfg.seqlen, cfg.head_dim
    T = cfg.steps if steps is None else steps
    for t in range(1, T + 1):
        qs = np.empty((len(sel), n, d), np.uint16)
        ks = np.empty_like(qs)
        vs = np.empty_like(qs)
        for i, s in enumerate(streams):
            qs[i], ks[i], vs[i] = s.next_step()
        if heads is None:
            shp = (cfg.batch, cfg.heads, n, d)
            qs, ks, vs = qs.reshape(shp), ks.reshape(shp), vs.reshape(shp)
        yield t, qs, ks, vs


def _head_all_steps(args):
    cfg, b, h, rank, T = args
    s = HeadStream(cfg, b, h, rank)
    n, d = cfg.seqlen, cfg.head_dim
    out = np.empty((T, 3, n, d), np.uint16)
    for t in range(T):
        out[t, 0], out[t, 1], out[t, 2] = s.next_step()
    return out


def generate_all_steps(cfg: WorkloadConfig, rank: int = 0, steps: int | None = None,
                       workers: int = 1) -> np.ndarray:
    """All steps at once: bf16 bits [T, 3, B, H, n, d] (3 = Q, K, V).

    ``workers > 1`` spreads heads over a spawn-started process pool; the
    result is identical to the serial one since every head has its own stream.
    """
    T = cfg.steps if steps is None else steps
    sel = all_heads(cfg)
    jobs = [(cfg, b, h, rank, T) for (b, h) in sel]
    if workers > 1:
        import multiprocessing as mp
        with mp.get_context("spawn").Pool(workers) as pool:
            parts = pool.map(_head_all_steps, jobs, chunksize=1)
    else:
        parts = [_head_all_steps(j) for j in jobs]
    arr = np.stack(parts, axis=2)  # [T, 3, BH, n, d]
    return arr.reshape(T, 3, cfg.batch, cfg.heads, cfg.seqlen, cfg.head_dim)


def _pool_worker(conn, cfg, heads, rank, T):
    streams = [HeadStream(cfg, b, h, rank) for (b, h) in heads]
    n, d = cfg.seqlen, cfg.head_dim
    for _ in range(T):
        if conn.recv() is None:
            break
        out = np.empty((len(streams), 3, n, d), np.uint16)
        for i, s in enumerate(streams):
            out[i, 0], out[i, 1], out[i, 2] = s.next_step()
        conn.send_bytes(out.tobytes())
    conn.close()


class StepPool:
    """Step-by-step generation of all heads, spread over spawn-started processes.

    Yields the same arrays as ``iter_steps(cfg)`` (every head owns its stream)
    while bounding host memory to one step.  Use as a context manager.
    """

    def __init__(self, cfg: WorkloadConfig, workers: int, rank: int = 0, steps: int | None = None):
        import multiprocessing as mp
        self.cfg = cfg
        self.T = cfg.steps if steps is None else steps
        heads = all_heads(cfg)
        workers = max(1, min(workers, len(heads)))
        self.parts = [heads[i::workers] for i in range(workers)]
        ctx = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for part in self.parts:
            a, b = ctx.Pipe()
            p = ctx.Process(target=_pool_worker, args=(b, cfg, part, rank, self.T), daemon=True)
            p.start()
            self.conns.append(a)
            self.procs.append(p)

    def __iter__(self):
        cfg = self.cfg
        n, d = cfg.seqlen, cfg.head_dim
        for t in range(1, self.T + 1):
            for c in self.conns:
                c.send(t)
            full = np.empty((cfg.batch * cfg.heads, 3, n, d), np.uint16)
            for wi, (c, part) in enumerate(zip(self.conns, self.parts)):
                arr = np.frombuffer(c.recv_bytes(), np.uint16).reshape(len(part), 3, n, d)
                full[wi::len(self.parts)] = arr
            shp = (cfg.batch, cfg.heads, n, d)
            yield t, full[:, 0].reshape(shp), full[:, 1].reshape(shp), full[:, 2].reshape(shp)

    def close(self):
        for c in self.conns:
            try:
                c.send(None)
            except (BrokenPipeError, OSError):
                pass
        for p in self.procs:
            p.join(timeout=10)
            if p.is_alive():
                p.kill()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
