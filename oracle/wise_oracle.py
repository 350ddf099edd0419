"""Plain CPU float64 oracle of the WISE attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or
run this module.  The product path (``recurrent_depth_lm_b200``) never does,
and this module imports nothing from it; the two share only the seeded input
generator ``wise_inputs``.

Source: Wan & Chen, "Attention Routing Stabilizes Early: Working-Set
Inference for Recurrent-Depth Language Models" (arXiv 2609.27373), called
"the WISE paper" below.  Every function cites the section or equation it
restates.  Everything is numpy float64 on bf16-exact inputs; no blocking,
fusion or reordering beyond what each definition states.

All functions work on ONE (recurrent block, head): arrays are [n, d].  Block
size B = 32 (WISE paper, §7.1 "WISE configuration").

Readings of points the paper leaves open (also listed in the design notes):

* ranking ties in the cumulative-eta support are broken by the lower block
  index first (the theory in §6.1 assumes strictly separated masses);
* the cut is "cumulative mass at least eta", i.e. cumsum >= eta (§3);
* if no prefix reaches eta (eta >= 1, or rounding), every admissible block is
  selected, which makes eta = 1 reproduce dense causal attention;
* admissible key blocks of query block q are b <= q (causal mask M of §3);
* block masses come from the full, unrestricted causal softmax of that step;
* a row with no kept admissible key (only possible for supports the method
  itself never produces) has O = 0 and lse = -inf;
* block sizes other than 32 (App. C.6): the block mass is the same definition
  at that size; 64 / 128-token supports run as 32 x 32 subtiles clipped to the
  causal part of the coarse diagonal block;
* MassMatched (App. B, whose formula for the control itself did not survive):
  the fewest step-1-ranked blocks whose step-1 mass reaches that of the WISE
  working set, with correctly rounded sums; TopK ties go to the lower index.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 32


def default_scale(d: int) -> float:
    """Softmax temperature 1/sqrt(d_h) (WISE paper §3, recurrent attention equation)."""
    return 1.0 / np.sqrt(d)


def _causal_scores(q: np.ndarray, k: np.ndarray, scale: float, rows: slice) -> np.ndarray:
    """Q K^T / sqrt(d_h) + M for query rows ``rows``; M_ij = -inf for j > i (§3)."""
    s = (q[rows] @ k.T) * scale
    i = np.arange(rows.start, rows.stop)[:, None]
    j = np.arange(k.shape[0])[None, :]
    s[j > i] = -np.inf
    return s


def causal_attention(q, k, v, scale=None, chunk: int = 1024):
    """Dense causal attention A = softmax(QK^T/sqrt(d_h) + M), O = A V (WISE paper §3).

    Returns (O [n, d], lse [n]) with lse_i = log sum_j exp(s_ij), the natural-log
    normaliser of row i.  Rows are processed in chunks only to bound memory;
    each row's softmax is the plain definition.
    """
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    n = q.shape[0]
    scale = default_scale(q.shape[1]) if scale is None else float(scale)
    o = np.empty_like(q)
    lse = np.empty(n)
    for r0 in range(0, n, chunk):
        rows = slice(r0, min(n, r0 + chunk))
        s = _causal_scores(q, k, scale, rows)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        o[rows] = (p / l) @ v
        lse[rows] = (m + np.log(l))[:, 0]
    return o, lse


def attention_probs(q, k, scale=None) -> np.ndarray:
    """The full causal attention matrix A (§3), [n, n]; small n only."""
    q, k = np.asarray(q, np.float64), np.asarray(k, np.float64)
    scale = default_scale(q.shape[1]) if scale is None else float(scale)
    s = _causal_scores(q, k, scale, slice(0, q.shape[0]))
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return p / p.sum(axis=1, keepdims=True)


def block_mass(q, k, scale=None, block: int = BLOCK) -> np.ndarray:
    """Block-level attention mass r_qb (WISE paper §5.1, the block-mass equation).

    r_qb = (1/|I_q|) * sum_{i in I_q} sum_{j in I_b} A_ij with blocks of ``block``
    tokens (B = 32 unless a block-size variant of App. C.6 is asked for) and A the
    unrestricted causal softmax of the step.  Returns r [n/B, n/B]; entries with
    b > q are exactly zero (no admissible key there).  Computed one query block at a
    time (the definition is per query block).
    """
    q, k = np.asarray(q, np.float64), np.asarray(k, np.float64)
    n = q.shape[0]
    assert n % block == 0
    nb = n // block
    scale = default_scale(q.shape[1]) if scale is None else float(scale)
    r = np.zeros((nb, nb))
    for qb in range(nb):
        rows = slice(qb * block, (qb + 1) * block)
        s = _causal_scores(q, k, scale, rows)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        a = p / p.sum(axis=1, keepdims=True)                 # rows of A for I_q
        per_block = a.reshape(block, nb, block).sum(axis=2)  # sum over j in I_b
        r[qb] = per_block.sum(axis=0) / block                # mean over i in I_q
    return r


def expand_support(sel: np.ndarray, factor: int) -> np.ndarray:
    """A support chosen on blocks of ``factor`` x 32 tokens, as 32 x 32 blocks.

    The WISE paper runs its larger block sizes as exact 32 x 32 physical subtiles
    (App. C.6, "Block-Size Tradeoff"): query block q (of 32) of coarse block Q = q // factor
    keeps key block b (of 32) iff its coarse block b // factor is in Q's support and
    b <= q (the causal part of the coarse diagonal block).  ``sel`` is the coarse
    [nQ, nQ] boolean support; returns the fine [nQ*factor, nQ*factor] one.
    """
    sel = np.asarray(sel, dtype=bool)
    fine = np.repeat(np.repeat(sel, factor, axis=0), factor, axis=1)
    return fine & np.tril(np.ones_like(fine))


def eta_order(r_row: np.ndarray) -> np.ndarray:
    """Admissible blocks of one query block ranked by mass, descending; ties -> lower index."""
    idx = np.arange(len(r_row))
    return np.array(sorted(idx, key=lambda b: (-r_row[b], b)), dtype=np.int64)


def eta_support(r_row: np.ndarray, eta: float) -> np.ndarray:
    """Cumulative-eta block support B_q^(t,eta) of one query block (WISE paper §3, §6.1).

    ``r_row`` holds r_qb for the admissible blocks b = 0..q only.  Rank blocks by
    mass (descending, ties by lower index) and keep the shortest prefix whose
    cumulative mass is at least eta.  If no prefix reaches eta, keep them all.
    Returns the kept block indices in ascending order.
    """
    r_row = np.asarray(r_row, np.float64)
    order = eta_order(r_row)
    if eta < 1.0:
        c = np.cumsum(r_row[order])
        hit = np.nonzero(c >= eta)[0]
        if len(hit):
            return np.sort(order[: hit[0] + 1])
    return np.arange(len(r_row), dtype=np.int64)


def select(r: np.ndarray, eta: float) -> np.ndarray:
    """Per-step selection for every query block: boolean [nq, nq], True = kept."""
    nq = r.shape[0]
    sel = np.zeros((nq, nq), dtype=bool)
    for qb in range(nq):
        sel[qb, eta_support(r[qb, : qb + 1], eta)] = True
    return sel


def cut_margins(r_row: np.ndarray, eta: float):
    """Distances of one row's eta cut to the boundaries of §6.1's nondegenerate margin.

    Returns (|cumsum_k - eta|, |cumsum_{k-1} - eta|, r_cut) where k is the size of
    the support and r_cut the mass of the last block kept.  A row whose cumulative
    masses or cut mass sit within rounding distance of these boundaries can
    legitimately select differently under another summation order.
    """
    r_row = np.asarray(r_row, np.float64)
    order = eta_order(r_row)
    c = np.cumsum(r_row[order])
    k = len(eta_support(r_row, eta))
    ck = c[k - 1]
    ck1 = c[k - 2] if k >= 2 else 0.0
    return abs(ck - eta), abs(ck1 - eta), r_row[order[k - 1]]


def temporal_union(selections) -> np.ndarray:
    """Working set B_q = union over the discovery window of B_q^(t,eta) (App. B, WISE configuration)."""
    u = None
    for s in selections:
        u = s.copy() if u is None else (u | s)
    return u


def csr_schedule(support: np.ndarray):
    """CSR schedule of one head (App. B, "Sparse-kernel implementation").

    ``support`` is boolean [nq, nq].  Row q lists its active key blocks in
    ascending order; row_offsets has nq + 1 entries.
    """
    nq = support.shape[0]
    row_offsets = np.zeros(nq + 1, np.int64)
    cols = []
    for qb in range(nq):
        active = np.nonzero(support[qb])[0]
        cols.extend(active.tolist())
        row_offsets[qb + 1] = row_offsets[qb] + len(active)
    return row_offsets, np.array(cols, dtype=np.int64)


def support_from_csr(row_offsets, col_idx, nq: int) -> np.ndarray:
    sup = np.zeros((nq, nq), dtype=bool)
    for qb in range(nq):
        sup[qb, np.asarray(col_idx[row_offsets[qb]: row_offsets[qb + 1]], np.int64)] = True
    return sup


def masked_attention(q, k, v, support: np.ndarray, scale=None, chunk: int = 1024,
                     block: int = BLOCK):
    """Attention under the reuse mask R of WISE paper §5.2 plus the causal mask M.

    R_ij = 0 if b(j) is in the support of q(i), else -inf, with blocks of ``block``
    tokens (32, or another size of App. C.6; ``support`` is [n/block, n/block]).
    Returns (O, lse).  Skipping absent blocks (§7.4, App. B) is exactly this masked
    softmax.  A row with no admissible kept key has O = 0 and lse = -inf.
    """
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    n = q.shape[0]
    scale = default_scale(q.shape[1]) if scale is None else float(scale)
    o = np.empty_like(q)
    lse = np.empty(n)
    blk = np.arange(n) // block
    for r0 in range(0, n, chunk):
        rows = slice(r0, min(n, r0 + chunk))
        s = _causal_scores(q, k, scale, rows)
        allowed = support[blk[rows]][:, blk]          # [rows, n]: b(j) in B_q(i)
        s[~allowed] = -np.inf
        m = s.max(axis=1, keepdims=True)
        empty = ~np.isfinite(m[:, 0])                 # no kept admissible key in the row
        m[empty] = 0.0
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        l[empty] = 1.0
        o[rows] = (p / l) @ v
        lse[rows] = np.where(empty, -np.inf, (m + np.log(l))[:, 0])
    return o, lse


def sparse_attention(q, k, v, row_offsets, col_idx, scale=None):
    """Late-step block-sparse attention over a CSR schedule (§5.2, §7.4)."""
    nq = q.shape[0] // BLOCK
    return masked_attention(q, k, v, support_from_csr(row_offsets, col_idx, nq), scale)


def block_density(support: np.ndarray) -> float:
    """Fraction of admissible (causal) query-key blocks retained (App. B, evaluation metrics)."""
    nq = support.shape[0]
    return float(np.tril(support).sum()) / (nq * (nq + 1) / 2)


def retained_mass(r: np.ndarray, support: np.ndarray) -> np.ndarray:
    """Share of one step's unrestricted attention mass that falls inside a support.

    WISE paper App. B, "Evaluation metrics": retained (future) attention mass is the
    fraction of the unrestricted Full-attention mass that lies inside the frozen
    support.  Per query block q this is sum over kept admissible blocks b <= q of
    r_qb (the block mass of that step, §5.1), which is the mean over the rows i of q
    of sum_{j : b(j) kept} A_ij.  Returns [nq]; the mean over query blocks is the
    per-token average, since every block has 32 rows.  Sums are correctly rounded
    (math.fsum), so they do not depend on summation order.
    """
    r = np.asarray(r, np.float64)
    keep = np.tril(np.asarray(support, dtype=bool))
    return np.array([math.fsum(r[qb][keep[qb]]) for qb in range(r.shape[0])])


def static_support(r1: np.ndarray, eta: float = 0.95) -> np.ndarray:
    """Static-95 control (App. B, "Intervention controls"): the cumulative-eta
    support of the FIRST recurrent step alone, S_q = B_q^(1, 0.95)."""
    return select(r1, eta)


def size_matched(r1: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """SizeMatched control (App. B, "Intervention controls"): per query block, the
    K_q admissible blocks of largest step-1 mass, K_q = |W_q| the size of the
    reference (WISE) working set row; TopK ties go to the lower block index."""
    nq = r1.shape[0]
    ref = np.tril(np.asarray(ref, dtype=bool))
    sel = np.zeros((nq, nq), dtype=bool)
    for qb in range(nq):
        k = int(ref[qb].sum())
        sel[qb, eta_order(r1[qb, : qb + 1])[:k]] = True
    return sel


def mass_matched(r1: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """MassMatched control (App. B, "Intervention controls"): m_q = sum over the
    reference (WISE) working set W_q of the step-1 block masses, and the control keeps
    the fewest step-1-ranked blocks (mass descending, ties to the lower index) whose
    step-1 mass reaches m_q: the cumulative-eta support of step 1 at eta = m_q.
    m_q and every prefix sum are correctly rounded (math.fsum), so a prefix holding
    the same blocks as W_q reaches m_q exactly; an empty W_q gives an empty row.
    """
    r1 = np.asarray(r1, np.float64)
    nq = r1.shape[0]
    m = retained_mass(r1, ref)
    sel = np.zeros((nq, nq), dtype=bool)
    for qb in range(nq):
        row = r1[qb, : qb + 1]
        order = eta_order(row)
        k = next((k for k in range(qb + 2) if math.fsum(row[order[:k]]) >= m[qb]), qb + 1)
        sel[qb, order[:k]] = True
    return sel


def head_trajectory(steps, t_d: int, window, eta: float, scale=None, keep_dense_o=True):
    """One head through a WISE trajectory (WISE paper §5, §7.1, App. B).

    ``steps`` yields (t, q, k, v) with [n, d] float64 arrays for t = 1..T.
    Steps t <= t_d use dense causal attention; window steps also select; after
    step t_d the union is frozen into a CSR schedule used for every later step.
    Returns a dict of per-step results.
    """
    out = {"dense_o": {}, "lse": {}, "mass": {}, "sel": {}, "sparse_o": {}}
    sels = []
    sched = None
    for t, q, k, v in steps:
        if t <= t_d:
            o, lse = causal_attention(q, k, v, scale)
            if keep_dense_o:
                out["dense_o"][t] = o
            out["lse"][t] = lse
            if window[0] <= t <= window[1]:
                r = block_mass(q, k, scale)
                s = select(r, eta)
                out["mass"][t] = r
                out["sel"][t] = s
                sels.append(s)
            if t == t_d:
                out["union"] = temporal_union(sels)
                sched = csr_schedule(out["union"])
                out["schedule"] = sched
        else:
            out["sparse_o"][t] = sparse_attention(q, k, v, *sched, scale)[0]
    return out
