"""Shared helpers of the GPU-vs-oracle parity tests (test code, not product code)."""

from __future__ import annotations

import numpy as np

from oracle import wise_oracle as O
from wise_inputs import bf16_bits_to_f64

# Tolerances.
#  * O: max-abs 2e-2 and mean-abs 2e-3 per compared output (bf16 inputs, fp32
#    accumulation), flat, as the workload contract states them.  The output is bf16,
#    so its own rounding already spends up to 2^-6 = 0.0156 where |O| is in [4, 8);
#    the kernel keeps the rest small by normalising with the sum of the bf16 P it
#    multiplies into V.
#  * lse: 2e-3 absolute.  Scores are exact bf16 products summed in fp32 (relative
#    error <= d * 2^-24 of sum |q_c k_c|, ~4e-4 in logit units at the largest logits
#    of these workloads); the row sum of up to 16384 fp32 terms adds <= n * 2^-24
#    relative (1e-3 at n = 16384) -> log error <= ~1.5e-3 in the worst case.
#  * block mass: 1e-4 absolute, the same band inside which the selection is allowed
#    to differ at the eta cut (typical error is ~1e-6).
#  * selections / unions / schedules: bit-exact, except rows whose cut lies within
#    1e-4 (cumulative mass at the cut or one block before it within 1e-4 of eta, or a
#    differing block's mass within 1e-4 of the cut block's mass).
O_MAX, O_MEAN = 2e-2, 2e-3
# every compare_o of the session appends (max-abs, mean-abs); conftest prints the worst
O_OBSERVED: list = []
LSE_TOL = 2e-3
MASS_TOL = 1e-4
CUT_TOL = 1e-4


def bits_to_bool(words: np.ndarray, nq: int) -> np.ndarray:
    """[..., nq, W] int32/uint32 words -> [..., nq, nq] bool (bit b%32 of word b//32)."""
    w = np.ascontiguousarray(words).astype(np.uint32)
    out = np.zeros(w.shape[:-1] + (nq,), dtype=bool)
    for b in range(nq):
        out[..., b] = (w[..., b // 32] >> np.uint32(b % 32)) & np.uint32(1)
    return out


def compare_o(o_gpu: np.ndarray, o_ref: np.ndarray, what: str = "O"):
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    mx, mean = float(err.max()), float(err.mean())
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    assert mx <= O_MAX, f"{what}: max-abs {mx:.3e} > {O_MAX}"
    assert mean <= O_MEAN, f"{what}: mean-abs {mean:.3e} > {O_MEAN}"
    O_OBSERVED.append((mx, mean))
    return mx, mean


def compare_selection(sel_gpu: np.ndarray, r_ref: np.ndarray, eta: float):
    """sel_gpu [nq, nq] bool vs the oracle's selection from fp64 masses r_ref [nq, nq].

    Returns the number of exempt (near-cut) rows; fails on any other mismatch.
    """
    nq = r_ref.shape[0]
    sel_ref = O.select(r_ref, eta)
    exempt = 0
    for qb in range(nq):
        if np.array_equal(sel_gpu[qb], sel_ref[qb]):
            continue
        row = r_ref[qb, : qb + 1]
        d_ck, d_ck1, r_cut = O.cut_margins(row, eta)
        diff = np.nonzero(sel_gpu[qb, : qb + 1] != sel_ref[qb, : qb + 1])[0]
        near = (d_ck <= CUT_TOL or d_ck1 <= CUT_TOL or
                any(abs(row[b] - r_cut) <= CUT_TOL for b in diff))
        assert not sel_gpu[qb, qb + 1:].any(), f"row {qb}: non-causal block selected"
        assert near, (f"row {qb}: selection differs away from the cut "
                      f"(gpu {np.nonzero(sel_gpu[qb])[0].tolist()} vs "
                      f"oracle {np.nonzero(sel_ref[qb])[0].tolist()})")
        exempt += 1
    return exempt


def check_csr(row_offsets: np.ndarray, col_idx: np.ndarray, support: np.ndarray):
    """row_offsets/col_idx of ONE head against a boolean support [nq, nq] (bit-exact)."""
    ro, ci = O.csr_schedule(np.tril(support))
    assert np.array_equal(row_offsets.astype(np.int64), ro)
    assert np.array_equal(col_idx.astype(np.int64), ci)


def head_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f64(bits)


def pool_mass(r: np.ndarray, factor: int) -> np.ndarray:
    """[..., nq, nq] 32-token block masses -> [..., nq/f, nq/f] masses of f x 32-token blocks.

    R_QB = (1/f) sum of r_qb over the f x f fine blocks (q in Q, b in B) with b <= q.
    The oracle pins check this against the block mass computed at the larger size.
    """
    r = np.asarray(r, np.float64)
    nq = r.shape[-1]
    r = r * np.tril(np.ones((nq, nq)))
    nQ = nq // factor
    shp = r.shape[:-2] + (nQ, factor, nQ, factor)
    return r.reshape(shp).sum(axis=(-3, -1)) / factor


def coarse_of_fine(fine: np.ndarray, factor: int) -> np.ndarray:
    """Coarse support read back from an expanded fine one: fine row Q f + f - 1, block B f."""
    return fine[..., factor - 1::factor, ::factor]
