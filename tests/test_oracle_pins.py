"""Pins of the CPU oracle against what the WISE paper and mathematics fix.

None of these compare the oracle with a retyped copy of itself: they use
brute-force scalar loops on tiny inputs, closed forms, a library attention
routine (torch's scaled_dot_product_attention in float64), hand-derived
golden values, exhaustive subset search, and invariants.  A second group
plants plausible mistakes in copies of oracle functions and checks that the
pins catch them.
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import wise_oracle as O
from wise_inputs import CONFIGS, bf16_bits_to_f64, iter_steps

B = 32


def rand_qkv(n, d, seed, scale_q=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n, d)) * scale_q
    k = rng.standard_normal((n, d))
    v = rng.standard_normal((n, d))
    return q, k, v


# --------------------------------------------------------------------------- attention

def brute_attention(q, k, v, scale):
    """Scalar loops: softmax over j <= i, then the weighted sum of value rows."""
    n, d = len(q), len(q[0])
    o, lse = [], []
    for i in range(n):
        logits = []
        for j in range(i + 1):
            acc = 0.0
            for c in range(d):
                acc += q[i][c] * k[j][c]
            logits.append(acc * scale)
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        z = sum(w)
        o.append([sum(w[j] * v[j][c] for j in range(i + 1)) / z for c in range(d)])
        lse.append(mx + math.log(z))
    return np.array(o), np.array(lse)


@pytest.mark.parametrize("n,d,seed", [(1, 3, 0), (5, 3, 1), (9, 4, 2)])
def test_attention_brute_force(n, d, seed):
    q, k, v = rand_qkv(n, d, seed, scale_q=2.0)
    o, lse = O.causal_attention(q, k, v)
    ob, lb = brute_attention(q.tolist(), k.tolist(), v.tolist(), 1 / math.sqrt(d))
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


def test_attention_matches_torch_sdpa_float64():
    torch = pytest.importorskip("torch")
    import torch.nn.functional as F
    q, k, v = rand_qkv(200, 16, 3, scale_q=1.5)
    o, _ = O.causal_attention(q, k, v, chunk=64)
    t = [torch.from_numpy(x)[None, None] for x in (q, k, v)]
    ref = F.scaled_dot_product_attention(*t, is_causal=True)[0, 0].numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_attention_golden_two_tokens(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "attention_two_tokens.json")))
    o, lse = O.causal_attention(np.array(g["q"]), np.array(g["k"]), np.array(g["v"]))
    np.testing.assert_allclose(o, np.array(g["o"]), atol=g["atol"], rtol=0)
    np.testing.assert_allclose(lse, np.array(g["lse"]), atol=g["atol"], rtol=0)


def test_attention_closed_forms():
    n, d = 96, 8
    q, k, v = rand_qkv(n, d, 4)
    # constant values -> output equals that value
    vc = np.tile(np.arange(d, dtype=np.float64), (n, 1))
    o, _ = O.causal_attention(q, k, vc)
    np.testing.assert_allclose(o, vc, atol=1e-12)
    # row 0 sees only key 0
    o, lse = O.causal_attention(q, k, v)
    np.testing.assert_allclose(o[0], v[0], atol=1e-12)
    np.testing.assert_allclose(lse[0], q[0] @ k[0] / math.sqrt(d), atol=1e-12)
    # Q = 0 -> uniform causal average (prefix mean), lse_i = log(i + 1)
    o, lse = O.causal_attention(np.zeros((n, d)), k, v)
    pref = np.cumsum(v, axis=0) / np.arange(1, n + 1)[:, None]
    np.testing.assert_allclose(o, pref, atol=1e-12)
    np.testing.assert_allclose(lse, np.log(np.arange(1, n + 1)), atol=1e-12)


def test_attention_chunking_is_invisible():
    q, k, v = rand_qkv(150, 8, 5)
    o1, l1 = O.causal_attention(q, k, v, chunk=7)
    o2, l2 = O.causal_attention(q, k, v, chunk=1000)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


# --------------------------------------------------------------------------- block mass

def brute_block_mass(q, k, scale):
    n = len(q)
    nq = n // B
    A = [[0.0] * n for _ in range(n)]
    for i in range(n):
        logits = [sum(q[i][c] * k[j][c] for c in range(len(q[0]))) * scale for j in range(i + 1)]
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        z = sum(w)
        for j in range(i + 1):
            A[i][j] = w[j] / z
    r = np.zeros((nq, nq))
    for qb in range(nq):
        for b in range(nq):
            tot = 0.0
            for i in range(qb * B, (qb + 1) * B):
                for j in range(b * B, (b + 1) * B):
                    tot += A[i][j]
            r[qb, b] = tot / B
    return r


def test_block_mass_brute_force():
    q, k, _ = rand_qkv(96, 3, 6, scale_q=2.0)
    r = O.block_mass(q, k)
    rb = brute_block_mass(q.tolist(), k.tolist(), 1 / math.sqrt(3))
    np.testing.assert_allclose(r, rb, atol=1e-13, rtol=0)


def test_block_mass_rows_sum_to_one_and_causal_zero():
    q, k, _ = rand_qkv(256, 16, 7, scale_q=3.0)
    r = O.block_mass(q, k)
    np.testing.assert_allclose(r.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(np.triu(r, 1) == 0.0)
    assert np.all(np.tril(r) >= 0.0)


def test_block_mass_uniform_closed_form():
    """Q = 0: row i spreads 1/(i+1) over keys 0..i, so r_qb = mean_i |I_b cap [0, i]| / (i + 1)."""
    n = 128
    nq = n // B
    _, k, _ = rand_qkv(n, 4, 8)
    r = O.block_mass(np.zeros((n, 4)), k)
    for qb in range(nq):
        for b in range(nq):
            exact = Fraction(0)
            for i in range(qb * B, (qb + 1) * B):
                seen = max(0, min(i, (b + 1) * B - 1) - b * B + 1)
                exact += Fraction(seen, i + 1)
            exact /= B
            assert abs(r[qb, b] - float(exact)) < 1e-14


def test_block_mass_equals_blocks_of_attention_matrix():
    q, k, _ = rand_qkv(160, 8, 9, scale_q=2.0)
    A = O.attention_probs(q, k)
    r = O.block_mass(q, k)
    nq = 5
    for qb in range(nq):
        for b in range(nq):
            assert abs(r[qb, b] - A[qb * B:(qb + 1) * B, b * B:(b + 1) * B].sum() / B) < 1e-13


# --------------------------------------------------------------------------- block-size variants

@pytest.mark.parametrize("block", [16, 64, 128])
def test_block_mass_uniform_closed_form_larger_blocks(block):
    """Q = 0 at B = 16 / 64 / 128: r_QB = mean_i |I_B cap [0, i]| / (i + 1), exact fractions."""
    nb = 3
    n = nb * block
    _, k, _ = rand_qkv(n, 4, 18)
    r = O.block_mass(np.zeros((n, 4)), k, block=block)
    assert r.shape == (nb, nb)
    for qb in range(nb):
        for b in range(nb):
            exact = Fraction(0)
            for i in range(qb * block, (qb + 1) * block):
                seen = max(0, min(i, (b + 1) * block - 1) - b * block + 1)
                exact += Fraction(seen, i + 1)
            exact /= block
            assert abs(r[qb, b] - float(exact)) < 1e-14


@pytest.mark.parametrize("block", [64, 128])
def test_block_mass_larger_blocks_pool_the_attention_matrix(block):
    """Brute force: r_QB is the mean over the B query rows of the attention mass inside I_B."""
    q, k, _ = rand_qkv(2 * block, 8, 19, scale_q=2.5)
    A = O.attention_probs(q, k)
    r = O.block_mass(q, k, block=block)
    np.testing.assert_allclose(r.sum(axis=1), 1.0, atol=1e-12)
    for qb in range(2):
        for b in range(2):
            ref = A[qb * block:(qb + 1) * block, b * block:(b + 1) * block].sum() / block
            assert abs(r[qb, b] - ref) < 1e-13
    assert r[0, 1] == 0.0



@pytest.mark.parametrize("factor", [2, 4])
def test_pooled_fine_mass_is_block_mass_at_larger_size(factor):
    """The identity the GPU selection relies on: pooling 32-token masses gives B = 32f masses."""
    from parity_utils import pool_mass
    q, k, _ = rand_qkv(3 * factor * B, 8, 21, scale_q=2.0)
    r = O.block_mass(q, k)
    np.testing.assert_allclose(pool_mass(r, factor), O.block_mass(q, k, block=B * factor),
                               atol=1e-13, rtol=0)

def test_block_mass_16_pools_to_block_mass_32():
    """Two by two 16-token blocks make one 32-token block: pooling the B = 16 masses
    (factor 2) gives the B = 32 masses."""
    from parity_utils import pool_mass
    q, k, _ = rand_qkv(192, 8, 22, scale_q=2.0)
    np.testing.assert_allclose(pool_mass(O.block_mass(q, k, block=16), 2), O.block_mass(q, k),
                               atol=1e-13, rtol=0)


def test_masked_attention_block16_brute_force():
    """Scalar loops: row i attends j <= i with sel16[i // 16][j // 16]; an empty row gives
    O = 0 and lse = -inf."""
    n, d, scale = 64, 4, 0.5
    q, k, v = rand_qkv(n, d, 23, scale_q=2.0)
    rng = np.random.default_rng(23)
    sel = np.tril(rng.random((4, 4)) < 0.5)
    sel[2] = False                                   # rows 32..47 keep nothing
    o, lse = O.masked_attention(q, k, v, sel, scale, block=16)
    for i in range(n):
        keep = [j for j in range(i + 1) if sel[i // 16][j // 16]]
        if not keep:
            assert np.all(o[i] == 0.0) and lse[i] == -np.inf
            continue
        logits = [scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in keep]
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        z = sum(w)
        ref = [sum(w[t] * v[keep[t]][c] for t in range(len(keep))) / z for c in range(d)]
        np.testing.assert_allclose(o[i], ref, atol=1e-13, rtol=0)
        assert abs(lse[i] - (mx + math.log(z))) < 1e-12


def test_masked_attention_block16_of_an_expanded_support_is_block32():
    """A B = 16 support that keeps 2 x 2 subblocks exactly where a B = 32 support keeps a
    block attends the same keys: identical results."""
    q, k, v = rand_qkv(160, 8, 24, scale_q=2.0)
    rng = np.random.default_rng(24)
    sel32 = np.tril(rng.random((5, 5)) < 0.6)
    np.fill_diagonal(sel32, True)
    sel16 = np.repeat(np.repeat(sel32, 2, axis=0), 2, axis=1)
    o16, l16 = O.masked_attention(q, k, v, sel16, block=16)
    o32, l32 = O.masked_attention(q, k, v, sel32)
    np.testing.assert_allclose(o16, o32, atol=1e-14, rtol=0)
    np.testing.assert_allclose(l16, l32, atol=1e-14, rtol=0)

def _element_mask_coarse(sel, factor, n):
    """Element (i, j) is attended iff j <= i and coarse block (i // 32f, j // 32f) is kept."""
    cb = B * factor
    return [[j <= i and bool(sel[i // cb][j // cb]) for j in range(n)] for i in range(n)]


def _element_mask_fine(fine, n):
    """Element (i, j) is attended iff j <= i and fine 32 x 32 block (i // 32, j // 32) is kept."""
    return [[j <= i and bool(fine[i // B][j // B]) for j in range(n)] for i in range(n)]


@pytest.mark.parametrize("factor", [2, 4])
def test_expand_support_is_the_same_element_mask(factor):
    """Running a coarse support as 32 x 32 subtiles attends exactly the same (i, j) pairs."""
    rng = np.random.default_rng(20 + factor)
    nQ = 3
    n = nQ * factor * B
    for _ in range(4):
        sel = np.tril(rng.random((nQ, nQ)) < 0.6)
        np.fill_diagonal(sel, True)
        fine = O.expand_support(sel, factor)
        assert fine.shape == (nQ * factor, nQ * factor)
        assert _element_mask_fine(fine, n) == _element_mask_coarse(sel, factor, n)


def test_expand_support_is_causal_and_keeps_fine_diagonal():
    sel = np.ones((4, 4), dtype=bool)
    for factor in (1, 2, 4):
        fine = O.expand_support(np.tril(sel), factor)
        assert not np.any(np.triu(fine, 1))
        assert np.all(np.diag(fine))
        # Full coarse support -> every causal fine block, nothing else.
        assert np.array_equal(fine, np.tril(np.ones_like(fine)))
    # factor 1 is the identity on a lower-triangular support.
    s = np.array([[1, 0, 0], [1, 1, 0], [0, 1, 1]], dtype=bool)
    assert np.array_equal(O.expand_support(s, 1), s)


# --------------------------------------------------------------------------- selection

def test_eta_support_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "eta_support_cases.json")))
    for c in g["cases"]:
        got = O.eta_support(np.array(c["r"]), c["eta"]).tolist()
        assert got == c["support"], c["why"]


def brute_min_support(r_row, eta):
    """Exhaustive: smallest subsets reaching eta; return (size, best mass at that size)."""
    m = len(r_row)
    for size in range(1, m + 1):
        best = None
        for sub in itertools.combinations(range(m), size):
            mass = sum(r_row[list(sub)])
            if mass >= eta and (best is None or mass > best):
                best = mass
        if best is not None:
            return size, best
    return m, sum(r_row)


@pytest.mark.parametrize("eta", [0.5, 0.8, 0.9, 0.95, 0.99])
def test_eta_support_is_minimum_cardinality_exhaustive(eta):
    q, k, _ = rand_qkv(256, 8, 10, scale_q=2.5)
    r = O.block_mass(q, k)
    for qb in range(8):
        row = r[qb, : qb + 1]
        sup = O.eta_support(row, eta)
        size, best = brute_min_support(row, eta)
        assert len(sup) == size
        assert abs(row[sup].sum() - best) < 1e-12       # the heaviest set of that size
        assert row[sup].sum() >= eta
        if len(sup) > 1:                                 # minimality
            assert row[sup].sum() - row[sup].min() < eta


def test_selection_retains_eta_on_generator_steps():
    cfg = CONFIGS["tiny"]
    for t, q, k, v in iter_steps(cfg, heads=[(0, 0), (0, 1)], steps=4):
        for h in range(2):
            r = O.block_mass(bf16_bits_to_f64(q[h]), bf16_bits_to_f64(k[h]), cfg.scale)
            sel = O.select(r, cfg.eta)
            for qb in range(cfg.nq):
                assert r[qb][sel[qb]].sum() >= cfg.eta
                assert not sel[qb, qb + 1:].any()


def test_cut_margins_golden():
    a, b, rc = O.cut_margins(np.array([0.5, 0.25, 0.25]), 0.75)
    assert a == 0.0 and b == 0.25 and rc == 0.25


# --------------------------------------------------------------------------- union / schedule

def test_union_and_csr_invariants():
    rng = np.random.default_rng(11)
    nq = 12
    sels = [np.tril(rng.random((nq, nq)) < 0.3) | np.eye(nq, dtype=bool) for _ in range(4)]
    U = O.temporal_union(sels)
    for s in sels:
        assert np.all(U[s])
    assert np.array_equal(U, sels[0] | sels[1] | sels[2] | sels[3])
    ro, ci = O.csr_schedule(U)
    assert ro[0] == 0 and ro[-1] == len(ci) == U.sum()
    assert np.all(np.diff(ro) >= 0)
    for qb in range(nq):
        row = ci[ro[qb]:ro[qb + 1]]
        assert np.all(np.diff(row) > 0) and np.all(row <= qb)
        assert len(row) == U[qb].sum()
    assert np.array_equal(O.support_from_csr(ro, ci, nq), U)



def test_block_density_exact_values():
    """Fraction of the nq(nq+1)/2 causal blocks kept: all causal -> 1, diagonal only ->
    2/(nq+1), blocks above the diagonal never count."""
    nq = 9
    assert O.block_density(np.tril(np.ones((nq, nq), bool))) == 1.0
    assert O.block_density(np.eye(nq, dtype=bool)) == 2.0 / (nq + 1)
    assert O.block_density(np.triu(np.ones((nq, nq), bool), 1)) == 0.0
    sup = np.zeros((nq, nq), bool)
    sup[4, :3] = True
    assert O.block_density(sup | np.triu(np.ones((nq, nq), bool), 1)) == 3 / 45

# --------------------------------------------------------------------------- sparse attention

def test_all_blocks_schedule_equals_dense():
    q, k, v = rand_qkv(192, 8, 12, scale_q=2.0)
    nq = 6
    full = np.tril(np.ones((nq, nq), bool))
    o1, l1 = O.sparse_attention(q, k, v, *O.csr_schedule(full))
    o2, l2 = O.causal_attention(q, k, v)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_diagonal_only_schedule_is_local_attention():
    q, k, v = rand_qkv(96, 4, 13, scale_q=2.0)
    o, _ = O.sparse_attention(q, k, v, *O.csr_schedule(np.eye(3, dtype=bool)))
    for qb in range(3):
        sl = slice(qb * B, (qb + 1) * B)
        ob, _ = brute_attention(q[sl].tolist(), k[sl].tolist(), v[sl].tolist(), 0.5)
        np.testing.assert_allclose(o[sl], ob, atol=1e-12)


def test_sparse_brute_force_with_holes():
    """Scalar loops over only the allowed keys of each row."""
    n, d = 128, 3
    q, k, v = rand_qkv(n, d, 14, scale_q=2.0)
    sup = np.array([[1, 0, 0, 0], [0, 1, 0, 0], [1, 0, 1, 0], [0, 1, 0, 1]], bool)
    o, lse = O.sparse_attention(q, k, v, *O.csr_schedule(sup))
    sc = 1 / math.sqrt(d)
    for i in range(0, n, 7):
        js = [j for j in range(i + 1) if sup[i // B, j // B]]
        lg = [float(q[i] @ k[j]) * sc for j in js]
        mx = max(lg)
        w = [math.exp(x - mx) for x in lg]
        ref = sum(w[a] * v[js[a]] for a in range(len(js))) / sum(w)
        np.testing.assert_allclose(o[i], ref, atol=1e-12)
        assert abs(lse[i] - (mx + math.log(sum(w)))) < 1e-12


def test_permuted_csr_rows_same_output():
    q, k, v = rand_qkv(160, 8, 15)
    rng = np.random.default_rng(0)
    sup = np.tril(rng.random((5, 5)) < 0.5) | np.eye(5, dtype=bool)
    ro, ci = O.csr_schedule(sup)
    ci2 = ci.copy()
    for qb in range(5):
        rng.shuffle(ci2[ro[qb]:ro[qb + 1]])
    o1, _ = O.sparse_attention(q, k, v, ro, ci)
    o2, _ = O.sparse_attention(q, k, v, ro, ci2)
    np.testing.assert_allclose(o1, o2, atol=1e-14)


def test_tiny_trajectory_eta_one_sparse_equals_dense():
    cfg = CONFIGS["tiny"]
    steps = [(t, *(bf16_bits_to_f64(x[0]) for x in (q, k, v)))
             for t, q, k, v in iter_steps(cfg, heads=[(0, 1)])]
    res = O.head_trajectory(steps, cfg.t_d, cfg.window, eta=1.0, scale=cfg.scale)
    assert res["union"].sum() == cfg.nq * (cfg.nq + 1) // 2
    for t, q, k, v in steps[cfg.t_d:]:
        dense, _ = O.causal_attention(q, k, v, cfg.scale)
        np.testing.assert_allclose(res["sparse_o"][t], dense, atol=1e-12)


def test_tiny_trajectory_structure():
    cfg = CONFIGS["tiny"]
    steps = [(t, *(bf16_bits_to_f64(x[0]) for x in (q, k, v)))
             for t, q, k, v in iter_steps(cfg, heads=[(0, 0)])]
    res = O.head_trajectory(steps, cfg.t_d, cfg.window, eta=cfg.eta, scale=cfg.scale)
    assert sorted(res["sel"]) == [3, 4]
    assert sorted(res["sparse_o"]) == [5, 6, 7, 8]
    U = res["union"]
    assert np.array_equal(U, res["sel"][3] | res["sel"][4])
    assert np.all(np.diag(U) | U.any(axis=1))
    assert 0 < O.block_density(U) <= 1



# --------------------------------------------------------------------------- controls and retained mass

def test_retained_mass_brute_force():
    """Retained mass of a support = mean over the rows of each query block of the attention
    probability that falls on kept key blocks (scalar loops on a tiny case)."""
    q, k, _ = rand_qkv(128, 3, 30, scale_q=2.0)
    nq, scale = 4, 1 / math.sqrt(3)
    rng = np.random.default_rng(30)
    sup = rng.random((nq, nq)) < 0.5
    ql, kl = q.tolist(), k.tolist()
    want = []
    for qb in range(nq):
        tot = 0.0
        for i in range(qb * B, (qb + 1) * B):
            logits = [sum(ql[i][c] * kl[j][c] for c in range(3)) * scale for j in range(i + 1)]
            mx = max(logits)
            w = [math.exp(x - mx) for x in logits]
            z = sum(w)
            tot += sum(w[j] for j in range(i + 1) if sup[qb][j // B]) / z
        want.append(tot / B)
    got = O.retained_mass(O.block_mass(q, k), sup)
    np.testing.assert_allclose(got, want, atol=1e-13, rtol=0)


def test_retained_mass_special_supports():
    q, k, _ = rand_qkv(256, 16, 31, scale_q=2.5)
    r = O.block_mass(q, k)
    nq = 8
    np.testing.assert_allclose(O.retained_mass(r, np.ones((nq, nq), bool)), 1.0, atol=1e-12)
    assert np.all(O.retained_mass(r, np.zeros((nq, nq), bool)) == 0.0)
    assert np.all(O.retained_mass(r, O.select(r, 0.9)) >= 0.9)
    # blocks above the diagonal carry no mass and are ignored even if set
    assert np.array_equal(O.retained_mass(r, np.triu(np.ones((nq, nq), bool), 1)), np.zeros(nq))


def _softmax_rows(rng, nq, temp=2.5):
    r = np.zeros((nq, nq))
    for qb in range(nq):
        lg = rng.standard_normal(qb + 1) * temp
        p = np.exp(lg - lg.max())
        r[qb, : qb + 1] = p / p.sum()
    return r


def test_size_matched_is_heaviest_k_subset_exhaustive():
    """TopK: the K_q-subset of admissible blocks with the largest step-1 mass (distinct masses:
    unique), K_q = |W_q| exactly, for random reference rows."""
    rng = np.random.default_rng(32)
    nq = 8
    r1 = _softmax_rows(rng, nq)
    ref = np.tril(rng.random((nq, nq)) < 0.45)
    sel = O.size_matched(r1, ref)
    for qb in range(nq):
        kq = int(ref[qb].sum())
        assert sel[qb].sum() == kq and not sel[qb, qb + 1:].any()
        best = max((sum(r1[qb, list(c)]) for c in itertools.combinations(range(qb + 1), kq)),
                   default=0.0)
        assert abs(r1[qb][sel[qb]].sum() - best) < 1e-12


def test_size_matched_golden_ties():
    """Hand-worked: masses (0.25, 0.25, 0.5), K = 2 -> {0, 2} (the tie goes to the lower
    index); K = 0 -> nothing; K = 3 -> everything."""
    r1 = np.array([[1.0, 0, 0], [0.5, 0.5, 0], [0.25, 0.25, 0.5]])
    for k, want in ((2, [0, 2]), (0, []), (3, [0, 1, 2]), (1, [2])):
        ref = np.zeros((3, 3), bool)
        ref[2, :k] = True
        assert np.nonzero(O.size_matched(r1, ref)[2])[0].tolist() == want


def test_mass_matched_is_min_cardinality_reaching_wise_mass_exhaustive():
    """The fewest blocks whose step-1 mass reaches m_q = step-1 mass of W_q; never more blocks
    than W_q itself (W_q is one such set)."""
    rng = np.random.default_rng(33)
    nq = 8
    r1 = _softmax_rows(rng, nq)
    ref = np.tril(rng.random((nq, nq)) < 0.5)
    np.fill_diagonal(ref, True)
    sel = O.mass_matched(r1, ref)
    for qb in range(nq):
        row = r1[qb, : qb + 1]
        m = math.fsum(row[ref[qb, : qb + 1]])
        size, best = brute_min_support(row, m)
        assert sel[qb].sum() == size <= ref[qb].sum()
        assert abs(row[sel[qb, : qb + 1]].sum() - best) < 1e-12
        assert math.fsum(row[sel[qb, : qb + 1]]) >= m


def test_mass_matched_reproduces_a_ranking_prefix():
    """If W_q is itself the eta-support of step 1, MassMatched gives back exactly W_q (its
    mass is reached by the same prefix; no extra block from rounding)."""
    q, k, _ = rand_qkv(512, 16, 34, scale_q=3.0)
    r1 = O.block_mass(q, k)
    for eta in (0.5, 0.9, 0.95, 0.99):
        w = O.select(r1, eta)
        assert np.array_equal(O.mass_matched(r1, w), w)
        assert np.array_equal(O.size_matched(r1, w), w)


def test_mass_matched_golden():
    """Hand-worked: step-1 masses (0.1, 0.2, 0.3, 0.4); W = {0, 1} holds 0.3 of it; the fewest
    blocks reaching 0.3 are {3} (0.4).  W = {0, 1, 2} holds 0.6 -> {2, 3} (0.7).  Empty W -> {}."""
    r1 = np.zeros((4, 4))
    r1[3] = [0.1, 0.2, 0.3, 0.4]
    r1[:3] = np.tril(np.ones((3, 4))) / np.arange(1, 4)[:, None]
    for w_row, want in (([0, 1], [3]), ([0, 1, 2], [2, 3]), ([], []), ([3], [3])):
        ref = np.zeros((4, 4), bool)
        ref[3, w_row] = True
        assert np.nonzero(O.mass_matched(r1, ref)[3])[0].tolist() == want


def test_static_support_is_a_one_step_window():
    """Static-95 is the union over the window {1}: the trajectory with window (1, 1)."""
    cfg = CONFIGS["tiny"]
    heads = [(0, 0)]
    steps = [(t, *(bf16_bits_to_f64(x[0]) for x in (q, k, v)))
             for t, q, k, v in iter_steps(cfg, heads=heads, steps=cfg.t_d)]
    out = O.head_trajectory(steps, cfg.t_d, (1, 1), 0.95, cfg.scale, keep_dense_o=False)
    t1, q1, k1, _ = steps[0]
    assert np.array_equal(out["union"], O.static_support(O.block_mass(q1, k1, cfg.scale)))


# --------------------------------------------------------------------------- planted mistakes

def _mutant_attention_no_scale(q, k, v, scale=None, chunk=1024):
    return O.causal_attention(q, k, v, scale=1.0, chunk=chunk)


def _mutant_attention_diag_masked(q, k, v, scale=None, chunk=1024):
    n = q.shape[0]
    o = np.zeros_like(q)
    lse = np.zeros(n)
    s = (q @ k.T) / math.sqrt(q.shape[1])
    s[np.arange(n)[None, :] >= np.arange(n)[:, None]] = -np.inf
    s[0, 0] = 0.0
    p = np.exp(s - s.max(1, keepdims=True))
    o[:] = (p / p.sum(1, keepdims=True)) @ v
    return o, lse


def _mutant_mass_transposed(q, k, scale=None):
    return O.block_mass(q, k, scale).T


def _mutant_support_strict(r_row, eta):
    order = O.eta_order(r_row)
    c = np.cumsum(np.asarray(r_row)[order])
    hit = np.nonzero(c > eta)[0]
    return np.sort(order[: hit[0] + 1]) if len(hit) else np.arange(len(r_row))


def _mutant_support_high_index_ties(r_row, eta):
    idx = np.arange(len(r_row))
    order = np.array(sorted(idx, key=lambda b: (-r_row[b], -b)))
    c = np.cumsum(np.asarray(r_row)[order])
    hit = np.nonzero(c >= eta)[0]
    return np.sort(order[: hit[0] + 1]) if len(hit) else idx


def test_pins_catch_planted_attention_mistakes():
    q, k, v = rand_qkv(9, 4, 2, scale_q=2.0)
    ob, _ = brute_attention(q.tolist(), k.tolist(), v.tolist(), 0.5)
    for mutant in (_mutant_attention_no_scale, _mutant_attention_diag_masked):
        o, _ = mutant(q, k, v)
        assert np.max(np.abs(o - ob)) > 1e-6


def test_pins_catch_planted_mass_mistake():
    q, k, _ = rand_qkv(256, 16, 7, scale_q=3.0)
    r = _mutant_mass_transposed(q, k)
    assert not np.allclose(r.sum(axis=1), 1.0, atol=1e-6)


def test_pins_catch_planted_selection_mistakes(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "eta_support_cases.json")))
    for mutant in (_mutant_support_strict, _mutant_support_high_index_ties):
        wrong = [c for c in g["cases"]
                 if mutant(np.array(c["r"]), c["eta"]).tolist() != c["support"]]
        assert wrong, mutant.__name__


def _mutant_expand_no_causal_clip(sel, factor):
    sel = np.asarray(sel, dtype=bool)
    return np.repeat(np.repeat(sel, factor, axis=0), factor, axis=1)


def _mutant_expand_transposed(sel, factor):
    sel = np.asarray(sel, dtype=bool).T
    fine = np.repeat(np.repeat(sel, factor, axis=0), factor, axis=1)
    return fine & np.tril(np.ones_like(fine))


def test_pins_catch_planted_expansion_mistakes():
    """Dropping the causal clip leaves future fine blocks; transposing keeps the wrong ones."""
    sel = np.array([[1, 0, 0], [1, 1, 0], [0, 1, 1]], dtype=bool)
    factor, n = 2, 3 * 2 * B
    want = _element_mask_coarse(sel, factor, n)
    assert np.any(np.triu(_mutant_expand_no_causal_clip(sel, factor), 1))
    assert _element_mask_fine(_mutant_expand_transposed(sel, factor), n) != want


def _mutant_size_matched_high_ties(r1, ref):
    nq = r1.shape[0]
    sel = np.zeros((nq, nq), dtype=bool)
    for qb in range(nq):
        k = int(np.tril(ref)[qb].sum())
        order = sorted(range(qb + 1), key=lambda b: (-r1[qb, b], -b))
        sel[qb, order[:k]] = True
    return sel


def _mutant_mass_matched_strict(r1, ref):
    nq = r1.shape[0]
    sel = np.zeros((nq, nq), dtype=bool)
    m = O.retained_mass(r1, ref)
    for qb in range(nq):
        row = r1[qb, : qb + 1]
        order = O.eta_order(row)
        k = next((k for k in range(qb + 2) if math.fsum(row[order[:k]]) > m[qb]), qb + 1)
        sel[qb, order[:k]] = True
    return sel


def test_pins_catch_planted_control_mistakes():
    r1 = np.array([[1.0, 0, 0], [0.5, 0.5, 0], [0.25, 0.25, 0.5]])
    ref = np.zeros((3, 3), bool)
    ref[2, :2] = True
    assert np.nonzero(_mutant_size_matched_high_ties(r1, ref)[2])[0].tolist() != [0, 2]
    q, k, _ = rand_qkv(512, 16, 34, scale_q=3.0)
    r = O.block_mass(q, k)
    w = O.select(r, 0.9)
    assert not np.array_equal(_mutant_mass_matched_strict(r, w), w)
