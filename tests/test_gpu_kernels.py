"""GPU-vs-oracle parity of each C-ABI entry point on seeded random inputs.

Sizes span several 128-row tiles, ragged tails (seqlen not a multiple of 128,
a single 32-token block), every supported head_dim and batch*heads > 1.
"""

import math

import numpy as np
import pytest

from oracle import wise_oracle as O
from parity_utils import (LSE_TOL, MASS_TOL, bits_to_bool, check_csr, coarse_of_fine, compare_o,
                          compare_selection, pool_mass)
from wise_inputs import bf16_bits_to_f64, f32_to_bf16_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ops():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from recurrent_depth_lm_b200 import ops as _ops
    return _ops


def rand_qkv_bits(b, h, n, d, seed, qscale=2.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((b, h, n, d), dtype=np.float32) * np.float32(qscale)
    k = rng.standard_normal((b, h, n, d), dtype=np.float32)
    v = rng.standard_normal((b, h, n, d), dtype=np.float32)
    return [f32_to_bf16_bits(x) for x in (q, k, v)]


def to_dev(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def dev_f32(t):
    return t.float().cpu().numpy()


SHAPES = [(1, 2, 256, 64), (1, 1, 32, 128), (2, 3, 160, 96), (1, 2, 544, 128), (1, 1, 1024, 96)]


@pytest.mark.parametrize("one_pass", [True, False])
@pytest.mark.parametrize("b,h,n,d", SHAPES)
def test_dense_attention_lse_and_mass(ops, b, h, n, d, one_pass):
    """Both block-mass paths: one pass (per-block log-sum-exps recorded by the
    attention kernel) and two passes (Q K^T recomputed with the final lse)."""
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=n + d)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    o, lse, mass = ops.full_attn_mass(q, k, v, with_mass=True, one_pass=one_pass)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    o, lse, mass = dev_f32(o), lse.cpu().numpy(), mass.cpu().numpy()
    for bi in range(b):
        for hi in range(h):
            qf, kf, vf = (bf16_bits_to_f64(x[bi, hi]) for x in (qb, kb, vb))
            o_ref, lse_ref = O.causal_attention(qf, kf, vf)
            compare_o(o[bi, hi], o_ref, f"O[{bi},{hi}]")
            assert np.abs(lse[bi, hi] - lse_ref).max() <= LSE_TOL
            r_ref = O.block_mass(qf, kf)
            m = np.tril(mass[bi, hi])
            assert np.abs(m - r_ref).max() <= MASS_TOL


def test_dense_without_lse(ops):
    qb, kb, vb = rand_qkv_bits(1, 2, 96, 64, seed=5)
    o, lse, mass = ops.full_attn_mass(to_dev(qb), to_dev(kb), to_dev(vb))
    assert lse is None and mass is None
    o = dev_f32(o)
    for hi in range(2):
        o_ref, _ = O.causal_attention(*(bf16_bits_to_f64(x[0, hi]) for x in (qb, kb, vb)))
        compare_o(o[0, hi], o_ref)


# More tiles than 2 x 148 tile slots: every CTA cycles both of its tile slots through
# several query tiles (tile switches, slot end markers, uneven slot progress).
MANY_TILES = [(2, 160, 256, 64), (1, 80, 512, 128), (1, 100, 384, 96)]


@pytest.mark.parametrize("b,h,n,d", MANY_TILES)
def test_dense_many_tiles_per_cta(ops, b, h, n, d):
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=3 * n + d)
    o, lse, mass = ops.full_attn_mass(to_dev(qb), to_dev(kb), to_dev(vb), with_mass=True)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    o, lse, mass = dev_f32(o), lse.cpu().numpy(), mass.cpu().numpy()
    for bi in range(b):
        for hi in range(h):
            qf, kf, vf = (bf16_bits_to_f64(x[bi, hi]) for x in (qb, kb, vb))
            o_ref, lse_ref = O.causal_attention(qf, kf, vf)
            compare_o(o[bi, hi], o_ref, f"O[{bi},{hi}]")
            assert np.abs(lse[bi, hi] - lse_ref).max() <= LSE_TOL
            if hi % 16 == 0:
                assert np.abs(np.tril(mass[bi, hi]) - O.block_mass(qf, kf)).max() <= MASS_TOL


# Grouped-query attention: K/V carry fewer heads; query head h reads K/V head h // (H // H_kv).
GQA_SHAPES = [(1, 8, 512, 128, 2), (2, 6, 256, 64, 3), (1, 32, 1024, 128, 8), (1, 4, 544, 96, 1)]


@pytest.mark.parametrize("b,h,n,d,hkv", GQA_SHAPES)
def test_gqa_dense_mass_and_sparse(ops, b, h, n, d, hkv):
    g = h // hkv
    nq = n // 32
    qb, _, _ = rand_qkv_bits(b, h, n, d, seed=11 * n + h)
    _, kb, vb = rand_qkv_bits(b, hkv, n, d, seed=13 * n + hkv)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    o, lse, mass = ops.full_attn_mass(q, k, v, with_mass=True)
    rng = np.random.default_rng(n + h)
    sups = [random_support(nq, rng, p=0.35) for _ in range(b * h)]
    ro, ci, nnz = csr_device(sups)
    o_s, _ = ops.sparse_attn(q, k, v, ro, ci, nnz)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    o, lse, mass, o_s = dev_f32(o), lse.cpu().numpy(), mass.cpu().numpy(), dev_f32(o_s)
    for bi in range(b):
        for hi in range(h):
            qf = bf16_bits_to_f64(qb[bi, hi])
            kf, vf = (bf16_bits_to_f64(x[bi, hi // g]) for x in (kb, vb))
            o_ref, lse_ref = O.causal_attention(qf, kf, vf)
            compare_o(o[bi, hi], o_ref, f"O[{bi},{hi}]")
            assert np.abs(lse[bi, hi] - lse_ref).max() <= LSE_TOL
            assert np.abs(np.tril(mass[bi, hi]) - O.block_mass(qf, kf)).max() <= MASS_TOL
            os_ref, _ = O.masked_attention(qf, kf, vf, sups[bi * h + hi])
            compare_o(o_s[bi, hi], os_ref, f"sparse O[{bi},{hi}]")


def random_support(nq, rng, p=0.4, diag=True, empty_rows=()):
    s = np.tril(rng.random((nq, nq)) < p)
    if diag:
        s |= np.eye(nq, dtype=bool)
    for r in empty_rows:
        s[r] = False
    return s


def csr_device(supports):
    """supports [BH][nq, nq] bool -> device row_offsets, col_idx (concatenated heads)."""
    ros, cis, base = [0], [], 0
    for s in supports:
        ro, ci = O.csr_schedule(s)
        ros.extend((ro[1:] + base).tolist())
        cis.extend(ci.tolist())
        base += len(ci)
    ro = torch.tensor(ros, dtype=torch.int32, device="cuda")
    ci = torch.tensor(cis if cis else [0], dtype=torch.int32, device="cuda")
    return ro, ci, base


@pytest.mark.parametrize("b,h,n,d", SHAPES)
def test_sparse_attention_random_schedule(ops, b, h, n, d):
    nq = n // 32
    rng = np.random.default_rng(100 + n)
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=7 * n + d)
    sups = [random_support(nq, rng, p=0.3) for _ in range(b * h)]
    ro, ci, nnz = csr_device(sups)
    lse = torch.empty(b, h, n, dtype=torch.float32, device="cuda")
    o, _ = ops.sparse_attn(to_dev(qb), to_dev(kb), to_dev(vb), ro, ci, nnz, lse=lse)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    o, lse = dev_f32(o), lse.cpu().numpy()
    for bi in range(b):
        for hi in range(h):
            qf, kf, vf = (bf16_bits_to_f64(x[bi, hi]) for x in (qb, kb, vb))
            o_ref, lse_ref = O.masked_attention(qf, kf, vf, sups[bi * h + hi])
            compare_o(o[bi, hi], o_ref, f"sparse O[{bi},{hi}]")
            assert np.abs(lse[bi, hi] - lse_ref).max() <= LSE_TOL


@pytest.mark.parametrize("b,h,n,d", MANY_TILES)
def test_sparse_many_tiles_per_cta(ops, b, h, n, d):
    nq = n // 32
    rng = np.random.default_rng(7 + n)
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=5 * n + d)
    sups = [random_support(nq, rng, p=rng.uniform(0.1, 0.9), empty_rows=(1,) if i % 7 == 0 else ())
            for i in range(b * h)]
    ro, ci, nnz = csr_device(sups)
    o, _ = ops.sparse_attn(to_dev(qb), to_dev(kb), to_dev(vb), ro, ci, nnz)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    o = dev_f32(o)
    for bi in range(b):
        for hi in range(h):
            sup = sups[bi * h + hi]
            qf, kf, vf = (bf16_bits_to_f64(x[bi, hi]) for x in (qb, kb, vb))
            o_ref, _ = O.masked_attention(qf, kf, vf, sup)
            rows = np.repeat(sup.any(axis=1), 32)
            compare_o(o[bi, hi][rows], o_ref[rows], f"sparse O[{bi},{hi}]")
            assert np.all(o[bi, hi][~rows] == 0.0)


def test_sparse_all_blocks_equals_dense(ops):
    b, h, n, d = 1, 2, 512, 128
    nq = n // 32
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=11)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    full = np.tril(np.ones((nq, nq), dtype=bool))
    ro, ci, nnz = csr_device([full] * (b * h))
    o_s, _ = ops.sparse_attn(q, k, v, ro, ci, nnz)
    o_d, _, _ = ops.full_attn_mass(q, k, v)
    torch.cuda.synchronize()
    # same kernel pipeline and block order; the dense kernel adds each block's row sum by
    # 16-column halves (for the 16-token masses), so the two may differ by the rounding of
    # that fp32 sum: at most one bf16 step of the output
    od = dev_f32(o_d)
    assert np.all(np.abs(dev_f32(o_s) - od) <= np.abs(od) * 2.0 ** -8 + 1e-30)
    o_ref, _ = O.causal_attention(*(bf16_bits_to_f64(x[0, 1]) for x in (qb, kb, vb)))
    compare_o(dev_f32(o_s)[0, 1], o_ref)


def test_sparse_diagonal_only_and_empty_rows(ops):
    b, h, n, d = 1, 1, 256, 64
    nq = n // 32
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=12)
    sup = np.eye(nq, dtype=bool)
    sup[3] = False      # an empty schedule row: O = 0, lse = -inf
    sup[5, 0] = True
    ro, ci, nnz = csr_device([sup])
    lse = torch.empty(b, h, n, dtype=torch.float32, device="cuda")
    o, _ = ops.sparse_attn(to_dev(qb), to_dev(kb), to_dev(vb), ro, ci, nnz, lse=lse)
    torch.cuda.synchronize()
    o, lse = dev_f32(o)[0, 0], lse.cpu().numpy()[0, 0]
    qf, kf, vf = (bf16_bits_to_f64(x[0, 0]) for x in (qb, kb, vb))
    rows = np.ones(n, dtype=bool)
    rows[96:128] = False
    o_ref, lse_ref = O.masked_attention(qf, kf, vf, sup)
    compare_o(o[rows], o_ref[rows])
    assert np.all(o[96:128] == 0.0) and np.all(np.isneginf(lse[96:128]))
    assert np.abs(lse[rows] - lse_ref[rows]).max() <= LSE_TOL


def test_sparse_bad_schedule_entries_are_skipped(ops):
    """Entries above the diagonal or out of range are ignored and flagged, never read."""
    b, h, n, d = 1, 1, 128, 64
    nq = n // 32
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=13)
    sup = np.tril(np.ones((nq, nq), dtype=bool))
    ro, ci, nnz = csr_device([sup])
    ci_h = ci.cpu().numpy()
    ro_h = ro.cpu().numpy()
    bad = ci_h.copy()
    bad[ro_h[1]] = 3          # row 1 gets block 3 (> 1) instead of block 0
    bad[ro_h[2]] = 1000       # row 2 gets an out-of-range block instead of block 0
    ops.device_status(clear=True)
    o, _ = ops.sparse_attn(to_dev(qb), to_dev(kb), to_dev(vb), ro,
                           torch.tensor(bad, dtype=torch.int32, device="cuda"), nnz)
    st = ops.device_status(clear=True)
    assert st & 0x2
    o = dev_f32(o)[0, 0]
    eff = sup.copy()
    eff[1, 0] = False
    eff[2, 0] = False
    o_ref, _ = O.masked_attention(*(bf16_bits_to_f64(x[0, 0]) for x in (qb, kb, vb)), eff)
    compare_o(o, o_ref)


def test_sparse_bad_row_offsets_are_empty_rows(ops):
    """A row whose offsets are not ascending within [0, col_count] is empty and flagged;
    its neighbour, whose range then covers foreign entries, keeps only entries <= q."""
    b, h, n, d = 1, 1, 256, 64
    nq = n // 32
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=17)
    sup = np.tril(np.ones((nq, nq), dtype=bool))
    ro, ci, nnz = csr_device([sup])
    ro_h = ro.cpu().numpy().copy()
    ci_h = ci.cpu().numpy()
    ro_h[4] = ro_h[5] + 3          # row 4 ends before it begins; row 3 now spans into row 4's entries
    expect = np.zeros_like(sup)
    for r in range(nq):
        beg, end = int(ro_h[r]), int(ro_h[r + 1])
        if beg < 0 or end < beg or end > nnz:
            continue
        for e in range(beg, end):
            if 0 <= ci_h[e] <= r:
                expect[r, ci_h[e]] = True
    assert not expect[4].any() and expect[3].sum() == 4
    ops.device_status(clear=True)
    o, _ = ops.sparse_attn(to_dev(qb), to_dev(kb), to_dev(vb),
                           torch.tensor(ro_h, dtype=torch.int32, device="cuda"), ci, nnz)
    st = ops.device_status(clear=True)
    assert st & 0x2
    o = dev_f32(o)[0, 0]
    o_ref, _ = O.masked_attention(*(bf16_bits_to_f64(x[0, 0]) for x in (qb, kb, vb)), expect)
    rows = np.repeat(expect.any(axis=1), 32)       # the empty row 4 has no softmax: O = 0
    compare_o(o[rows], o_ref[rows])
    assert np.all(o[~rows] == 0.0)


@pytest.mark.parametrize("nq,bh", [(8, 2), (37, 3), (128, 2), (512, 1)])
def test_select_union_matches_oracle(ops, nq, bh):
    rng = np.random.default_rng(nq)
    eta = 0.95
    # masses from real softmax rows: peaky logits over admissible blocks
    masses = np.zeros((bh, nq, nq))
    for x in range(bh):
        for q in range(nq):
            lg = rng.standard_normal(q + 1) * 2.5
            p = np.exp(lg - lg.max())
            masses[x, q, : q + 1] = p / p.sum()
    m32 = masses.astype(np.float32)
    mass = torch.from_numpy(m32).reshape(1, bh, nq, nq).cuda()
    union = ops.new_bitmask(1, bh, nq, "cuda")
    step = torch.empty_like(union)
    ops.select_union(mass, union, eta, step_bits=step)
    # union accumulates: a second, different step ORs in
    m2 = np.roll(m32, 1, axis=2) * np.tril(np.ones((nq, nq), np.float32))
    m2 /= np.maximum(m2.sum(axis=2, keepdims=True), 1e-30)
    step2 = torch.empty_like(union)
    ops.select_union(torch.from_numpy(m2).reshape(1, bh, nq, nq).cuda(), union, eta,
                     step_bits=step2)
    torch.cuda.synchronize()
    s1 = bits_to_bool(step.cpu().numpy()[0], nq)
    s2 = bits_to_bool(step2.cpu().numpy()[0], nq)
    u = bits_to_bool(union.cpu().numpy()[0], nq)
    assert np.array_equal(u, s1 | s2)
    for x in range(bh):
        compare_selection(s1[x], m32[x].astype(np.float64), eta)
        compare_selection(s2[x], m2[x].astype(np.float64), eta)
        for q in range(nq):   # retained mass reaches eta
            assert m32[x, q][s1[x, q]].astype(np.float64).sum() >= eta - 1e-6


def test_select_eta_one_keeps_everything(ops):
    nq, bh = 40, 2
    m = np.tril(np.full((bh, nq, nq), 1.0 / nq, np.float32))
    union = ops.new_bitmask(1, bh, nq, "cuda")
    ops.select_union(torch.from_numpy(m).reshape(1, bh, nq, nq).cuda(), union, 1.0)
    u = bits_to_bool(union.cpu().numpy()[0], nq)
    assert np.array_equal(u, np.broadcast_to(np.tril(np.ones((nq, nq), bool)), u.shape))


def test_select_golden_ties_and_exact_cut(ops):
    """The hand-worked cases of tests/golden/eta_support_cases.json through the kernel."""
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "eta_support_cases.json")))
    for c in g["cases"]:
        r = np.array(c["r"], np.float32)
        nq = len(r)
        m = np.zeros((nq, nq), np.float32)
        m[nq - 1, :] = r           # the case is the last query block's row
        m[: nq - 1] = np.tril(np.ones((nq - 1, nq), np.float32)) / np.arange(1, nq)[:, None]
        union = ops.new_bitmask(1, 1, nq, "cuda")
        ops.select_union(torch.from_numpy(m).reshape(1, 1, nq, nq).cuda(), union, c["eta"])
        u = bits_to_bool(union.cpu().numpy()[0, 0], nq)
        assert np.nonzero(u[nq - 1])[0].tolist() == c["support"], c["why"]



def _peaky_masses(rng, bh, nq):
    masses = np.zeros((bh, nq, nq))
    for x in range(bh):
        for q in range(nq):
            lg = rng.standard_normal(q + 1) * 2.5
            p = np.exp(lg - lg.max())
            masses[x, q, : q + 1] = p / p.sum()
    return masses


def _check_blocks_selection(sel_fine, m_fine, f, eta):
    """Fine support of one head: exactly the expansion of a coarse support, and that coarse
    support is the oracle's selection on the pooled masses (near-cut rows exempt)."""
    coarse = coarse_of_fine(sel_fine, f)
    assert np.array_equal(sel_fine, O.expand_support(coarse, f))
    R = pool_mass(np.tril(m_fine), f)
    exempt = compare_selection(coarse, R, eta)
    for Q in range(R.shape[0]):   # a row whose total is below eta keeps everything
        assert R[Q][coarse[Q]].sum() >= min(eta, R[Q, : Q + 1].sum()) - 1e-6
    return exempt


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("nq,bh", [(8, 2), (40, 3), (128, 2), (512, 1)])
def test_select_union_blocks_matches_oracle(ops, block, nq, bh):
    """Block-size variant: selection on 64 / 128-token blocks, written as 32 x 32 subtiles."""
    f = block // 32
    rng = np.random.default_rng(nq * 5 + f)
    eta = 0.95
    m32 = _peaky_masses(rng, bh, nq).astype(np.float32)
    garbage = m32.copy()
    garbage[:, np.triu_indices(nq, 1)[0], np.triu_indices(nq, 1)[1]] = np.nan  # b > q: not read
    union = ops.new_bitmask(1, bh, nq, "cuda")
    step = torch.empty_like(union)
    ops.select_union(torch.from_numpy(garbage).reshape(1, bh, nq, nq).cuda(), union, eta,
                     step_bits=step, block=block)
    m2 = np.roll(m32, 1, axis=2) * np.tril(np.ones((nq, nq), np.float32))
    m2 /= np.maximum(m2.sum(axis=2, keepdims=True), 1e-30)
    step2 = torch.empty_like(union)
    ops.select_union(torch.from_numpy(m2).reshape(1, bh, nq, nq).cuda(), union, eta,
                     step_bits=step2, block=block)
    torch.cuda.synchronize()
    s1 = bits_to_bool(step.cpu().numpy()[0], nq)
    s2 = bits_to_bool(step2.cpu().numpy()[0], nq)
    u = bits_to_bool(union.cpu().numpy()[0], nq)
    assert np.array_equal(u, s1 | s2)
    exempt = 0
    for x in range(bh):
        exempt += _check_blocks_selection(s1[x], m32[x].astype(np.float64), f, eta)
        exempt += _check_blocks_selection(s2[x], m2[x].astype(np.float64), f, eta)
    assert exempt <= 2


@pytest.mark.parametrize("block", [64, 128])
def test_select_union_blocks_real_masses(ops, block):
    """Fine masses of a real causal softmax; the reference is the oracle's block mass computed
    directly at the larger block size (not pooled)."""
    f = block // 32
    n, d, eta = 1280, 16, 0.9
    rng = np.random.default_rng(block)
    q = rng.standard_normal((n, d)) * 2.0
    k = rng.standard_normal((n, d))
    r32 = O.block_mass(q, k).astype(np.float32)
    nq = n // 32
    union = ops.new_bitmask(1, 1, nq, "cuda")
    ops.select_union(torch.from_numpy(r32).reshape(1, 1, nq, nq).cuda(), union, eta, block=block)
    fine = bits_to_bool(union.cpu().numpy()[0, 0], nq)
    coarse = coarse_of_fine(fine, f)
    assert np.array_equal(fine, O.expand_support(coarse, f))
    assert compare_selection(coarse, O.block_mass(q, k, block=block), eta) <= 1


def test_select_union_blocks_32_is_the_plain_selection(ops):
    """block = 32 through the variant entry point is exactly wise_select_union."""
    nq, bh = 45, 2
    m = _peaky_masses(np.random.default_rng(3), bh, nq).astype(np.float32)
    dm = torch.from_numpy(m).reshape(1, bh, nq, nq).cuda()
    a = ops.new_bitmask(1, bh, nq, "cuda")
    b = ops.new_bitmask(1, bh, nq, "cuda")
    ops.select_union(dm, a, 0.95)
    from recurrent_depth_lm_b200._lib import lib, check
    shp = ops.shape_of(torch.empty(1, bh, nq * 32, 128, dtype=torch.bfloat16, device="meta"))
    check(lib.wise_select_union_blocks(dm.data_ptr(), b.data_ptr(), None, 0.95, 32, shp,
                                       torch.cuda.current_stream().cuda_stream),
          "wise_select_union_blocks")
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ---------------------------------------------------------------- controls and retained mass

def _bits_of(sel):
    """[bh, nq, nq] bool -> [1, bh, nq, W] int32 device words."""
    bh, nq, _ = sel.shape
    W = (nq + 31) // 32
    words = np.zeros((bh, nq, W), np.uint32)
    for b in range(nq):
        words[..., b // 32] |= sel[..., b].astype(np.uint32) << np.uint32(b % 32)
    return torch.from_numpy(words.view(np.int32)).reshape(1, bh, nq, W).cuda()


def _control_inputs(nq, bh, seed):
    rng = np.random.default_rng(seed)
    m32 = _peaky_masses(rng, bh, nq).astype(np.float32)
    ref = rng.random((bh, nq, nq)) < 0.3
    ref[:, np.arange(nq), np.arange(nq)] = True
    ref[0, nq // 2] = False                 # one empty reference row
    ref |= np.triu(np.ones((nq, nq), bool), 1)   # bits b > q are set and must be ignored
    return m32, ref


@pytest.mark.parametrize("nq,bh", [(8, 2), (45, 3), (128, 2), (512, 1)])
def test_size_matched_bit_exact(ops, nq, bh):
    """TopK involves only comparisons of the same fp32 masses: bit-exact against the oracle."""
    m32, ref = _control_inputs(nq, bh, 40 + nq)
    out = ops.select_size_matched(torch.from_numpy(m32).reshape(1, bh, nq, nq).cuda(), _bits_of(ref))
    got = bits_to_bool(out.cpu().numpy()[0], nq)
    for x in range(bh):
        want = O.size_matched(m32[x].astype(np.float64), ref[x])
        assert np.array_equal(got[x], want)
        assert np.array_equal(got[x].sum(axis=1), np.tril(ref[x]).sum(axis=1))


def test_size_matched_ties_go_to_lower_index(ops):
    nq = 40
    m = np.tril(np.full((nq, nq), 1.0, np.float32))
    m /= m.sum(axis=1, keepdims=True)       # uniform rows: every admissible block ties
    ref = np.zeros((1, nq, nq), bool)
    for qb in range(nq):
        ref[0, qb, : (qb + 1) // 2 + 1] = True
    out = ops.select_size_matched(torch.from_numpy(m).reshape(1, 1, nq, nq).cuda(), _bits_of(ref))
    got = bits_to_bool(out.cpu().numpy()[0], nq)[0]
    for qb in range(nq):
        k = (qb + 1) // 2 + 1
        assert np.nonzero(got[qb])[0].tolist() == list(range(min(k, qb + 1)))


@pytest.mark.parametrize("nq,bh", [(8, 2), (45, 3), (128, 2), (512, 1)])
def test_mass_matched_matches_oracle(ops, nq, bh):
    m32, ref = _control_inputs(nq, bh, 50 + nq)
    dm = torch.from_numpy(m32).reshape(1, bh, nq, nq).cuda()
    got = bits_to_bool(ops.select_mass_matched(dm, _bits_of(ref)).cpu().numpy()[0], nq)
    exempt = 0
    for x in range(bh):
        r = m32[x].astype(np.float64)
        want = O.mass_matched(r, ref[x])
        for qb in range(nq):
            if np.array_equal(got[x, qb], want[qb]):
                continue
            row = r[qb, : qb + 1]
            m = O.retained_mass(r, ref[x])[qb]
            d_ck, d_ck1, r_cut = O.cut_margins(row, m)
            assert not got[x, qb, qb + 1:].any()
            assert min(d_ck, d_ck1) <= 1e-5, (x, qb)   # fp32 sums vs correctly rounded ones
            exempt += 1
        # a reference that is itself a ranking prefix comes back exactly
        w = O.select(r, 0.9)
        back = ops.select_mass_matched(dm[:, x:x + 1].contiguous(), _bits_of(w[None]))
        assert np.array_equal(bits_to_bool(back.cpu().numpy()[0], nq)[0], w)
    assert exempt <= 2


@pytest.mark.parametrize("nq,bh", [(8, 2), (45, 3), (512, 1)])
def test_support_mass_matches_oracle(ops, nq, bh):
    """fp32 sum of <= 512 non-negative masses with total <= 1: error <= 21 * 2^-24 (16
    sequential adds per lane, a 5-level tree), 2e-6 with margin."""
    m32, ref = _control_inputs(nq, bh, 60 + nq)
    out = ops.support_mass(torch.from_numpy(m32).reshape(1, bh, nq, nq).cuda(), _bits_of(ref))
    got = out.cpu().numpy()[0]
    for x in range(bh):
        want = O.retained_mass(m32[x].astype(np.float64), ref[x])
        assert np.abs(got[x] - want).max() <= 2e-6
    assert got[0, nq // 2] == 0.0

@pytest.mark.parametrize("nq,bh", [(1, 1), (8, 2), (45, 3), (512, 2)])
def test_build_schedule_bit_exact(ops, nq, bh):
    rng = np.random.default_rng(nq * 7 + bh)
    bits = rng.integers(0, 2 ** 32, size=(1, bh, nq, (nq + 31) // 32), dtype=np.uint64)
    dev_bits = torch.from_numpy(bits.astype(np.uint32).view(np.int32)).cuda()
    ro, ci, nnz = ops.build_schedule(dev_bits, head_dim=64)
    ro, ci = ro.cpu().numpy(), ci.cpu().numpy()
    sup = np.tril(bits_to_bool(bits.astype(np.uint32)[0], nq))
    assert nnz == int(sup.sum()) == ro[-1]
    for x in range(bh):
        r0, r1 = x * nq, (x + 1) * nq
        check_csr(ro[r0:r1 + 1] - ro[r0], ci[ro[r0]:ro[r1]], sup[x])


def test_build_schedule_capacity_error(ops):
    from recurrent_depth_lm_b200._lib import WiseError
    nq, bh = 16, 1
    bits = torch.full((1, bh, nq, 1), -1, dtype=torch.int32, device="cuda")
    small = torch.empty(10, dtype=torch.int32, device="cuda")
    with pytest.raises(WiseError) as e:
        ops.build_schedule(bits, col_idx=small, exact_nnz=True)
    assert e.value.code == -4
    with pytest.raises(WiseError):
        ops.build_schedule(bits, col_idx=small, exact_nnz=False)


def test_bounded_wait_times_out_and_context_survives(ops):
    """Failure detection without a GPU fault: a pipeline wait that nothing completes
    gives up after its limit, records WISE_STATUS_TIMEOUT, and the context stays
    usable (an attention call right after still matches the oracle)."""
    import time
    from recurrent_depth_lm_b200._lib import WISE_STATUS_TIMEOUT, check, lib
    ops.device_status(clear=True)
    t0 = time.perf_counter()
    check(lib.wise_diag_wait_timeout(50_000_000, torch.cuda.current_stream().cuda_stream),
          "wise_diag_wait_timeout")
    st = ops.device_status(clear=True)
    elapsed = time.perf_counter() - t0
    assert st & WISE_STATUS_TIMEOUT
    assert 0.04 <= elapsed < 5.0
    assert ops.device_status() == 0
    qb, kb, vb = rand_qkv_bits(1, 1, 128, 64, seed=21)
    o, _, _ = ops.full_attn_mass(to_dev(qb), to_dev(kb), to_dev(vb))
    o_ref, _ = O.causal_attention(*(bf16_bits_to_f64(x[0, 0]) for x in (qb, kb, vb)))
    compare_o(dev_f32(o)[0, 0], o_ref)


# ---------------------------------------------------------------- block size 16

def _words_of(sel):
    """[..., rows, cols] bool -> [..., rows, ceil(cols/32)] int32 words (bit c % 32 of word c // 32)."""
    cols = sel.shape[-1]
    W = (cols + 31) // 32
    words = np.zeros(sel.shape[:-1] + (W,), np.uint32)
    for c in range(cols):
        words[..., c // 32] |= sel[..., c].astype(np.uint32) << np.uint32(c % 32)
    return words.view(np.int32)


def _decode_b16(ro, ci, sub, nq):
    """One head's 32-token CSR plus sub-masks -> the 16-token support [2nq, 2nq]."""
    sel = np.zeros((2 * nq, 2 * nq), bool)
    for q in range(nq):
        for e in range(ro[q], ro[q + 1]):
            b = int(ci[e])
            assert 0 < sub[e] < 16, "entries carry at least one sub-block"
            for a in range(2):
                for c in range(2):
                    if (sub[e] >> (2 * a + c)) & 1:
                        sel[2 * q + a, 2 * b + c] = True
    return sel


B16_SHAPES = [(1, 2, 256, 64), (2, 3, 544, 96), (1, 2, 1024, 128)]


@pytest.mark.parametrize("b,h,n,d", B16_SHAPES)
def test_block_mass_b16_matches_oracle(ops, b, h, n, d):
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=7 * n + d)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    _, lse, _ = ops.full_attn_mass(q, k, v, with_mass=False, lse=torch.empty(b, h, n, device="cuda"))
    m16 = ops.block_mass_b16(q, k, lse).cpu().numpy()
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    n16 = n // 16
    for bi in range(b):
        for hi in range(h):
            qf, kf = (bf16_bits_to_f64(x[bi, hi]) for x in (qb, kb))
            r16 = O.block_mass(qf, kf, block=16)
            assert np.abs(np.tril(m16[bi, hi]) - r16).max() <= MASS_TOL
            # the one above-diagonal 16-block inside each diagonal 32-block is written 0
            assert np.all(m16[bi, hi][np.arange(0, n16, 2), np.arange(1, n16, 2)] == 0.0)


@pytest.mark.parametrize("b,h,n,d,hkv", [(1, 2, 256, 64, 2), (2, 3, 544, 96, 1),
                                         (1, 4, 1024, 128, 2), (1, 1, 16384, 128, 1)])
def test_one_pass_mass_b16(ops, b, h, n, d, hkv):
    """wise_full_attn_mass_b16: O and lse bit-identical to wise_full_attn_mass, the 16-token
    mass equal to the recomputing wise_block_mass_b16 (to fp32 rounding) and to the oracle's
    block mass at B = 16, the diagonal 32-block's upper 16 x 16 quarter written 0."""
    g = h // hkv
    qb, _, _ = rand_qkv_bits(b, h, n, d, seed=3 * n + d)
    _, kb, vb = rand_qkv_bits(b, hkv, n, d, seed=3 * n + d + 1)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    o1, lse1, m1 = ops.full_attn_mass_b16(q, k, v)
    o2, lse2, _ = ops.full_attn_mass(q, k, v, lse=torch.empty(b, h, n, device="cuda"))
    m2 = ops.block_mass_b16(q, k, lse2)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)
    n16 = n // 16
    low = torch.ones(n16, n16, dtype=torch.bool, device="cuda").tril()
    quarter = torch.zeros(n16, n16, dtype=torch.bool, device="cuda")
    quarter[torch.arange(0, n16, 2), torch.arange(1, n16, 2)] = True
    assert (m1[..., low] - m2[..., low]).abs().max().item() <= 2e-6
    assert torch.all(m1[..., quarter] == 0.0)
    m1 = m1.cpu().numpy()
    for bi, hi in sorted({(0, 0), (b - 1, h - 1)}):
        qf = bf16_bits_to_f64(qb[bi, hi])
        kf = bf16_bits_to_f64(kb[bi, hi // g])
        assert np.abs(np.tril(m1[bi, hi]) - O.block_mass(qf, kf, block=16)).max() <= MASS_TOL


@pytest.mark.parametrize("n16,bh", [(16, 2), (90, 3), (1024, 1)])
def test_select_union_b16_matches_oracle(ops, n16, bh):
    rng = np.random.default_rng(n16 + 1)
    m32 = _peaky_masses(rng, bh, n16).astype(np.float32)
    union = ops.new_bitmask_b16(1, bh, n16 * 16, "cuda")
    step = torch.empty_like(union)
    ops.select_union_b16(torch.from_numpy(m32).reshape(1, bh, n16, n16).cuda(), union, 0.95,
                         step_bits=step)
    s = bits_to_bool(step.cpu().numpy()[0], n16)
    assert np.array_equal(bits_to_bool(union.cpu().numpy()[0], n16), s)
    exempt = sum(compare_selection(s[x], m32[x].astype(np.float64), 0.95) for x in range(bh))
    assert exempt <= 2


@pytest.mark.parametrize("nq,bh", [(1, 1), (5, 2), (45, 3), (512, 1)])
def test_build_schedule_b16_bit_exact(ops, nq, bh):
    """The schedule decodes back to exactly the causal part of the 16-token working set;
    its 32-token CSR lists exactly the blocks with a kept sub-block, ascending."""
    rng = np.random.default_rng(nq * 3 + bh)
    n16 = 2 * nq
    sel = rng.random((bh, n16, n16)) < 0.3           # includes bits above the diagonal
    words = torch.from_numpy(_words_of(sel)).reshape(1, bh, n16, -1).cuda()
    ro, ci, sub, nnz = ops.build_schedule_b16(words, head_dim=64)
    ro, ci, sub = ro.cpu().numpy(), ci.cpu().numpy(), sub.cpu().numpy()
    assert nnz == ro[-1]
    for x in range(bh):
        r0, r1 = x * nq, (x + 1) * nq
        hro = ro[r0:r1 + 1] - ro[r0]
        hci, hsub = ci[ro[r0]:ro[r1]], sub[ro[r0]:ro[r1]]
        causal = np.tril(sel[x])
        assert np.array_equal(_decode_b16(hro, hci, hsub, nq), causal)
        fold = causal.reshape(nq, 2, nq, 2).any(axis=(1, 3))
        check_csr(hro, hci, fold)


def _b16_support(nq, rng, p=0.45, empty_row16=None):
    sel = np.tril(rng.random((2 * nq, 2 * nq)) < p)
    np.fill_diagonal(sel, True)
    if empty_row16 is not None:
        sel[empty_row16] = False
    return sel


@pytest.mark.parametrize("b,h,n,d,hkv", [(1, 2, 256, 64, 2), (1, 3, 544, 96, 3),
                                         (2, 2, 1024, 128, 2), (1, 4, 512, 128, 1)])
def test_sparse_attn_b16_matches_oracle(ops, b, h, n, d, hkv):
    """Random 16-token supports (one 16-row left empty: O = 0, lse = -inf) through the GPU
    schedule builder and the sub-masked kernel, against masked attention at B = 16."""
    nq = n // 32
    rng = np.random.default_rng(n + h)
    qb, _, _ = rand_qkv_bits(b, h, n, d, seed=n + 5)
    _, kb, vb = rand_qkv_bits(b, hkv, n, d, seed=n + 6)
    sups = np.stack([_b16_support(nq, rng, empty_row16=(3 if x == 0 else None))
                     for x in range(b * h)])
    words = torch.from_numpy(_words_of(sups)).reshape(b, h, 2 * nq, -1).cuda()
    ro, ci, sub, nnz = ops.build_schedule_b16(words, head_dim=d)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    lse = torch.empty(b, h, n, device="cuda")
    o, _ = ops.sparse_attn_b16(q, k, v, ro, ci, sub, nnz, lse=lse)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    o, lse = dev_f32(o), lse.cpu().numpy()
    g = h // hkv
    for bi in range(b):
        for hi in range(h):
            x = bi * h + hi
            qf = bf16_bits_to_f64(qb[bi, hi])
            kf, vf = (bf16_bits_to_f64(t[bi, hi // g]) for t in (kb, vb))
            o_ref, lse_ref = O.masked_attention(qf, kf, vf, sups[x], block=16)
            rows = np.isfinite(lse_ref)
            compare_o(o[bi, hi][rows], o_ref[rows], f"B16 O[{bi},{hi}]")
            assert np.abs(lse[bi, hi][rows] - lse_ref[rows]).max() <= LSE_TOL
            assert np.all(o[bi, hi][~rows] == 0.0) and np.all(np.isneginf(lse[bi, hi][~rows]))
            if x == 0:
                assert (~rows).sum() == 16


def test_sparse_attn_b16_all_blocks_equals_dense(ops):
    b, h, n, d = 1, 2, 544, 128
    nq = n // 32
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=99)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    sel = np.broadcast_to(np.tril(np.ones((2 * nq, 2 * nq), bool)), (b * h, 2 * nq, 2 * nq))
    words = torch.from_numpy(_words_of(np.ascontiguousarray(sel))).reshape(b, h, 2 * nq, -1).cuda()
    ro, ci, sub, nnz = ops.build_schedule_b16(words, head_dim=d)
    o16, _ = ops.sparse_attn_b16(q, k, v, ro, ci, sub, nnz)
    od, _, _ = ops.full_attn_mass(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o16, od)


# ---------------------------------------------------------------- score jumps inside an entry

@pytest.mark.parametrize("jump", [20.0, 200.0])
def test_score_jump_inside_an_entry(ops, jump):
    """Key block 3 scores `jump` (log2 units) above blocks 0-2 for every query that sees
    it: the softmax meets a row max far above its running reference partway through an
    entry of 4 key blocks, after P of the earlier blocks is written (and, at 200, beyond
    the fp32 range of 2^-126 for those earlier blocks).  Dense and all-blocks sparse
    against the oracle."""
    b, h, n, d = 1, 2, 256, 64
    rng = np.random.default_rng(int(jump))
    q = rng.standard_normal((b, h, n, d), dtype=np.float32) * np.float32(0.3)
    k = rng.standard_normal((b, h, n, d), dtype=np.float32) * np.float32(0.3)
    v = rng.standard_normal((b, h, n, d), dtype=np.float32)
    scale = 1.0 / math.sqrt(d)
    q[..., 0] = 1.0
    k[..., 0] = 0.0
    k[:, :, 96:128, 0] = np.float32(jump / (scale * math.log2(math.e)))
    qb, kb, vb = (f32_to_bf16_bits(x) for x in (q, k, v))
    dq, dk, dv = to_dev(qb), to_dev(kb), to_dev(vb)
    nq = n // 32
    per_head = nq * (nq + 1) // 2
    ro = torch.tensor([x * per_head + r * (r + 1) // 2 for x in range(b * h) for r in range(nq)]
                      + [b * h * per_head], dtype=torch.int32, device="cuda")
    ci = torch.tensor([c for x in range(b * h) for r in range(nq) for c in range(r + 1)],
                      dtype=torch.int32, device="cuda")
    od, lse_d, _ = ops.full_attn_mass(dq, dk, dv, lse=torch.empty(b, h, n, device="cuda"))
    lse_s = torch.empty(b, h, n, device="cuda")
    os_, _ = ops.sparse_attn(dq, dk, dv, ro, ci, ci.numel(), lse=lse_s)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    for hi in range(h):
        qf, kf, vf = (bf16_bits_to_f64(x[0, hi]) for x in (qb, kb, vb))
        o_ref, lse_ref = O.causal_attention(qf, kf, vf)
        for name, o, l in (("dense", od, lse_d), ("sparse", os_, lse_s)):
            compare_o(dev_f32(o)[0, hi], o_ref, f"{name} jump {jump} head {hi}")
            assert np.abs(l.cpu().numpy()[0, hi] - lse_ref).max() <= LSE_TOL


def test_sparse_attn_b16_maximum_length(ops):
    """n = 16384 (512 query blocks: every word of the sub-mask planes in use), one head
    against masked attention at B = 16."""
    b, h, n, d = 1, 1, 16384, 64
    nq = n // 32
    rng = np.random.default_rng(16384)
    qb, kb, vb = rand_qkv_bits(b, h, n, d, seed=77)
    sel = _b16_support(nq, rng, p=0.3)
    words = torch.from_numpy(_words_of(sel[None])).reshape(b, h, 2 * nq, -1).cuda()
    ro, ci, sub, nnz = ops.build_schedule_b16(words, head_dim=d)
    lse = torch.empty(b, h, n, device="cuda")
    o, _ = ops.sparse_attn_b16(to_dev(qb), to_dev(kb), to_dev(vb), ro, ci, sub, nnz, lse=lse)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    qf, kf, vf = (bf16_bits_to_f64(x[0, 0]) for x in (qb, kb, vb))
    o_ref, lse_ref = O.masked_attention(qf, kf, vf, sel, block=16)
    compare_o(dev_f32(o)[0, 0], o_ref, "B16 n=16384")
    assert np.abs(lse.cpu().numpy()[0, 0] - lse_ref).max() <= LSE_TOL


@pytest.mark.parametrize("d", [64, 96])
def test_maximum_length_dense_and_sparse(ops, d):
    """n = 16384 (512 query blocks, 16 schedule words per row) at the head dims other than
    128, with two query heads on one K/V head: dense attention with lse and the one-pass
    block mass, and block-sparse attention with lse, each head against the oracle."""
    b, h, hkv, n = 1, 2, 1, 16384
    nq = n // 32
    qb, _, _ = rand_qkv_bits(b, h, n, d, seed=16384 + d)
    _, kb, vb = rand_qkv_bits(b, hkv, n, d, seed=16385 + d)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    o, lse, mass = ops.full_attn_mass(q, k, v, with_mass=True)
    rng = np.random.default_rng(d)
    sups = [random_support(nq, rng, p=0.3) for _ in range(b * h)]
    ro, ci, nnz = csr_device(sups)
    lse_s = torch.empty(b, h, n, device="cuda")
    o_s, _ = ops.sparse_attn(q, k, v, ro, ci, nnz, lse=lse_s)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    o, lse, mass = dev_f32(o), lse.cpu().numpy(), mass.cpu().numpy()
    o_s, lse_s = dev_f32(o_s), lse_s.cpu().numpy()
    kf, vf = (bf16_bits_to_f64(x[0, 0]) for x in (kb, vb))
    for hi in range(h):
        qf = bf16_bits_to_f64(qb[0, hi])
        o_ref, lse_ref = O.causal_attention(qf, kf, vf)
        compare_o(o[0, hi], o_ref, f"dense n=16384 d={d} head {hi}")
        assert np.abs(lse[0, hi] - lse_ref).max() <= LSE_TOL
        if hi == 0:
            assert np.abs(np.tril(mass[0, hi]) - O.block_mass(qf, kf)).max() <= MASS_TOL
        o_ref, lse_ref = O.masked_attention(qf, kf, vf, sups[hi])
        compare_o(o_s[0, hi], o_ref, f"sparse n=16384 d={d} head {hi}")
        assert np.abs(lse_s[0, hi] - lse_ref).max() <= LSE_TOL


# nq = 17 (a ragged group of query blocks), GQA, d = 96, and n = 16384 (16 mask words per row)
WINDOW_SHAPES = [(1, 3, 544, 64, 3), (2, 4, 1024, 128, 2), (1, 2, 4096, 96, 1),
                 (1, 1, 16384, 128, 1)]


@pytest.mark.parametrize("b,h,n,d,hkv", WINDOW_SHAPES)
def test_window_step_is_attention_mass_and_selection(ops, b, h, n, d, hkv):
    """wise_window_step = wise_full_attn_mass + wise_select_union, bit for bit, ORing into
    a working set from earlier steps; its masses and step support against the oracle."""
    g, nq = h // hkv, n // 32
    w = (nq + 31) // 32
    qb, _, _ = rand_qkv_bits(b, h, n, d, seed=5 * n + h)
    _, kb, vb = rand_qkv_bits(b, hkv, n, d, seed=5 * n + hkv + 1)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    eta = 0.9
    rng = np.random.default_rng(n + d)
    prior_np = (rng.integers(0, 2**32, (b, h, nq, w), dtype=np.uint64) &
                rng.integers(0, 2**32, (b, h, nq, w), dtype=np.uint64) &
                rng.integers(0, 2**32, (b, h, nq, w), dtype=np.uint64))
    prior = torch.from_numpy(prior_np.astype(np.uint32).view(np.int32)).cuda()
    u1, u2 = prior.clone(), prior.clone()
    st1, st2 = torch.empty_like(prior), torch.empty_like(prior)
    o1, lse1, m1 = ops.window_step(q, k, v, u1, eta, step_bits=st1)
    o2, lse2, m2 = ops.full_attn_mass(q, k, v, with_mass=True)
    ops.select_union(m2, u2, eta, step_bits=st2, head_dim=d)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)
    tri = torch.ones(nq, nq, dtype=torch.bool, device="cuda").tril()
    assert torch.equal(m1[..., tri], m2[..., tri])
    assert torch.equal(st1, st2) and torch.equal(u1, u2)
    assert torch.equal(u1, prior | st1)
    m1, st1 = m1.cpu().numpy(), st1.cpu().numpy()
    exempt = 0
    for bi, hi in sorted({(0, 0), (b - 1, h - 1)}):
        qf = bf16_bits_to_f64(qb[bi, hi])
        kf = bf16_bits_to_f64(kb[bi, hi // g])
        r_ref = O.block_mass(qf, kf)
        assert np.abs(np.tril(m1[bi, hi]) - r_ref).max() <= MASS_TOL
        exempt += compare_selection(bits_to_bool(st1[bi, hi], nq), r_ref, eta)
    assert exempt <= max(2, nq // 16)


@pytest.mark.parametrize("nq,bh", [(128, 3), (512, 2)])
def test_select_exact_on_dyadic_masses(ops, nq, bh):
    """Masses that are multiples of 2^-12 (each row sums to exactly 1, many exact ties):
    every cumulative sum is exact in the kernel's units and in fp64, so the support must
    equal the oracle's bit for bit with no near-cut exemption.  A few entries are above 1,
    negative, -0 or NaN: the kernel counts them as clamp(r, 0, 1), NaN as 0."""
    rng = np.random.default_rng(7 * nq + bh)
    m = np.zeros((bh, nq, nq), np.float32)
    for x in range(bh):
        for q in range(nq):
            w = rng.random(q + 1) ** 6 + 1e-3          # a few heavy blocks, long light tail
            m[x, q, : q + 1] = rng.multinomial(4096, w / w.sum()) / 4096.0
    odd = []
    for x in range(bh):
        for q in rng.choice(np.arange(8, nq), 6, replace=False):
            b = int(rng.integers(0, q + 1))
            val = [1.5, -0.25, -0.0, np.nan, 1.0, 0.0][len(odd) % 6]
            m[x, q, b] = val
            odd.append((x, q, b))
    clean = np.nan_to_num(np.clip(m, 0.0, 1.0), nan=0.0).astype(np.float64)
    mass = torch.from_numpy(m).reshape(1, bh, nq, nq).cuda()
    for eta in (0.5, 0.75, 0.875, 0.9, 0.99):
        union = ops.new_bitmask(1, bh, nq, "cuda")
        step = torch.empty_like(union)
        ops.select_union(mass, union, eta, step_bits=step)
        torch.cuda.synchronize()
        got = bits_to_bool(step.cpu().numpy()[0], nq)
        e32 = float(np.float32(eta))
        for x in range(bh):
            want = O.select(clean[x], e32)
            bad = np.nonzero((got[x] != want).any(axis=1))[0]
            assert bad.size == 0, f"eta={eta} head {x}: rows {bad[:8].tolist()} differ"
    assert ops.device_status() == 0
