"""The seeded workload generator: determinism, per-head streams, bf16 rounding."""

import numpy as np
import pytest

from wise_inputs import (CONFIGS, HeadStream, bf16_bits_to_f32, f32_to_bf16_bits,
                         generate_all_steps, iter_steps)


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * 10.0 ** rng.integers(-5, 5, 100000)).astype(np.float32)
    ours = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_deterministic_and_head_subsets_agree():
    cfg = CONFIGS["tiny"]
    full = [(t, q.copy(), k.copy(), v.copy()) for t, q, k, v in iter_steps(cfg)]
    again = [(t, q, k, v) for t, q, k, v in iter_steps(cfg)]
    one = [(t, q, k, v) for t, q, k, v in iter_steps(cfg, heads=[(0, 1)])]
    for (t, q, k, v), (_, q2, k2, v2), (_, q1, k1, v1) in zip(full, again, one):
        assert np.array_equal(q, q2) and np.array_equal(v, v2)
        assert np.array_equal(q[0, 1], q1[0]) and np.array_equal(k[0, 1], k1[0])
        assert np.array_equal(v[0, 1], v1[0])
    allsteps = generate_all_steps(cfg)
    assert allsteps.shape == (8, 3, 1, 2, 256, 64)
    assert np.array_equal(allsteps[2, 1], full[2][2])


def test_ranks_draw_different_data():
    cfg = CONFIGS["tiny"]
    a = next(iter_steps(cfg, rank=0))[1]
    b = next(iter_steps(cfg, rank=1))[1]
    assert not np.array_equal(a, b)


def test_recipe_structure():
    cfg = CONFIGS["tiny"]
    s = HeadStream(cfg, 0, 0)
    assert len(s.hot_blocks) == 2 and len(set(s.hot_blocks.tolist())) == 2
    q0, k0, v0 = (x.copy() for x in s.masters)
    q1, k1, v1 = (bf16_bits_to_f32(x) for x in s.next_step())
    drift = np.std(q1 - q0)
    assert 0.2 < drift < 0.3            # sigma_1 = 0.3 * 0.8 (plus bf16 rounding)
    assert abs(np.mean(v1)) < 0.05 and 0.9 < np.std(v1) < 1.1
    c2 = CONFIGS["2k_b4_h40_d96"].with_(batch=1, heads=3, seqlen=256)
    for h in range(3):
        m = len(HeadStream(c2, 0, h).hot_blocks)
        assert 1 <= m <= 2
