"""The attention kernel's barrier protocol, checked on a discrete-event model (CPU):
no hazard, early/late phase or deadlock over random tile mixes, ring sizes and
timings; and every wait that the protocol relies on is shown to be necessary."""

import pytest

from protocol_model import run_seeds


def test_protocol_has_no_hazard_or_deadlock():
    bad = run_seeds(range(600))
    assert not bad, {s: e[:2] for s, e in list(bad.items())[:3]}


# o_free is left out: it is implied by p_full.  The epilogue and the next tile's softmax
# run on the same threads, so the next tile's first P, and with it its first PV, comes
# after O was read; the kernel keeps the o_free wait as a second guard.
@pytest.mark.parametrize("bar", ["o_done", "k_empty", "v_empty", "k_full", "v_full", "s_full",
                                 "p_full", "e_full", "e_empty", "q_full", "q_empty", "s_free"])
def test_each_wait_is_needed(bar):
    """Skipping the waits on one barrier makes the model report a hazard, a wrong phase, a
    broken invariant or a deadlock for some tile mix (a planted protocol mistake)."""
    assert run_seeds(range(600), drop={bar}), f"dropping the {bar} waits went unnoticed"


def test_issue_order_is_what_lets_qk_follow_pv():
    """The issuer starts a slot's next QK right after the PV that reads the slot's P,
    without waiting for that PV: if MMAs could touch their operands out of issue order,
    the model would see the QK overwrite P before the PV read it."""
    bad = run_seeds(range(600), mma_in_order=False)
    assert any("before its PV read it" in e for errs in bad.values() for e in errs)
