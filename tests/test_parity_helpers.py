"""CPU checks of the comparison helpers of the GPU parity tests (tests/parity.py):
the near-cut acceptance for selections that differ at a near-margin cut, and
the bf16 output allowance."""
import numpy as np

from tests import parity


def test_near_cut_accepts_the_other_side_of_a_tie_and_rejects_short_sets():
    # P = (0.4, 0.3, 0.3): at p = 0.7 the oracle keeps {0, 1} (tie to the lower
    # index); {0, 2} has the same mass and size, {0} falls short of p.
    P = np.array([0.4, 0.3, 0.3])
    assert parity.near_cut_ok(P, [True, False, True], 0.7)
    assert not parity.near_cut_ok(P, [True, False, False], 0.7)
    # one entry more than needed is still within one of k* ...
    assert parity.near_cut_ok(P, [True, True, True], 0.7)
    # ... two more is not (k* = 1 at p = 0.3)
    assert not parity.near_cut_ok(np.array([0.5, 0.25, 0.25]), [True, True, True], 0.3)


def test_near_cut_top_k_needs_k_entries_of_nearly_maximal_mass():
    P = np.array([0.5, 0.2, 0.2, 0.1])
    assert parity.near_cut_ok(P, [True, False, True, False], None, k=2)
    assert not parity.near_cut_ok(P, [True, False, False, True], None, k=2)
    assert not parity.near_cut_ok(P, [True, True, True, False], None, k=2)


def test_bf16_allowance_only_from_eight():
    want = np.array([1.0, 7.9, 8.0, 20.0])
    # 0.021 off at |ref| < 8 exceeds 2e-2; at |ref| >= 8 one ulp (1/16, 1/8) is allowed
    got = want + np.array([0.021, 0.0, 0.0, 0.0])
    assert parity.excess_over_bf16(got, want) > 2e-2
    got = want + np.array([0.0, 0.019, 0.0625 + 0.019, 0.125 + 0.019])
    assert parity.excess_over_bf16(got, want) <= 2e-2
