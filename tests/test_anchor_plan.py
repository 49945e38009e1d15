"""The native anchor planner (kascade_plan_anchors, host code of the
library) against the oracle's recursion and exhaustive search, on the CPU."""
import numpy as np
import pytest

import oracle as O

RNG = np.random.default_rng(5)


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


@pytest.mark.parametrize("n,m", [(1, 1), (5, 1), (8, 3), (12, 4), (32, 4), (36, 4), (20, 20)])
def test_native_plan_matches_oracle(n, m):
    kc = _kc()
    for _ in range(3):
        sim = np.triu(RNG.random((n, n)))
        np.fill_diagonal(sim, 1.0)
        got, val = kc.plan_anchors(sim, m)
        want, wval = O.plan_anchors(sim, m)
        assert got == want and abs(val - wval) < 1e-9
        assert got[0] == 0 and got == sorted(set(got))


def test_native_plan_closed_forms_and_errors():
    kc = _kc()
    sim = np.zeros((6, 6))
    sim[:3, :3] = 1.0
    sim[3:, 3:] = 1.0
    assert kc.plan_anchors(sim, 2) == ([0, 3], 6.0)
    assert kc.plan_anchors(np.ones((5, 5)), 3) == ([0, 1, 2], 5.0)
    for bad in (0, 7):
        with pytest.raises(kc.KascadeError):
            kc.plan_anchors(np.eye(6), bad)
