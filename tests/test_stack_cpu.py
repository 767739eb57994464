"""Host arithmetic of the composed workloads (no GPU): the Sirius round's effective density from
the drafts' active-list sizes against the oracle's from the masks."""
import numpy as np
import pytest

import oracle
from contextual_sparsity_ffn_b200 import stack


@pytest.mark.parametrize("T,h,p", [(16, 28672, 0.5), (16, 28672, 0.1), (1, 7, 0.3), (5, 1000, 0.0), (3, 64, 1.0)])
def test_round_effective_density_matches_oracle(T, h, p):
    m = np.random.default_rng(T * 1000 + h).random((T, h)) < p
    got = stack.round_effective_density(m.sum(axis=1).tolist(), h)
    assert got == pytest.approx(oracle.round_effective_density(m)["effective_density"], rel=1e-12)


def test_round_effective_density_limits():
    # all drafts dense: T + 1 dense passes for T tokens; all drafts empty: the gate only, plus the verify
    assert stack.round_effective_density([10] * 4, 10) == pytest.approx(5 / 4)
    assert stack.round_effective_density([0] * 4, 10) == pytest.approx((4 * 10 + 30) / (3 * 10 * 4))
