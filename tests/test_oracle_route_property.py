"""The oracle's route against exhaustive search, on many random rows (hypothesis).

The oracle keeps the shortest prefix of the (score desc, index asc) order whose mass is
>= p, lengthened to the Top-k floor, plus the own block.  The exhaustive search finds,
over all subsets, the smallest size whose best subset reaches p, then the heaviest subset
of size max(that, k) with ties to the lexicographically smallest, plus the own block: the
same set by a different route.  Logits come from a small integer grid, so exactly tied
scores occur; draws where some subset's mass lies within 1e-9 of p are discarded, since
there the summation order alone could decide."""
import itertools
import math

import numpy as np
from hypothesis import assume, given, settings
from hypothesis import strategies as st

import oracle as O


@st.composite
def rows(draw):
    nB = draw(st.integers(1, 8))
    logits = draw(st.lists(st.integers(-3, 3), min_size=nB, max_size=nB))
    own = draw(st.integers(0, nB - 1))
    p = draw(st.sampled_from([0.0, 0.05, 0.2, 0.33, 0.5, 0.61, 0.75, 0.9, 0.95, 0.999, 1.0]))
    k = draw(st.integers(0, nB + 2))
    return nB, logits, own, p, k


@settings(max_examples=400, derandomize=True, deadline=None)
@given(rows())
def test_route_row_equals_exhaustive_search(case):
    nB, logits, own, p, k = case
    scale = 0.5
    # one query row `own` with logits l: Kp = identity, Qp[own] = l / scale
    Kp = np.eye(nB)[None, None]
    Qp = np.zeros((1, 1, nB, nB))
    Qp[0, 0, own] = np.asarray(logits, dtype=np.float64) / scale
    r = O.route(Qp, Kp, p, k, scale)
    s = r.scores[0, 0, own]
    if p < 1.0:
        for c in range(1, nB + 1):
            for S in itertools.combinations(range(nB), c):
                assume(abs(float(s[list(S)].sum()) - p) > 1e-9)
    want = O.brute_force_route_row(s, own, p, k)
    assert (r.keep[0, 0, own] == want).all(), (logits, own, p, k)
    assert r.counts[0, 0, own] == want.sum()
    # the scores are the softmax of the logits
    e = np.exp(np.asarray(logits, dtype=np.float64) - max(logits))
    assert np.allclose(s, e / e.sum(), rtol=0, atol=1e-15)
    # and the kept count never falls below the floor nor exceeds nB
    assert min(k, nB) <= want.sum() <= nB
    assert want[own]
    if p >= 1.0 or k >= nB:
        assert want.all()
    assert math.isclose(float(s.sum()), 1.0, rel_tol=0, abs_tol=1e-12)
