"""Property tests of the oracle (hypothesis): the route against exhaustive search on many
random rows, and masked attention against torch's scaled_dot_product_attention in fp64
on random ragged geometries and block masks.

The route: the oracle keeps the shortest prefix of the (score desc, index asc) order whose mass is
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


@st.composite
def attn_cases(draw):
    T, Hs, Ws = draw(st.integers(1, 3)), draw(st.integers(1, 7)), draw(st.integers(1, 9))
    bt, bh, bw = draw(st.integers(1, 2)), draw(st.integers(1, 4)), draw(st.integers(1, 5))
    d = draw(st.sampled_from([4, 8, 16]))
    seed = draw(st.integers(0, 2**31 - 1))
    density = draw(st.sampled_from([0.1, 0.4, 0.8]))
    return T, Hs, Ws, bt, bh, bw, d, seed, density


@settings(max_examples=60, derandomize=True, deadline=None)
@given(attn_cases())
def test_masked_attention_equals_sdpa_with_token_mask(case):
    """masked_attn on random ragged geometries and block masks (each row keeps its own
    block) equals scaled_dot_product_attention in fp64 with the token-level mask."""
    import torch
    T, Hs, Ws, bt, bh, bw, d, seed, density = case
    g = O.block_geometry(T, Hs, Ws, bt, bh, bw)
    rng = np.random.default_rng(seed)
    N = T * Hs * Ws
    Q, K, V = (rng.standard_normal((1, 2, N, d)) * s for s in (1.5, 1.0, 1.0))
    keep = rng.random((1, 2, g.nB, g.nB)) < density
    keep[..., np.arange(g.nB), np.arange(g.nB)] = True
    scale = 1.0 / math.sqrt(d)
    tokens, out, lse = O.masked_attn(Q, K, V, keep, g, scale)
    bt_of = g.block_of_token
    tok_mask = torch.from_numpy(keep[:, :, bt_of][:, :, :, bt_of])
    tq, tk, tv = (torch.from_numpy(a) for a in (Q, K, V))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=tok_mask, scale=scale)
    np.testing.assert_allclose(out, ref.numpy()[:, :, tokens], atol=1e-12)
    logits = torch.einsum("bhid,bhjd->bhij", tq, tk) * scale
    ref_lse = torch.logsumexp(logits.masked_fill(~tok_mask, float("-inf")), dim=-1)
    np.testing.assert_allclose(lse, ref_lse.numpy()[:, :, tokens], atol=1e-12)


@st.composite
def pool_cases(draw):
    return (draw(st.integers(1, 4)), draw(st.integers(1, 9)), draw(st.integers(1, 11)),
            draw(st.integers(1, 3)), draw(st.integers(1, 5)), draw(st.integers(1, 6)),
            draw(st.integers(0, 2**31 - 1)))


@settings(max_examples=80, derandomize=True, deadline=None)
@given(pool_cases())
def test_pool_equals_mean_over_latent_ranges(case):
    """pool on random ragged geometries equals, for every block (tb, yb, xb), the mean of
    the tokens at t in [tb bt, min(T, tb bt + bt)), y and x likewise, taken from the
    latent grid."""
    T, Hs, Ws, bt, bh, bw, seed = case
    g = O.block_geometry(T, Hs, Ws, bt, bh, bw)
    X = np.random.default_rng(seed).standard_normal((1, 2, T * Hs * Ws, 3))
    got = O.pool(X, g)
    grid = X.reshape(1, 2, T, Hs, Ws, 3)
    nBt, nBy, nBx = -(-T // bt), -(-Hs // bh), -(-Ws // bw)
    for tb in range(nBt):
        for yb in range(nBy):
            for xb in range(nBx):
                j = (tb * nBy + yb) * nBx + xb
                sub = grid[:, :, tb * bt:(tb + 1) * bt, yb * bh:(yb + 1) * bh, xb * bw:(xb + 1) * bw]
                want = sub.reshape(1, 2, -1, 3).mean(axis=2)
                np.testing.assert_allclose(got[:, :, j], want, rtol=0, atol=1e-13)
