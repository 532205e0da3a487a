"""Pins for the fp64 oracle against things other than itself: closed forms, brute force on
tiny inputs, hand-derived golden routing cases and library routines (torch SDPA)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from free_adaptive_block_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ geometry / pool
def test_block_geometry_480p_real_size_mix():
    # 30 x 52 latent frames cut into 8 x 16 blocks: per frame 4 x 4 blocks with
    # real sizes 9 x 128, 3 x 96 (H edge, 6 rows), 3 x 32 (W edge, 4 cols), 1 x 24.
    g = O.block_geometry(21, 30, 52, 1, 8, 16)
    assert g.nB == 21 * 16
    assert g.real_count.sum() == 21 * 30 * 52
    per_frame = sorted(g.real_count[:16].tolist())
    assert per_frame == sorted([128] * 9 + [96] * 3 + [32] * 3 + [24])
    # a token belongs to the block of its (t // bt, y // bh, x // bw)
    n = (5 * 30 + 29) * 52 + 50
    assert g.block_of_token[n] == (5 * 4 + 3) * 4 + 3
    assert n in set(g.tokens_of_block[(5 * 4 + 3) * 4 + 3].tolist())


def test_block_geometry_720p_and_t_edge():
    g = O.block_geometry(21, 45, 80, 1, 8, 16)
    assert g.nB == 21 * 6 * 5
    assert sorted(set(g.real_count.tolist())) == [80, 128]
    g2 = O.block_geometry(5, 12, 20, 2, 4, 8)       # T, H, W all ragged
    assert g2.nB == 3 * 3 * 3
    assert g2.real_count.sum() == 5 * 12 * 20
    assert g2.real_count.min() == 1 * 4 * 4          # the corner on the T and W edges


def test_pool_closed_form_when_blocks_divide_the_latent():
    rng = np.random.default_rng(0)
    T, Hs, Ws, bt, bh, bw, d = 4, 8, 8, 2, 4, 4, 6
    X = rng.standard_normal((2, 3, T * Hs * Ws, d))
    g = O.block_geometry(T, Hs, Ws, bt, bh, bw)
    got = O.pool(X, g)
    r = X.reshape(2, 3, T // bt, bt, Hs // bh, bh, Ws // bw, bw, d).mean(axis=(3, 5, 7))
    want = r.reshape(2, 3, -1, d)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


def test_pool_ragged_against_explicit_loops():
    rng = np.random.default_rng(1)
    T, Hs, Ws, bt, bh, bw, d = 3, 5, 7, 2, 2, 3, 4
    X = rng.standard_normal((1, 2, T * Hs * Ws, d))
    g = O.block_geometry(T, Hs, Ws, bt, bh, bw)
    got = O.pool(X, g)
    nBy, nBx = -(-Hs // bh), -(-Ws // bw)
    for h in range(2):
        for tb in range(-(-T // bt)):
            for yb in range(nBy):
                for xb in range(nBx):
                    acc, n = np.zeros(d), 0
                    for t in range(tb * bt, min(T, tb * bt + bt)):
                        for y in range(yb * bh, min(Hs, yb * bh + bh)):
                            for x in range(xb * bw, min(Ws, xb * bw + bw)):
                                acc += X[0, h, (t * Hs + y) * Ws + x]
                                n += 1
                    j = (tb * nBy + yb) * nBx + xb
                    np.testing.assert_allclose(got[0, h, j], acc / n, atol=1e-14)


# ------------------------------------------------------------------ routing
def _route_row(scores, own, p, k):
    """Route one hand-made row: Kp = identity and Qp rows = ln(scores) make the routing
    logits equal ln(scores), so the routing scores are the given ones."""
    s = np.asarray(scores, dtype=np.float64)
    nB = s.size
    logits = np.log(np.maximum(s, 1e-300))
    Qp = np.tile(logits, (nB, 1))[None, None]
    Kp = np.eye(nB)[None, None]
    r = O.route(Qp, Kp, p, k, 1.0)
    np.testing.assert_allclose(r.scores[0, 0, own], s / s.sum(), rtol=1e-12, atol=1e-300)
    return r.keep[0, 0, own], int(r.counts[0, 0, own])


def test_route_golden_hand_cases():
    cases = json.load(open(os.path.join(GOLDEN, "route_cases.json")))["cases"]
    for c in cases:
        keep, count = _route_row(c["scores"], c["own"], c["p"], c["k"])
        assert keep.astype(int).tolist() == c["keep"], c["name"]
        assert count == c["count"], c["name"]


def test_route_against_brute_force_on_tiny_config():
    w = W.TINY
    x = W.generate(w)
    g = O.block_geometry(w.T, w.Hs, w.Ws, w.bt, w.bh, w.bw)
    Qp, Kp = O.pool(x["q"], g), O.pool(x["k"], g)
    scale = 1.0 / math.sqrt(w.d)
    for p, k in itertools.product([0.0, 0.3, 0.6, 0.9, 0.97, 1.0], [0, 1, 2, 5, 8, 11]):
        r = O.route(Qp, Kp, p, k, scale)
        for h in range(w.H):
            for qb in range(g.nB):
                s_row = r.scores[0, h, qb]
                want = O.brute_force_route_row(s_row, qb, p, k)
                assert (r.keep[0, h, qb] == want).all(), (p, k, h, qb)
                assert r.counts[0, h, qb] == want.sum()


@pytest.mark.parametrize("wl", [W.SMALL_RAGGED, W.SMALL_RAGGED_T, W.TINY])
def test_route_invariants_every_row(wl):
    x = W.generate(wl)
    g = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    Qp, Kp = O.pool(x["q"], g), O.pool(x["k"], g)
    scale = 1.0 / math.sqrt(wl.d)
    for p, k in [(wl.p, wl.k_floor), (0.5, 1), (0.95, 16), (0.0, 0), (1.0, 0)]:
        r = O.route(Qp, Kp, p, k, scale)
        for b in range(wl.B):
            for h in range(wl.H):
                for qb in range(g.nB):
                    why = O.check_route_invariants(r.keep[b, h, qb], r.scores[b, h, qb], qb, p, k,
                                                   tol=1e-12)
                    assert why is None, (p, k, b, h, qb, why)
                    assert r.keep[b, h, qb].sum() == r.counts[b, h, qb]


def test_route_special_cases():
    rng = np.random.default_rng(5)
    Qp = rng.standard_normal((1, 2, 9, 8)) * 3
    Kp = rng.standard_normal((1, 2, 9, 8))
    assert O.route(Qp, Kp, 1.0, 0, 0.5).keep.all()
    assert O.route(Qp, Kp, 0.3, 9, 0.5).keep.all()
    assert O.route(Qp, Kp, 0.3, 50, 0.5).keep.all()
    r = O.route(Qp, Kp, 0.0, 0, 0.5)
    logits = np.einsum("bhid,bhjd->bhij", Qp, Kp)
    for h in range(2):
        for i in range(9):
            want = {int(np.argmax(logits[0, h, i])), i}
            assert set(np.nonzero(r.keep[0, h, i])[0].tolist()) == want


def test_invariant_checker_rejects_planted_mistakes():
    s = np.array([0.05, 0.4, 0.1, 0.25, 0.2])
    good = np.array([1, 1, 0, 1, 1], bool)
    assert O.check_route_invariants(good, s, 0, 0.7, 2) is None
    assert O.check_route_invariants(np.array([1, 1, 1, 1, 0], bool), s, 0, 0.7, 2) is not None
    assert O.check_route_invariants(np.array([0, 1, 0, 1, 1], bool), s, 0, 0.7, 2) is not None
    assert O.check_route_invariants(np.array([1, 1, 1, 1, 1], bool), s, 0, 0.7, 2) is not None
    assert O.check_route_invariants(np.array([1, 1, 0, 1, 0], bool), s, 0, 0.7, 2) is not None


def test_pack_unpack_roundtrip_and_bit_order():
    keep = np.zeros((1, 40), bool)
    keep[0, [0, 33, 39]] = True
    words = O.pack_mask(keep)
    assert words.tolist() == [[1, (1 << 1) | (1 << 7)]]
    rng = np.random.default_rng(2)
    k2 = rng.random((3, 4, 70)) < 0.4
    assert (O.unpack_mask(O.pack_mask(k2), 70) == k2).all()


# ------------------------------------------------------------------ attention
def _small_inputs(seed=3, B=1, H=2, T=2, Hs=6, Ws=10, d=16):
    rng = np.random.default_rng(seed)
    N = T * Hs * Ws
    Q = rng.standard_normal((B, H, N, d)) * 1.5
    K = rng.standard_normal((B, H, N, d))
    V = rng.standard_normal((B, H, N, d))
    return Q, K, V, O.block_geometry(T, Hs, Ws, 1, 4, 4)


def test_masked_all_blocks_equals_dense():
    Q, K, V, g = _small_inputs()
    keep = np.ones((1, 2, g.nB, g.nB), bool)
    tokens, out, lse = O.masked_attn(Q, K, V, keep, g, 0.25)
    dout, dlse = O.dense_attn(Q, K, V, 0.25, tokens)
    np.testing.assert_allclose(out, dout, atol=1e-12)
    np.testing.assert_allclose(lse, dlse, atol=1e-12)


def test_dense_matches_torch_sdpa_fp64():
    Q, K, V, g = _small_inputs(seed=4)
    out, lse = O.dense_attn(Q, K, V, 0.3)
    tq, tk, tv = (torch.from_numpy(a) for a in (Q, K, V))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.3)
    np.testing.assert_allclose(out, ref.numpy(), atol=1e-12)
    ref_lse = torch.logsumexp(tq @ tk.transpose(-1, -2) * 0.3, dim=-1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), atol=1e-12)


def test_masked_matches_torch_sdpa_with_boolean_mask():
    Q, K, V, g = _small_inputs(seed=6)
    rng = np.random.default_rng(7)
    keep = rng.random((1, 2, g.nB, g.nB)) < 0.4
    keep[..., np.arange(g.nB), np.arange(g.nB)] = True
    tokens, out, lse = O.masked_attn(Q, K, V, keep, g, 0.2)
    bt = g.block_of_token
    tok_mask = keep[:, :, bt][:, :, :, bt]                    # [B,H,N,N] token-level mask
    tq, tk, tv = (torch.from_numpy(a) for a in (Q, K, V))
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=torch.from_numpy(tok_mask), scale=0.2)
    np.testing.assert_allclose(out, ref.numpy()[:, :, tokens], atol=1e-12)


def test_lse_merge_identity_over_disjoint_key_sets():
    Q, K, V, g = _small_inputs(seed=8)
    rng = np.random.default_rng(9)
    keep = rng.random((1, 2, g.nB, g.nB)) < 0.6
    keep[..., np.arange(g.nB), np.arange(g.nB)] = True
    split = rng.random(keep.shape) < 0.5
    A = keep & split
    Bm = keep & ~split
    # make sure both halves are non-empty in every row
    own = np.arange(g.nB)
    A[..., own, own] = True
    Bm[..., own, own] = False
    Bm |= keep & ~A
    Bm[..., own, (own + 1) % g.nB] |= ~Bm.any(-1)
    full = A | Bm
    _, out, lse = O.masked_attn(Q, K, V, full, g, 0.3)
    _, oa, la = O.masked_attn(Q, K, V, A, g, 0.3)
    _, ob, lb = O.masked_attn(Q, K, V, Bm, g, 0.3)
    np.testing.assert_allclose(np.logaddexp(la, lb), lse, atol=1e-12)
    wa, wb = np.exp(la - lse)[..., None], np.exp(lb - lse)[..., None]
    np.testing.assert_allclose(wa * oa + wb * ob, out, atol=1e-12)


def test_masked_attention_brute_force_loops():
    Q, K, V, g = _small_inputs(seed=10, H=1, T=1, Hs=4, Ws=8, d=4)
    keep = np.zeros((1, 1, g.nB, g.nB), bool)
    keep[0, 0, 0, [0]] = True          # a single kept block: softmax over that block only
    keep[0, 0, 1, [0, 1]] = True
    tokens, out, lse = O.masked_attn(Q, K, V, keep, g, 0.7)
    for row, i in enumerate(tokens.tolist()):
        qb = g.block_of_token[i]
        keys = [j for j in range(Q.shape[2]) if keep[0, 0, qb, g.block_of_token[j]]]
        z = [math.exp(0.7 * sum(Q[0, 0, i, c] * K[0, 0, j, c] for c in range(4))) for j in keys]
        tot = sum(z)
        assert abs(lse[0, 0, row] - math.log(tot)) < 1e-12
        for c in range(4):
            o = sum(zj * V[0, 0, j, c] for zj, j in zip(z, keys)) / tot
            assert abs(out[0, 0, row, c] - o) < 1e-12


def test_layer_composes_the_three_steps():
    w = W.TINY
    x = W.generate(w)
    g = O.block_geometry(w.T, w.Hs, w.Ws, w.bt, w.bh, w.bw)
    res = O.layer(x["q"], x["k"], x["v"], g, 1.0, 0, 1 / 8.0)
    dout, dlse = O.dense_attn(x["q"], x["k"], x["v"], 1 / 8.0, res["tokens"])
    np.testing.assert_allclose(res["out"], dout, atol=1e-12)
    np.testing.assert_allclose(res["lse"], dlse, atol=1e-12)


def test_comparison_band_flags_rows_near_p():
    # scores 0.5, 0.3, 0.2: with p = 0.8 the second prefix sum equals p, so fp32
    # rounding may move the cut; the row must be reported ambiguous.
    s = np.array([0.5, 0.3, 0.2])
    Qp = np.tile(np.log(s), (3, 1))[None, None]
    r = O.route(Qp, np.eye(3)[None, None], 0.8, 1, 1.0)
    ex, amb = O.comparison_band(r, 0.8, 1)
    assert amb[0, 0].all()
    r2 = O.route(Qp, np.eye(3)[None, None], 0.6, 1, 1.0)
    ex2, amb2 = O.comparison_band(r2, 0.6, 1)
    assert not amb2.any()


def _route_one(scores, p, k):
    """Every row of a hand-made routing problem has the given scores (Kp = identity, Qp
    rows = ln(scores)); row i differs only in its own block, i."""
    s = np.asarray(scores, dtype=np.float64)
    nB = s.size
    Qp = np.tile(np.log(s), (nB, 1))[None, None]
    r = O.route(Qp, np.eye(nB)[None, None], p, k, 1.0)
    np.testing.assert_allclose(r.scores[0, 0, 0], s / s.sum(), rtol=1e-12)
    return r


# Scores (hand-made, summing to 1):  block 2 is the Top-p cutoff at p = 0.75 (prefix
# 0.5 + 0.2 + 0.1 = 0.8 >= 0.75, two blocks give 0.7); block 3 lies 0.5e-5 below the
# cutoff, block 4 lies 2e-5 below it.
_BAND_ROW = [0.5, 0.2, 0.1, 0.099995, 0.09998, 0.000025]


def test_comparison_band_excludes_only_near_cutoff_blocks_across_the_cut():
    r = _route_one(_BAND_ROW, 0.75, 1)
    assert r.m_keep[0, 0].tolist() == [3] * 6
    ex, amb = O.comparison_band(r, 0.75, 1)
    assert not amb.any()
    # own block 5 (outside the prefix): blocks 2 and 3 may swap places; 4 (2e-5 away) may not
    assert np.nonzero(ex[0, 0, 5])[0].tolist() == [2, 3]
    # own block 3: it is kept either way, so it is not excluded; block 2 still is
    assert np.nonzero(ex[0, 0, 3])[0].tolist() == [2]
    # own block 2 (the cutoff block itself): only block 3 can flip
    assert np.nonzero(ex[0, 0, 2])[0].tolist() == [3]
    # a plain row with no near-cutoff block on the far side excludes nothing
    r2 = _route_one([0.5, 0.2, 0.1, 0.09, 0.08, 0.03], 0.75, 1)
    assert not O.comparison_band(r2, 0.75, 1)[0].any()


def test_comparison_band_cutoff_is_taken_after_the_floor():
    # p = 0.5 keeps one block (0.6); the floor k = 4 lengthens the prefix to block 3
    # (0.05), and block 4 lies 4e-6 below it: the band sits at block 3, not at block 0.
    row = [0.6, 0.2, 0.1, 0.05, 0.049996, 0.000004]
    r = _route_one(row, 0.5, 4)
    assert r.m_p[0, 0, 0] == 1 and r.m_keep[0, 0, 0] == 4
    ex, amb = O.comparison_band(r, 0.5, 4)
    assert np.nonzero(ex[0, 0, 5])[0].tolist() == [3, 4]
    assert not ex[0, 0, 5, :3].any()
    # with the floor at 5 the cut moves past block 4: nothing near it lies outside
    r5 = _route_one(row, 0.5, 5)
    assert not O.comparison_band(r5, 0.5, 5)[0].any()
    # when the floor keeps every block no bit can flip
    r6 = _route_one(row, 0.5, 6)
    assert r6.keep.all() and not O.comparison_band(r6, 0.5, 6)[0].any()


def test_candidate_cuts_and_keep_for_cut():
    # cumulative masses 0.5, 0.8, 1.0: at p = 0.8 the second sum sits on p, so an fp32
    # sum may need one more block (cut 3) -- and the floor takes precedence over both
    s = [0.5, 0.3, 0.2]
    r = _route_one(s, 0.8, 1)
    m_p = int(r.m_p[0, 0, 0])
    cands = O.candidate_cuts(r, 0.8, 1)
    assert sorted(set(cands[0, 0, 0].tolist())) in ([1, 2], [2, 3])
    assert m_p in cands[0, 0, 0]
    assert O.comparison_band(r, 0.8, 1)[1].all()
    r_fl = _route_one(s, 0.8, 3)
    assert (O.candidate_cuts(r_fl, 0.8, 3) == 3).all()
    assert not O.comparison_band(r_fl, 0.8, 3)[1].any()
    # a floor two blocks past m_p: moving the Top-p cut by one changes nothing
    s4 = [0.5, 0.3, 0.1, 0.1]
    for pp in (0.8 - 1e-7, 0.8 + 1e-7):      # the sum at the cut just above / below p
        r4 = _route_one(s4, pp, 4)
        assert (O.candidate_cuts(r4, pp, 4) == 4).all()
        assert not O.comparison_band(r4, pp, 4)[1].any()
        # without the floor the other side of the cut is a candidate: cut 2 moves up to
        # 3 (sum at the cut just above p), or cut 3 down to 2 (just below)
        r1 = _route_one(s4, pp, 1)
        assert r1.m_p[0, 0, 0] == (2 if pp < 0.8 else 3)
        assert sorted(set(O.candidate_cuts(r1, pp, 1)[0, 0, 0].tolist())) == [2, 3]
    # far from p: every candidate is m_keep
    r2 = _route_one(s, 0.6, 1)
    assert (O.candidate_cuts(r2, 0.6, 1) == r2.m_keep[..., None]).all()
    # keep_for_cut: prefix of the order plus the own block
    keep = O.keep_for_cut(r2, np.full((1, 1, 3), 1))
    assert keep[0, 0].astype(int).tolist() == [[1, 0, 0], [1, 1, 0], [1, 0, 1]]
    assert (O.keep_for_cut(r2, r2.m_keep) == r2.keep).all()


# ------------------------------------------------------------------ next rows of the path
def test_token_topp_against_token_level_brute_force():
    """Top-p over tokens, decided per block, against an explicit expansion of every row
    into real tokens (ragged block sizes: partial blocks on every edge)."""
    wl = W.SMALL_RAGGED_T
    x = W.generate(wl)
    g = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    assert len(set(g.real_count.tolist())) > 2
    Qp, Kp = O.pool(x["q"], g), O.pool(x["k"], g)
    scale = 1.0 / math.sqrt(wl.d)
    rng = np.random.default_rng(11)
    ts = O.token_scores(Qp, Kp, scale, g.real_count)
    for p, k in [(0.5, 1), (0.8, 3), (0.95, 0), (1.0, 0), (0.3, 30)]:
        r = O.route(Qp, Kp, p, k, scale, real_count=g.real_count)
        assert np.allclose(r.mass.sum(-1), 1.0)
        for b, h, qb in zip(rng.integers(0, wl.B, 12), rng.integers(0, wl.H, 12), rng.integers(0, g.nB, 12)):
            want = O.brute_force_token_route_row(ts[b, h, qb], g.real_count, qb, p, k)
            assert (r.keep[b, h, qb] == want).all(), (p, k, b, h, qb)
            assert O.check_route_invariants(r.keep[b, h, qb], r.scores[b, h, qb], qb, p, k, 1e-12,
                                            r.mass[b, h, qb]) is None


def test_token_topp_equals_block_topp_when_blocks_are_equal():
    w = W.TINY                                   # every block holds 32 tokens
    x = W.generate(w)
    g = O.block_geometry(w.T, w.Hs, w.Ws, w.bt, w.bh, w.bw)
    Qp, Kp = O.pool(x["q"], g), O.pool(x["k"], g)
    for p, k in [(0.6, 1), (0.9, 2)]:
        a = O.route(Qp, Kp, p, k, 0.125)
        t = O.route(Qp, Kp, p, k, 0.125, real_count=g.real_count)
        assert (a.keep == t.keep).all()
        np.testing.assert_allclose(t.mass, a.scores, rtol=1e-12)


def test_token_topp_hand_row():
    # blocks 0 and 1 share one pooled logit, block 2's is ln 0.5 lower; block 0 holds 96
    # tokens and blocks 1, 2 hold 32 each, so the token masses are 96, 32 and 16 over 144
    # (0.667, 0.222, 0.111) although blocks 0 and 1 tie by score.  At p = 0.6 block 0
    # alone reaches p by token mass.
    nB = 3
    logits = np.log(np.array([1.0, 1.0, 0.5]))
    Qp = np.tile(logits, (nB, 1))[None, None]
    counts = np.array([96, 32, 32])
    r = O.route(Qp, np.eye(nB)[None, None], 0.6, 1, 1.0, real_count=counts)
    np.testing.assert_allclose(r.mass[0, 0, 2], np.array([96, 32, 16]) / 144.0)
    assert r.keep[0, 0, 2].astype(int).tolist() == [1, 0, 1]     # block 0, plus own 2
    # the plain block rule needs both tied blocks (scores 0.4, 0.4, 0.2)
    r0 = O.route(Qp, np.eye(nB)[None, None], 0.6, 1, 1.0)
    assert r0.keep[0, 0, 2].astype(int).tolist() == [1, 1, 1]


def test_keyframe_blocks_hand_cases():
    g = O.block_geometry(10, 4, 4, 1, 4, 4)         # 10 frames, one block per frame
    assert np.nonzero(O.keyframe_blocks(g, 4, 1))[0].tolist() == [1, 5, 9]
    assert np.nonzero(O.keyframe_blocks(g, 4, 0))[0].tolist() == [0, 4, 8]
    assert np.nonzero(O.keyframe_blocks(g, 20, 0))[0].tolist() == [0]
    assert not O.keyframe_blocks(g, 0, 0).any()
    g2 = O.block_geometry(7, 4, 8, 2, 4, 4)         # 2-frame blocks, 4 time blocks x 2 columns
    # keyframes 1 and 4 (stride 3, phase 1; frame 7 does not exist): time blocks 0 and 2
    assert np.nonzero(O.keyframe_blocks(g2, 3, 1))[0].tolist() == [0, 1, 4, 5]
    # phase 2: frames 2 and 5 -> time blocks 1 and 2
    assert np.nonzero(O.keyframe_blocks(g2, 3, 2))[0].tolist() == [2, 3, 4, 5]
    keep = np.zeros((1, 1, 8, 8), bool)
    keep[..., 3, 6] = True
    got = O.add_keyframes(keep, O.keyframe_blocks(g2, 3, 2))
    assert np.nonzero(got[0, 0, 3])[0].tolist() == [2, 3, 4, 5, 6]
    assert np.nonzero(got[0, 0, 0])[0].tolist() == [2, 3, 4, 5]


def test_keyframes_do_not_move_the_topp_cut():
    w = W.SMALL_RAGGED
    x = W.generate(w)
    g = O.block_geometry(w.T, w.Hs, w.Ws, w.bt, w.bh, w.bw)
    Qp, Kp = O.pool(x["q"], g), O.pool(x["k"], g)
    r = O.route(Qp, Kp, 0.8, 2, 1 / math.sqrt(w.d))
    kf = O.keyframe_blocks(g, 2, 1)
    got = O.add_keyframes(r.keep, kf)
    assert (got == (r.keep | kf)).all() and got[..., kf].all()


def _repair_by_coordinates(keep, g):
    out = keep.copy()
    for j in range(g.nB):
        tb, r = divmod(j, g.nBy * g.nBx)
        yb, xb = divmod(r, g.nBx)
        for dt, dy, dx in ((1, 0, 0), (0, 1, 0), (0, 0, 1)):
            a = (tb - dt, yb - dy, xb - dx)
            c = (tb + dt, yb + dy, xb + dx)
            if min(a) < 0 or c[0] >= g.nBt or c[1] >= g.nBy or c[2] >= g.nBx:
                continue
            ja = (a[0] * g.nBy + a[1]) * g.nBx + a[2]
            jc = (c[0] * g.nBy + c[1]) * g.nBx + c[2]
            out[..., j] |= keep[..., ja] & keep[..., jc]
    return out


def test_repair_mask_against_coordinate_loops():
    rng = np.random.default_rng(3)
    for dims in [(4, 3, 5), (1, 1, 7), (3, 1, 1), (2, 4, 4)]:
        g = O.block_geometry(dims[0] * 2, dims[1] * 4, dims[2] * 8 - 3, 2, 4, 8)
        assert (g.nBt, g.nBy, g.nBx) == dims
        for dens in (0.2, 0.5, 0.8):
            keep = rng.random((2, 3, g.nB, g.nB)) < dens
            np.testing.assert_array_equal(O.repair_mask(keep, g), _repair_by_coordinates(keep, g))


def test_repair_mask_hand_case():
    g = O.block_geometry(1, 1, 5, 1, 1, 1)          # five blocks in a row (x axis)
    keep = np.array([1, 0, 1, 0, 0], bool)[None, None, None, :]
    # block 1 is a hole between kept 0 and 2; block 3 is not (4 is dropped); one pass only
    assert O.repair_mask(keep, g)[0, 0, 0].astype(int).tolist() == [1, 1, 1, 0, 0]
    keep2 = np.array([1, 0, 1, 0, 1], bool)[None, None, None, :]
    assert O.repair_mask(keep2, g)[0, 0, 0].astype(int).tolist() == [1, 1, 1, 1, 1]
    # blocks at the ends of an axis have no hole to fill
    keep3 = np.array([0, 1, 0, 0, 1], bool)[None, None, None, :]
    assert O.repair_mask(keep3, g)[0, 0, 0].astype(int).tolist() == [0, 1, 0, 0, 1]


def test_tile_costs_by_token_pairs():
    g = O.block_geometry(3, 5, 7, 2, 4, 4)          # ragged on every axis
    rng = np.random.default_rng(4)
    keep = rng.random((1, 2, g.nB, g.nB)) < 0.4
    cost = O.tile_costs(keep, g.real_count)
    for h in range(2):
        for qb in range(g.nB):
            pairs = sum(len(g.tokens_of_block[qb]) * len(g.tokens_of_block[kb])
                        for kb in range(g.nB) if keep[0, h, qb, kb])
            assert cost[0, h, qb] == pairs


def test_slack_augment_hand_case():
    # a 1 x 1 x 4 latent cut into 1-token blocks: four tiles whose costs are their kept
    # counts.  Rows keep {0}, {0,1}, {0,1,2}, {0,1,2,3}: costs 1, 2, 3, 4.  With 2 SMs the
    # final wave is the two cheapest tiles (rows 0 and 1), c* = 2: row 0 may add one block,
    # row 1 none.
    g = O.block_geometry(1, 1, 4, 1, 1, 1)
    keep = np.zeros((1, 1, 4, 4), bool)
    for i in range(4):
        keep[0, 0, i, :i + 1] = True
    s = np.array([[0.1, 0.2, 0.3, 0.4]] * 4)[None, None]      # block 3 scores highest
    got = O.slack_augment(keep, s, g.real_count, 2, 0.0)
    assert got[0, 0, 0].astype(int).tolist() == [1, 0, 0, 1]      # block 3, then full
    assert (got[0, 0, 1:] == keep[0, 0, 1:]).all()
    # a threshold above every candidate adds nothing
    assert (O.slack_augment(keep, s, g.real_count, 2, 0.5) == keep).all()
    # a threshold between: row 0's best candidate (0.4) passes
    assert O.slack_augment(keep, s, g.real_count, 2, 0.35)[0, 0, 0].astype(int).tolist() == [1, 0, 0, 1]
    # with 4 SMs every tile is in the final wave and c* = 4: rows 0-2 fill to 4 blocks
    got4 = O.slack_augment(keep, s, g.real_count, 4, 0.0)
    assert got4.all()
    # ties in cost: the later index is later in the order (row 1 and a second row 1')
    keep2 = np.zeros((1, 2, 4, 4), bool)
    keep2[0, :, :, 0] = True                       # every tile costs 1
    got2 = O.slack_augment(keep2, np.broadcast_to(s, (1, 2, 4, 4)), g.real_count, 3, 0.0)
    # the final wave is the last three tiles in index order: (h=1, qb 1..3); c* = 1, nothing fits
    assert (got2 == keep2).all()


def test_slack_augment_never_exceeds_the_wave_cap():
    w = W.SMALL_RAGGED
    x = W.generate(w)
    g = O.block_geometry(w.T, w.Hs, w.Ws, w.bt, w.bh, w.bw)
    r = O.route(O.pool(x["q"], g), O.pool(x["k"], g), 0.6, 1, 1 / math.sqrt(w.d))
    for n_sm in (4, 16, 64):
        got = O.slack_augment(r.keep, r.scores, g.real_count, n_sm, 1e-4)
        assert (got >= r.keep).all()
        c0 = O.tile_costs(r.keep, g.real_count).reshape(-1)
        c1 = O.tile_costs(got, g.real_count).reshape(-1)
        order = np.lexsort((np.arange(c0.size), -c0))
        wave = order[-n_sm:]
        assert (c1[wave] <= c0[wave].max()).all()
        changed = np.nonzero(c1 != c0)[0]
        assert set(changed.tolist()) <= set(wave.tolist())
        # added blocks pass the threshold and are the best dropped ones of their row
        fk, fg, fs = r.keep.reshape(c0.size, -1), got.reshape(c0.size, -1), r.scores.reshape(c0.size, -1)
        for t in changed:
            added = fg[t] & ~fk[t]
            assert (fs[t][added] >= 1e-4).all()
            dropped = ~fg[t] & (fs[t] >= 1e-4)
            if dropped.any():
                assert fs[t][added].min() >= fs[t][dropped].max()
