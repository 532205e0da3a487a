"""GPU parity of slack-aware augmentation (fvattn_slack_augment) against the oracle.

FVAttn explainer, 核心方法 §3: the slack idle workers leave before the critical path ends is
filled with high-value blocks filtered by a score threshold.  The kernels take the GPU's
own routed mask and the route workspace's logits; the oracle (oracle.slack_augment) takes
the same mask and fp64 routing scores.  The final wave (integer costs) must match exactly;
a wave row is compared bit for bit unless two of its candidate scores lie within 1e-5 of
each other or of tau (an fp32 order may then differ), where it is checked for the rule's
invariants instead: only candidates of score >= tau added, in score order, cost <= c*."""
import math

import numpy as np
import pytest

import oracle as O
from free_adaptive_block_b200 import workloads as W
from tests import _parity as P



def _tau_in_gap(scores, near):
    """A threshold near `near` with no score within 1e-4 relative of it."""
    s = np.unique(scores.reshape(-1))
    i = int(np.searchsorted(s, near))
    for j in range(max(1, i - 50), min(len(s) - 1, i + 50)):
        lo, hi = s[j - 1], s[j]
        if hi - lo > 2e-4 * hi:
            return float(np.float32((lo + hi) / 2))
    return float(np.float32(near))


@pytest.mark.gpu
@pytest.mark.parametrize("wl,n_sm", [(W.SMALL_RAGGED, 8), (W.SMALL_RAGGED, 64), (W.WAN21_480P, 148),
                                     (W.WAN21_480P, 40)], ids=lambda v: getattr(v, "name", str(v)))
def test_augment_matches_oracle(wl, n_sm):
    import torch
    import free_adaptive_block_b200 as fv
    x = W.generate(wl)
    g = P.geometry(wl)
    og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    sc = P.scale_of(wl.d)
    q, k = P.to_dev(x["q"]), P.to_dev(x["k"])
    b = fv.LayerBuffers.allocate(g)
    fv.fvattn_pool_route(g, q, k, 0.7, 1, sc, b.q_pool, b.k_pool, b.mask, b.counts, b.pool_route_ws)
    torch.cuda.synchronize()
    keep0 = O.unpack_mask(b.mask.cpu().numpy().view(np.uint32), og.nB)
    qp, kp = O.pool(x["q"], og), O.pool(x["k"], og)
    scores = O.routing_scores(qp, kp, sc)
    tau = _tau_in_gap(scores, 1.0 / og.nB)
    fv.fvattn_slack_augment(g, b.pool_route_ws, tau, b.mask, b.counts, b.workspace, n_sm=n_sm)
    torch.cuda.synchronize()
    got = O.unpack_mask(b.mask.cpu().numpy().view(np.uint32), og.nB)
    np.testing.assert_array_equal(b.counts.cpu().numpy(), got.sum(-1))
    want = O.slack_augment(keep0, scores, og.real_count, n_sm, tau)
    T = keep0.shape[0] * keep0.shape[1] * og.nB
    cost0 = O.tile_costs(keep0, og.real_count).reshape(-1)
    order = np.lexsort((np.arange(T), -cost0))
    wave = set(order[-min(n_sm, T):].tolist())
    cap = cost0[list(wave)].max()
    fk, fg, fw, fs = (a.reshape(T, og.nB) for a in (keep0, got, want, scores))
    rc = og.real_count
    exact = loose = 0
    for t in range(T):
        if t not in wave:
            assert (fg[t] == fk[t]).all(), f"tile {t} is outside the wave but changed"
            continue
        cand = fs[t][~fk[t]]
        cs = np.sort(cand[cand >= tau - 1e-5])[::-1]
        near = (np.abs(cand - tau) < 1e-5).any() or (len(cs) > 1 and (np.diff(cs) > -1e-5).any())
        if not near:
            assert (fg[t] == fw[t]).all(), f"wave tile {t} differs from the oracle"
            exact += 1
            continue
        loose += 1
        added = fg[t] & ~fk[t]
        assert (fs[t][added] >= tau - 1e-5).all()
        qb = t % og.nB
        assert rc[qb] * (rc @ fg[t]) <= cap
        rest = ~fg[t] & (fs[t] >= tau + 1e-5)
        if added.any() and rest.any():
            assert fs[t][added].min() >= fs[t][rest].max() - 1e-5
    added_bits = int((got & ~keep0).sum())
    print(wl.name, n_sm, "tau", tau, "wave rows exact", exact, "loose", loose, "bits added", added_bits,
          "cap", int(cap))
    assert exact > 0


def test_augment_argument_checks():
    """Rejected on the host, before any CUDA call."""
    import ctypes
    import free_adaptive_block_b200 as fv
    g = P.geometry(W.WAN21_480P)
    cg = g.c()
    E = {v: k for k, v in fv.STATUS_NAMES.items()}
    L = fv.lib()
    need_r = fv.fvattn_route_workspace_size(g)
    need_s = fv.fvattn_attn_workspace_size(g)
    call = lambda tau=0.01, n_sm=0, ws=0x10000, nr=need_r, scr=0x20000, ns=need_s: L.fvattn_slack_augment(  # noqa
        ctypes.byref(cg), ws, nr, ctypes.c_float(tau), n_sm, 0x3000, 0x4000, scr, ns, None)
    assert call(tau=-1.0) == E["FVATTN_ERR_INVALID_ARG"]
    assert call(tau=math.nan) == E["FVATTN_ERR_INVALID_ARG"]
    assert call(n_sm=-1) == E["FVATTN_ERR_INVALID_ARG"]
    assert call(ws=None) == E["FVATTN_ERR_WORKSPACE"]
    assert call(nr=need_r - 1) == E["FVATTN_ERR_WORKSPACE"]
    assert call(scr=None) == E["FVATTN_ERR_WORKSPACE"]
    assert call(ns=need_s - 1) == E["FVATTN_ERR_WORKSPACE"]
    assert call(ws=0x10004) == E["FVATTN_ERR_UNSUPPORTED"]
    big = fv.Geometry(1, 1, 512, 64, 64, 128, 1, 8, 16)      # 128 * 2^21 tokens >= 2^26
    cb = big.c()
    assert L.fvattn_slack_augment(ctypes.byref(cb), 0x10000, 1 << 40, ctypes.c_float(0.1), 0, 0x3000, 0x4000,
                                  0x20000, 1 << 40, None) == E["FVATTN_ERR_UNSUPPORTED"]
