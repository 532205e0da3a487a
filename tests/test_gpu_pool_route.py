"""fvattn_pool_route (pool and route in one call) against the two separate calls,
fvattn_block_pool + fvattn_route_ws, whose results the parity tests check against the
oracle: pooled Q and K, mask and counts must be equal bit for bit, on every call."""
import numpy as np
import pytest

from free_adaptive_block_b200 import workloads as W

from tests._parity import geometry, scale_of, to_dev

pytestmark = pytest.mark.gpu

CASES = [W.TINY, W.SMALL_RAGGED, W.SMALL_RAGGED_T, W.WAN21_480P]


def separate(g, q, k, p, kf, sc):
    import torch
    import free_adaptive_block_b200 as fv
    b = fv.LayerBuffers.allocate(g)
    fv.fvattn_block_pool(g, q, k, b.q_pool, b.k_pool)
    fv.fvattn_route_ws(g, b.q_pool, b.k_pool, p, kf, sc, b.mask, b.counts, b.route_ws)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (b.q_pool, b.k_pool, b.mask, b.counts)]


def fused(g, q, k, p, kf, sc, b=None):
    import torch
    import free_adaptive_block_b200 as fv
    b = b or fv.LayerBuffers.allocate(g)
    for t in (b.q_pool, b.k_pool):
        t.fill_(float("nan"))
    b.mask.fill_(-1)
    b.counts.fill_(-1)
    fv.fvattn_pool_route(g, q, k, p, kf, sc, b.q_pool, b.k_pool, b.mask, b.counts, b.pool_route_ws)
    torch.cuda.synchronize()
    assert fv.fvattn_device_status(b.pool_route_ws) == 0
    return [t.cpu().numpy() for t in (b.q_pool, b.k_pool, b.mask, b.counts)]


def assert_same(a, b):
    for x, y, name in zip(a, b, ("q_pool", "k_pool", "mask", "counts")):
        assert x.dtype == y.dtype and x.shape == y.shape, name
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), name


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("p,kf", [(None, None), (0.5, 1), (1.0, 0), (0.0, 0)])
def test_fused_equals_separate(wl, p, kf):
    p = wl.p if p is None else p
    kf = wl.k_floor if kf is None else kf
    x = W.generate(wl)
    g = geometry(wl)
    q, k = to_dev(x["q"]), to_dev(x["k"])
    sc = scale_of(wl.d)
    assert_same(fused(g, q, k, p, kf, sc), separate(g, q, k, p, kf, sc))


def test_fused_repeats_bitwise_480p():
    import free_adaptive_block_b200 as fv
    wl = W.WAN21_480P
    x = W.generate(wl)
    g = geometry(wl)
    q, k = to_dev(x["q"]), to_dev(x["k"])
    sc = scale_of(wl.d)
    ref = separate(g, q, k, wl.p, wl.k_floor, sc)
    b = fv.LayerBuffers.allocate(g)
    for _ in range(20):
        assert_same(fused(g, q, k, wl.p, wl.k_floor, sc, b), ref)


def test_fused_720p():
    wl = W.WAN22_720P
    x = W.generate(wl)
    g = geometry(wl)
    q, k = to_dev(x["q"]), to_dev(x["k"])
    sc = scale_of(wl.d)
    assert_same(fused(g, q, k, wl.p, wl.k_floor, sc), separate(g, q, k, wl.p, wl.k_floor, sc))
