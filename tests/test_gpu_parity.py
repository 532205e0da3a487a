"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases are compared element by element over every query block; the Wan-shaped
workloads compare every mask row and 64 seeded query blocks per head of out / lse
(the sample holds every real-size class of block)."""
import numpy as np
import pytest

import oracle as O
from free_adaptive_block_b200 import workloads as W
from tests import _parity as P

pytestmark = pytest.mark.gpu

SMALL = [W.TINY, W.SMALL_RAGGED, W.SMALL_RAGGED_T]


@pytest.fixture(scope="module")
def inputs():
    cache = {}

    def get(wl):
        if wl.name not in cache:
            cache[wl.name] = W.generate(wl)
        return cache[wl.name]
    return get


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_full_parity(wl, inputs):
    x = inputs(wl)
    res = P.gpu_layer(wl, x, wl.p, wl.k_floor)
    qp, kp = P.check_pool(wl, x, res)
    P.check_route(wl, qp, kp, res, wl.p, wl.k_floor)
    keep = O.unpack_mask(res["mask"], wl.nB)
    P.check_attn(wl, x, keep, res)
    # the oracle's own mask end to end
    r = O.route(qp, kp, float(np.float32(wl.p)), wl.k_floor, P.scale_of(wl.d))
    if (r.keep == keep).all():
        P.check_attn(wl, x, r.keep, res)


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_dense_parity(wl, inputs):
    x = inputs(wl)
    res = P.gpu_layer(wl, x, wl.p, wl.k_floor, dense=True)
    keep = np.ones((wl.B, wl.H, wl.nB, wl.nB), bool)
    P.check_attn(wl, x, keep, res)


@pytest.mark.parametrize("p,k", [(1.0, 0), (0.0, 0), (0.3, 100), (0.5, 1), (0.99, 2)])
def test_small_edge_settings(p, k, inputs):
    wl = W.SMALL_RAGGED
    x = inputs(wl)
    res = P.gpu_layer(wl, x, p, k)
    qp, kp = P.check_pool(wl, x, res)
    P.check_route(wl, qp, kp, res, p, k)
    keep = O.unpack_mask(res["mask"], wl.nB)
    if p >= 1.0 or k >= wl.nB:
        assert keep.all()
    P.check_attn(wl, x, keep, res)


def test_single_block_latent():
    wl = W.Workload("one_block", B=2, H=2, d=128, T=1, Hs=5, Ws=7, bt=1, bh=8, bw=16,
                    p=0.9, k_floor=1, seed=99, kind="block")
    x = W.generate(wl)
    res = P.gpu_layer(wl, x, 0.9, 1)
    assert res["mask"].reshape(-1).tolist() == [1] * 4
    P.check_attn(wl, x, np.ones((2, 2, 1, 1), bool), res)


def test_wan21_480p(inputs):
    wl = W.WAN21_480P
    x = inputs(wl)
    res = P.gpu_layer(wl, x, wl.p, wl.k_floor)
    qp, kp = P.check_pool(wl, x, res)
    st = P.check_route(wl, qp, kp, res, wl.p, wl.k_floor)
    keep = O.unpack_mask(res["mask"], wl.nB)
    P.check_attn(wl, x, keep, res, W.sample_qblocks(wl, 64))
    busy = res["busy"]
    assert (busy > 0).sum() >= min(148, wl.H * wl.nB) * 0.9
    print("480p route", st)


def test_wan21_480p_dense(inputs):
    wl = W.WAN21_480P
    x = inputs(wl)
    res = P.gpu_layer(wl, x, wl.p, wl.k_floor, dense=True)
    keep = np.ones((wl.B, wl.H, wl.nB, wl.nB), bool)
    P.check_attn(wl, x, keep, res, W.sample_qblocks(wl, 16))
