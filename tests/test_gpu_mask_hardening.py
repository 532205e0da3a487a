"""Masks that break what fvattn_route guarantees still give defined results in the
attention kernel: set bits at j >= nB in a row's last word are ignored, and a row that
keeps no block gets out = 0 and lse = -inf for its tokens.  Every other row matches the
run on the route's own mask."""
import numpy as np
import pytest

import oracle as O
from free_adaptive_block_b200 import workloads as W

from tests._parity import LSE_MAX_ABS, OUT_MAX_ABS, bf16_to_np, geometry, gpu_layer, scale_of, to_dev

pytestmark = pytest.mark.gpu

CASES = [W.SMALL_RAGGED, W.SMALL_RAGGED_T, W.WAN21_480P]


def attn(wl, dev, mask_np):
    import torch
    import free_adaptive_block_b200 as fv
    g = geometry(wl)
    b = fv.LayerBuffers.allocate(g)
    b.mask.copy_(torch.from_numpy(np.ascontiguousarray(mask_np).view(np.int32)))
    b.out.fill_(float("nan"))
    b.lse.fill_(float("nan"))
    q, k, v = dev
    fv.fvattn_block_sparse_attn(g, q, k, v, b.mask, scale_of(wl.d), b.out, b.lse, b.workspace,
                                b.sm_busy_ns)
    torch.cuda.synchronize()
    assert fv.fvattn_device_status(b.workspace) == 0
    return bf16_to_np(b.out), b.lse.cpu().numpy()


@pytest.fixture(scope="module", params=CASES, ids=lambda w: w.name)
def case(request):
    wl = request.param
    x = W.generate(wl)
    dev = (to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]))
    clean = gpu_layer(wl, x, wl.p, wl.k_floor, dev=dev)["mask"]
    return wl, dev, clean


def test_bits_past_the_last_block_are_ignored(case):
    wl, dev, clean = case
    nB = geometry(wl).nB
    tail = nB % 32
    assert tail, "the cases have a partial last mask word"
    dirty = clean.copy()
    dirty[..., -1] |= np.uint32((0xFFFFFFFF << tail) & 0xFFFFFFFF)
    out0, lse0 = attn(wl, dev, clean)
    out1, lse1 = attn(wl, dev, dirty)
    assert np.array_equal(out0, out1)
    assert np.array_equal(lse0, lse1)


def test_a_row_that_keeps_nothing(case):
    wl, dev, clean = case
    og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    # an interior-side block, and the first two W-edge query blocks of frame 0, which form
    # (part of) a query group when the edge is narrow
    rows = [0, og.nBx - 1, 2 * og.nBx - 1]
    empty = clean.copy()
    for qb in rows:
        empty[0, 0, qb, :] = 0
    out0, lse0 = attn(wl, dev, clean)
    out1, lse1 = attn(wl, dev, empty)
    emptied = np.zeros(out0.shape[2], dtype=bool)
    for qb in rows:
        toks = og.tokens_of_block[qb]
        emptied[toks] = True
        assert np.all(out1[0, 0, toks, :] == 0.0)
        assert np.all(np.isneginf(lse1[0, 0, toks]))
    # every other token: as with the route's mask (the schedule may differ, so within the
    # parity tolerance rather than bit for bit)
    keep = np.ones(out0.shape[:3], dtype=bool)
    keep[0, 0, emptied] = False
    assert np.isfinite(out1[keep]).all() and np.isfinite(lse1[keep]).all()
    assert np.abs(out1[keep] - out0[keep]).max() <= OUT_MAX_ABS
    assert np.abs(lse1[keep] - lse0[keep]).max() <= LSE_MAX_ABS
