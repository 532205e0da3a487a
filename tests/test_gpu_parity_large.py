"""GPU parity on the large Wan-shaped workloads and the p x k sweep.

Every mask row is compared with the oracle (bit-exact outside the 1e-5 score band and the
ambiguous rows, invariants on those); out / lse are compared on seeded samples of query
blocks per head that always contain every real-size class of block."""
import numpy as np
import pytest

import oracle as O
from free_adaptive_block_b200 import workloads as W
from tests import _parity as P

pytestmark = pytest.mark.gpu


def _run(wl, x, p, k, sample):
    res = P.gpu_layer(wl, x, p, k)
    og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    qp, kp = P.check_pool(wl, x, res, og)
    st = P.check_route(wl, qp, kp, res, p, k)
    keep = O.unpack_mask(res["mask"], wl.nB)
    at = P.check_attn(wl, x, keep, res, W.sample_qblocks(wl, sample), og)
    busy = res["busy"]
    busy = busy[busy > 0]
    print(f"{wl.name} p={p} k={k}: kept {st['kept_frac']:.3f}, ambiguous rows {st['ambiguous']}/{st['rows']}, "
          f"out max {at['out_max']:.2e} mean {at['out_mean']:.2e}, lse max {at['lse_max']:.2e}, "
          f"SM busy max/mean {busy.max() / busy.mean():.3f}")
    return res


def test_wan22_720p():
    wl = W.WAN22_720P
    _run(wl, W.generate(wl), wl.p, wl.k_floor, 64)


def test_wan21_6x_horizon():
    wl = W.WAN21_6X
    _run(wl, W.generate(wl), wl.p, wl.k_floor, 64)


def test_sweep_480p():
    wl0 = W.WAN21_480P
    x = W.generate(wl0)
    fracs = []
    for wl in W.sweep():
        res = _run(wl, x, wl.p, wl.k_floor, 16)
        fracs.append(O.unpack_mask(res["mask"], wl.nB).mean())
    # more mass or a higher floor never keeps fewer blocks
    f = np.asarray(fracs).reshape(len(W.SWEEP_P), len(W.SWEEP_K))
    assert (np.diff(f, axis=0) >= -1e-12).all() and (np.diff(f, axis=1) >= -1e-12).all()
    assert f[-1].min() == 1.0          # p = 1 keeps everything


def test_route_forms_720p():
    """Both route forms against the oracle at 720p (20 mask words, 630 blocks): the
    one-kernel fvattn_route (fp32 FMA logits, bitwise threshold search) and the workspace
    form (tensor-core logits, histogram selection).  Their arithmetic differs, so each is
    held to the oracle's band on its own."""
    import torch
    import free_adaptive_block_b200 as fv
    wl = W.WAN22_720P
    x = W.generate(wl)
    g = P.geometry(wl)
    sc = P.scale_of(wl.d)
    q, k = P.to_dev(x["q"]), P.to_dev(x["k"])
    b = fv.LayerBuffers.allocate(g)
    fv.fvattn_block_pool(g, q, k, b.q_pool, b.k_pool)
    og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    qp, kp = O.pool(x["q"], og), O.pool(x["k"], og)
    for form in ("route", "route_ws"):
        b.mask.fill_(-1)
        if form == "route":
            fv.fvattn_route(g, b.q_pool, b.k_pool, wl.p, wl.k_floor, sc, b.mask, b.counts)
        else:
            fv.fvattn_route_ws(g, b.q_pool, b.k_pool, wl.p, wl.k_floor, sc, b.mask, b.counts, b.route_ws)
        torch.cuda.synchronize()
        res = dict(mask=b.mask.cpu().numpy().view(np.uint32), counts=b.counts.cpu().numpy())
        print(form, P.check_route(wl, qp, kp, res, wl.p, wl.k_floor))
