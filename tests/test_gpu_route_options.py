"""GPU parity of the routing options (fvattn_route_ex) and of runtime mask repair
(fvattn_mask_repair) against the oracle.

* Top-p over tokens (FVAttn explainer, 核心方法 §1: the minimal token set reaching p,
  decided per 3D block): masks bit-exact outside the 1e-5 band on ragged geometries whose
  edge blocks hold fewer tokens, and at 480p.
* Keyframe blocks (LVSA README, rotating keyframes): every row keeps the blocks holding a
  keyframe frame, at several phases, on the 6x-horizon workload; the attention over that
  mask matches the oracle on sampled query blocks.
* Mask repair (explainer §1, 运行时修补): bit-exact against the oracle's repair of the
  same mask, for the GPU's own routed masks and for random masks with stray bits past nB.
* With every option off, fvattn_route_ex equals fvattn_route_ws bit for bit."""
import numpy as np
import pytest

import oracle as O
from free_adaptive_block_b200 import workloads as W
from tests import _parity as P

pytestmark = pytest.mark.gpu


def _route_ex(wl, x, **kw):
    import torch
    import free_adaptive_block_b200 as fv
    g = P.geometry(wl)
    q, k = P.to_dev(x["q"]), P.to_dev(x["k"])
    b = fv.LayerBuffers.allocate(g)
    fv.fvattn_block_pool(g, q, k, b.q_pool, b.k_pool)
    o = fv.RouteOpts(p=kw.pop("p", wl.p), k_floor=kw.pop("k_floor", wl.k_floor), scale=P.scale_of(wl.d), **kw)
    fv.fvattn_route_ex(g, b.q_pool, b.k_pool, o, b.mask, b.counts, b.route_ws)
    torch.cuda.synchronize()
    return b, dict(q_pool=b.q_pool.cpu().numpy(), k_pool=b.k_pool.cpu().numpy(),
                   mask=b.mask.cpu().numpy().view(np.uint32), counts=b.counts.cpu().numpy())


@pytest.mark.parametrize("wl", [W.SMALL_RAGGED, W.SMALL_RAGGED_T, W.WAN21_480P], ids=lambda w: w.name)
@pytest.mark.parametrize("pk", [None, (0.5, 1), (0.95, 2)])
def test_token_topp(wl, pk):
    p, k = pk if pk else (wl.p, wl.k_floor)
    x = W.generate(wl)
    og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    _, res = _route_ex(wl, x, p=p, k_floor=k, token_mass=1)
    qp, kp = P.check_pool(wl, x, res, og)
    st = P.check_route(wl, qp, kp, res, p, k, real_count=og.real_count)
    # the rule differs from the block rule wherever edge blocks are kept or cut
    plain = O.route(qp, kp, float(np.float32(p)), k, P.scale_of(wl.d))
    print(wl.name, p, k, st, "rows differing from the block rule",
          int((O.unpack_mask(res["mask"], og.nB) != plain.keep).any(-1).sum()))


def test_token_topp_long_rows():
    """Top-p over tokens on rows of more than 16 mask words (720p: 630 blocks, 20 words),
    where the workspace route takes the tensor-core logits and the histogram selection
    with token-weighted masses."""
    wl = W.WAN22_720P
    x = W.generate(wl)
    og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    _, res = _route_ex(wl, x, token_mass=1)
    qp, kp = P.check_pool(wl, x, res, og)
    st = P.check_route(wl, qp, kp, res, wl.p, wl.k_floor, real_count=og.real_count)
    print(wl.name, st)


@pytest.mark.parametrize("stride,phase", [(20, 0), (20, 7), (13, 5)])
def test_keyframes_6x(stride, phase):
    import torch
    import free_adaptive_block_b200 as fv
    wl = W.WAN21_6X
    x = W.generate(wl)
    og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    b, res = _route_ex(wl, x, kf_stride=stride, kf_phase=phase)
    qp, kp = P.check_pool(wl, x, res, og)
    kf = O.keyframe_blocks(og, stride, phase)
    st = P.check_route(wl, qp, kp, res, wl.p, wl.k_floor, kf=kf)
    gk = O.unpack_mask(res["mask"], og.nB)
    assert gk[..., kf].all()
    if (stride, phase) == (20, 0):
        g = P.geometry(wl)
        q, k, v = P.to_dev(x["q"]), P.to_dev(x["k"]), P.to_dev(x["v"])
        b.out.fill_(float("nan"))
        b.lse.fill_(float("nan"))
        fv.fvattn_block_sparse_attn(g, q, k, v, b.mask, P.scale_of(wl.d), b.out, b.lse, b.workspace, None)
        torch.cuda.synchronize()
        assert fv.fvattn_device_status(b.workspace) == 0
        assert bool(torch.isfinite(b.out).all()) and bool(torch.isfinite(b.lse).all())
        at = P.check_attn(wl, x, gk, dict(out=P.bf16_to_np(b.out), lse=b.lse.cpu().numpy()),
                          W.sample_qblocks(wl, 16), og)
        print("6x keyframes", st, at)


@pytest.mark.parametrize("wl", [W.SMALL_RAGGED, W.WAN21_480P, W.WAN21_6X], ids=lambda w: w.name)
def test_repair_of_routed_mask(wl):
    import torch
    import free_adaptive_block_b200 as fv
    x = W.generate(wl)
    og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    b, res = _route_ex(wl, x)
    g = P.geometry(wl)
    out = torch.empty_like(b.mask)
    cnt = torch.empty_like(b.counts)
    fv.fvattn_mask_repair(g, b.mask, out, cnt)
    torch.cuda.synchronize()
    keep = O.unpack_mask(res["mask"], og.nB)
    want = O.repair_mask(keep, og)
    got = O.unpack_mask(out.cpu().numpy().view(np.uint32), og.nB)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(cnt.cpu().numpy(), want.sum(-1))
    # the same through the route option, in place
    b2, res2 = _route_ex(wl, x, repair=1)
    np.testing.assert_array_equal(O.unpack_mask(res2["mask"], og.nB), want)
    np.testing.assert_array_equal(res2["counts"], want.sum(-1))
    print(wl.name, "bits restored", int(want.sum() - keep.sum()), "of", int(keep.size))


def test_repair_random_masks_with_stray_bits():
    import torch
    import free_adaptive_block_b200 as fv
    rng = np.random.default_rng(8)
    for wl in (W.SMALL_RAGGED_T, W.TINY, W.WAN22_720P):
        og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
        g = P.geometry(wl)
        for dens in (0.1, 0.5, 0.9):
            keep = rng.random((wl.B, wl.H, og.nB, og.nB)) < dens
            words = O.pack_mask(keep)
            if og.nB % 32:                                  # stray bits past nB
                words[..., -1] |= np.uint32(0xFFFFFFFF) << np.uint32(og.nB % 32)
            m = torch.from_numpy(words.view(np.int32)).cuda()
            cnt = torch.empty((wl.B, wl.H, og.nB), dtype=torch.int32, device="cuda")
            fv.fvattn_mask_repair(g, m, m, cnt)            # in place
            torch.cuda.synchronize()
            got_w = m.cpu().numpy().view(np.uint32)
            want = O.repair_mask(keep, og)
            np.testing.assert_array_equal(O.unpack_mask(got_w, og.nB), want)
            if og.nB % 32:
                assert not (got_w[..., -1] >> np.uint32(og.nB % 32)).any()
            np.testing.assert_array_equal(cnt.cpu().numpy(), want.sum(-1))


@pytest.mark.parametrize("wl", [W.SMALL_RAGGED_T, W.WAN22_720P], ids=lambda w: w.name)
def test_route_ex_defaults_equal_route_ws(wl):
    import torch
    import free_adaptive_block_b200 as fv
    x = W.generate(wl)
    b, res = _route_ex(wl, x)
    g = P.geometry(wl)
    m2, c2 = torch.empty_like(b.mask), torch.empty_like(b.counts)
    fv.fvattn_route_ws(g, b.q_pool, b.k_pool, wl.p, wl.k_floor, P.scale_of(wl.d), m2, c2, b.route_ws)
    torch.cuda.synchronize()
    assert torch.equal(b.mask, m2) and torch.equal(b.counts, c2)
