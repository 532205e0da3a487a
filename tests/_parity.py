"""Helpers for the GPU parity tests: run the CUDA path through the Python binding of the
C ABI, and compare with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

import oracle as O
from free_adaptive_block_b200 import workloads as W

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
MASK_BAND = 1e-5


def geometry(wl):
    import free_adaptive_block_b200 as fv
    return fv.Geometry(**wl.geom())


def scale_of(d: int) -> float:
    return float(np.float32(1.0 / math.sqrt(d)))


def to_dev(a: np.ndarray):
    import torch
    return torch.from_numpy(W.bf16_bits(a)).view(torch.bfloat16).cuda()


def bf16_to_np(t) -> np.ndarray:
    import torch
    u = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32)


def gpu_layer(wl, x: Dict[str, np.ndarray], p: float, k: int, dev=None, dense: bool = False):
    """pool -> route -> attention on the GPU; returns host copies of every output."""
    import torch
    import free_adaptive_block_b200 as fv
    g = geometry(wl)
    sc = scale_of(wl.d)
    q, kk, v = dev if dev is not None else (to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]))
    b = fv.LayerBuffers.allocate(g)
    b.out.fill_(float("nan"))
    b.lse.fill_(float("nan"))
    fv.fvattn_block_pool(g, q, kk, b.q_pool, b.k_pool)
    fv.fvattn_route(g, b.q_pool, b.k_pool, p, k, sc, b.mask, b.counts)
    if dense:
        fv.fvattn_dense_attn(g, q, kk, v, sc, b.out, b.lse, b.workspace, b.sm_busy_ns)
    else:
        fv.fvattn_block_sparse_attn(g, q, kk, v, b.mask, sc, b.out, b.lse, b.workspace, b.sm_busy_ns)
    torch.cuda.synchronize()
    assert fv.fvattn_device_status(b.workspace) == 0
    return dict(q_pool=b.q_pool.cpu().numpy(), k_pool=b.k_pool.cpu().numpy(),
                mask=b.mask.cpu().numpy().view(np.uint32), counts=b.counts.cpu().numpy(),
                out=bf16_to_np(b.out), lse=b.lse.cpu().numpy(),
                busy=b.sm_busy_ns.cpu().numpy())


def check_pool(wl, x, res, og=None):
    og = og or O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    qp, kp = O.pool(x["q"], og), O.pool(x["k"], og)
    for got, want in ((res["q_pool"], qp), (res["k_pool"], kp)):
        err = np.abs(got - want).max()
        assert err <= 1e-5 * max(1.0, np.abs(want).max()), f"pool max err {err}"
    return qp, kp


def check_route(wl, qp, kp, res, p, k) -> Dict[str, float]:
    """Bit-exact mask outside the 1e-5 score band and the ambiguous rows; invariants
    (with the oracle's fp64 scores) on the ambiguous rows; counts = popcount."""
    pp = float(np.float32(p))
    r = O.route(qp, kp, pp, k, scale_of(wl.d))
    nB = r.keep.shape[-1]
    gk = O.unpack_mask(res["mask"], nB)
    words = res["mask"].shape[-1]
    if nB % 32:
        tail = res["mask"][..., -1] >> np.uint32(nB % 32)
        assert not tail.any(), "bits past nB must be zero"
    assert (gk.sum(-1) == res["counts"]).all(), "counts must equal the popcount"
    excluded, amb = O.comparison_band(r, pp, k, MASK_BAND)
    diff = (gk != r.keep) & ~excluded
    diff[amb] = False
    bad = np.argwhere(diff.any(-1))
    assert bad.size == 0, f"{len(bad)} rows differ outside the band, first {bad[:3].tolist()}"
    for b, h, qb in np.argwhere(amb):
        why = O.check_route_invariants(gk[b, h, qb], r.scores[b, h, qb], qb, pp, k, tol=MASK_BAND)
        assert why is None, (b, h, qb, why)
    own = np.arange(nB)
    assert gk[..., own, own].all()
    return dict(rows=int(np.prod(amb.shape)), ambiguous=int(amb.sum()),
                excluded=int(excluded.sum()), kept_frac=float(gk.mean()), words=words)


def check_attn(wl, x, keep: np.ndarray, res, qblocks: Optional[Sequence[int]] = None, og=None):
    og = og or O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    tokens, out, lse = O.masked_attn(x["q"], x["k"], x["v"], keep, og, scale_of(wl.d), qblocks)
    got = res["out"][:, :, tokens].astype(np.float64)
    gl = res["lse"][:, :, tokens].astype(np.float64)
    assert np.isfinite(got).all() and np.isfinite(gl).all(), "unwritten or non-finite outputs"
    e = np.abs(got - out)
    el = np.abs(gl - lse)
    assert e.max() <= OUT_MAX_ABS, f"out max-abs {e.max()}"
    assert e.mean() <= OUT_MEAN_ABS, f"out mean-abs {e.mean()}"
    assert el.max() <= LSE_MAX_ABS, f"lse max-abs {el.max()}"
    return dict(out_max=float(e.max()), out_mean=float(e.mean()), lse_max=float(el.max()))
