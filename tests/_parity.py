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


CANARY = 128      # elements of guard on each side of every output buffer (>= 256 bytes)


def guarded(shape, dtype, fill, canary_bits: int):
    """An output buffer with CANARY elements of a known bit pattern on both sides, so that a
    write past either end is seen (the kernels index outputs by token, block and row)."""
    import torch
    n = int(np.prod(shape))
    store = torch.empty(n + 2 * CANARY, dtype=dtype, device="cuda")
    ints = {torch.bfloat16: torch.int16, torch.float32: torch.int32, torch.int32: torch.int32}[dtype]
    store.view(ints).fill_(canary_bits)
    body = store[CANARY:CANARY + n].view(shape)
    body.fill_(fill)
    return store, body


def canaries_intact(store, canary_bits: int) -> bool:
    import torch
    ints = {torch.bfloat16: torch.int16, torch.float32: torch.int32, torch.int32: torch.int32}[store.dtype]
    v = store.view(ints)
    return bool((v[:CANARY] == canary_bits).all()) and bool((v[-CANARY:] == canary_bits).all())


def gpu_layer(wl, x: Dict[str, np.ndarray], p: float, k: int, dev=None, dense: bool = False):
    """pool -> route -> attention on the GPU; returns host copies of every output.  Every
    output buffer sits between guard bands that must be unchanged afterwards, and out and
    lse start as NaN and must be finite on every token afterwards."""
    import torch
    import free_adaptive_block_b200 as fv
    g = geometry(wl)
    sc = scale_of(wl.d)
    q, kk, v = dev if dev is not None else (to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]))
    b = fv.LayerBuffers.allocate(g)
    s_out, b.out = guarded(b.out.shape, torch.bfloat16, float("nan"), 0x1357)
    s_lse, b.lse = guarded(b.lse.shape, torch.float32, float("nan"), 0x2468ACE)
    s_mask, b.mask = guarded(b.mask.shape, torch.int32, -1, 0x5A5A5A5)
    s_cnt, b.counts = guarded(b.counts.shape, torch.int32, -1, 0x3C3C3C3)
    fv.fvattn_block_pool(g, q, kk, b.q_pool, b.k_pool)
    fv.fvattn_route(g, b.q_pool, b.k_pool, p, k, sc, b.mask, b.counts)
    if dense:
        fv.fvattn_dense_attn(g, q, kk, v, sc, b.out, b.lse, b.workspace, b.sm_busy_ns)
    else:
        fv.fvattn_block_sparse_attn(g, q, kk, v, b.mask, sc, b.out, b.lse, b.workspace, b.sm_busy_ns)
    torch.cuda.synchronize()
    assert fv.fvattn_device_status(b.workspace) == 0
    for st, bits, name in ((s_out, 0x1357, "out"), (s_lse, 0x2468ACE, "lse"), (s_mask, 0x5A5A5A5, "mask"),
                           (s_cnt, 0x3C3C3C3, "counts")):
        assert canaries_intact(st, bits), f"a kernel wrote outside {name}"
    assert bool(torch.isfinite(b.out).all()), "out has unwritten or non-finite tokens"
    assert bool(torch.isfinite(b.lse).all()), "lse has unwritten or non-finite tokens"
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


def check_route(wl, qp, kp, res, p, k, real_count=None, kf=None) -> Dict[str, float]:
    """Bit-exact mask outside the 1e-5 score band; rows where a prefix sum next to the
    Top-p cut lies within 1e-5 of p must equal the keep set of one of the candidate cuts
    (outside that cut's band) and satisfy the invariants; counts = popcount; bits past nB
    are zero.  Inside the band at most 1 % of the excluded bits may differ (fp32 scores
    reorder only blocks whose fp64 scores nearly tie).  `real_count`: the Top-p runs over
    tokens; `kf` (bool [nB]): keyframe blocks every row keeps on top of the route."""
    pp = float(np.float32(p))
    r = O.route(qp, kp, pp, k, scale_of(wl.d), real_count=real_count)
    post = (lambda keep: keep) if kf is None else (lambda keep: O.add_keyframes(keep, kf))
    r.keep = post(r.keep)
    nB = r.keep.shape[-1]
    gk = O.unpack_mask(res["mask"], nB)
    words = res["mask"].shape[-1]
    if nB % 32:
        tail = res["mask"][..., -1] >> np.uint32(nB % 32)
        assert not tail.any(), "bits past nB must be zero"
    assert (gk.sum(-1) == res["counts"]).all(), "counts must equal the popcount"
    excluded, amb = O.comparison_band(r, pp, k, MASK_BAND)
    diff = (gk != r.keep) & ~excluded
    row_ok = ~diff.any(-1)
    if amb.any():
        cands = O.candidate_cuts(r, pp, k, MASK_BAND)
        for c in (1, 2):
            if (cands[..., c] != r.m_keep).any():
                m = cands[..., c]
                row_ok |= ~((gk != post(O.keep_for_cut(r, m))) & ~O.band_for_cut(r, m, MASK_BAND)).any(-1)
    bad = np.argwhere(~row_ok)
    assert bad.size == 0, f"{len(bad)} rows differ outside the band, first {bad[:3].tolist()}"
    if kf is None:
        for b, h, qb in np.argwhere(amb):
            why = O.check_route_invariants(gk[b, h, qb], r.scores[b, h, qb], qb, pp, k, tol=MASK_BAND,
                                           mass_row=r.mass[b, h, qb])
            assert why is None, (b, h, qb, why)
    own = np.arange(nB)
    assert gk[..., own, own].all()
    in_band = int(((gk != r.keep) & excluded).sum())
    n_ex = int(excluded.sum())
    assert in_band <= max(4, n_ex // 100), f"{in_band} of {n_ex} excluded bits differ"
    return dict(rows=int(np.prod(amb.shape)), ambiguous=int(amb.sum()),
                ambiguous_rows_moved=int((amb & ((gk != r.keep) & ~excluded).any(-1)).sum()),
                excluded=n_ex, excluded_differ=in_band, kept_frac=float(gk.mean()), words=words)


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
