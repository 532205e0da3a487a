"""The allocation-free attention entry point (fvattn_block_sparse_attn_noalloc).

Some callers cannot allocate device memory where they call the library: runtimes that
plan all device memory ahead and forbid allocation on the serving path, plugins whose
host framework owns every buffer.  For them the library offers a variant of the
block-sparse attention call that takes no workspace and uses a static scratch area of
its own.  This test calls it through the C ABI, twice in a row (the scratch area keeps
the previous call's contents), and checks each result against the workspace-taking
entry point on the same inputs (bit for bit: the kernel is the same and deterministic).
The file is named to be collected last."""
import ctypes

import numpy as np
import pytest

from free_adaptive_block_b200 import workloads as W
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl", [W.SMALL_RAGGED, W.WAN21_480P], ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point(wl):
    import torch
    import free_adaptive_block_b200 as fv
    x = W.generate(wl)
    g = P.geometry(wl)
    sc = P.scale_of(wl.d)
    q, k, v = P.to_dev(x["q"]), P.to_dev(x["k"]), P.to_dev(x["v"])
    b = fv.LayerBuffers.allocate(g)
    fv.fvattn_block_pool(g, q, k, b.q_pool, b.k_pool)
    fv.fvattn_route(g, b.q_pool, b.k_pool, wl.p, wl.k_floor, sc, b.mask, b.counts)
    fv.fvattn_block_sparse_attn(g, q, k, v, b.mask, sc, b.out, b.lse, b.workspace, None)
    torch.cuda.synchronize()
    assert fv.fvattn_device_status(b.workspace) == 0
    ref_out = P.bf16_to_np(b.out).astype(np.float64)
    ref_lse = b.lse.cpu().numpy().astype(np.float64)

    L = fv.lib()
    cg = g.c()
    for _ in range(2):
        out = torch.full_like(b.out, float("nan"))
        lse = torch.full_like(b.lse, float("nan"))
        status = L.fvattn_block_sparse_attn_noalloc(
            ctypes.byref(cg), q.data_ptr(), k.data_ptr(), v.data_ptr(), b.mask.data_ptr(),
            ctypes.c_float(sc), out.data_ptr(), lse.data_ptr(), None,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert status == 0, fv.fvattn_status_string(status)
        torch.cuda.synchronize()
        assert L.fvattn_noalloc_device_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
        got_out = P.bf16_to_np(out).astype(np.float64)
        got_lse = lse.cpu().numpy().astype(np.float64)
        assert np.isfinite(got_out).all() and np.isfinite(got_lse).all()
        e = np.abs(got_out - ref_out)
        assert e.max() <= P.OUT_MAX_ABS and e.mean() <= P.OUT_MEAN_ABS
        assert np.abs(got_lse - ref_lse).max() <= P.LSE_MAX_ABS
        # every tile's result is independent of which CTA ran it and when, so the two
        # entry points agree bit for bit, not just within the tolerance
        assert torch.equal(out.view(torch.int16), b.out.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), b.lse.view(torch.int32))


def test_noalloc_rejects_geometries_beyond_its_scratch():
    import free_adaptive_block_b200 as fv
    # 8 x 64 heads x 2048 blocks = 1 048 576 tiles: more than the 1 MiB scratch holds
    g = fv.Geometry(B=8, H=64, T=128, Hs=16, Ws=16, d=64, bt=1, bh=1, bw=128 // 16 * 2)
    nB, _ = fv.fvattn_num_blocks(g)
    assert 8 * 64 * nB * 8 > (1 << 20)
    cg = g.c()
    st = fv.lib().fvattn_block_sparse_attn_noalloc(ctypes.byref(cg), 16, 16, 16, 16, ctypes.c_float(0.1),
                                                   16, 16, None, None)
    assert fv.STATUS_NAMES[st] == "FVATTN_ERR_WORKSPACE"
