"""The attention kernel's bounded waits, driven to give up on a real GPU without a fault.

fvattn_testing_attn_stall makes every CTA wait, at its first tile, on a barrier that
nothing completes, with a limit of a millisecond.  The wait gives up the way any stuck
wait of the kernel would: the CTA raises its abort flag and the workspace's error word,
every role leaves its loop, armed TMA copies and issued MMAs are drained, tensor memory
is released and the kernel returns.  The host then reads FVATTN_ERR_DEVICE_TIMEOUT from
the workspace, the context stays usable, and the next normal call on the same workspace
reports no error and matches the oracle."""
import ctypes

import numpy as np
import pytest

import oracle as O
from free_adaptive_block_b200 import workloads as W
from tests import _parity as P

@pytest.mark.gpu
@pytest.mark.parametrize("wl", [W.SMALL_RAGGED, W.WAN21_480P], ids=lambda w: w.name)
def test_stalled_wait_reports_timeout_then_recovers(wl):
    import torch
    import free_adaptive_block_b200 as fv
    x = W.generate(wl)
    g = P.geometry(wl)
    sc = P.scale_of(wl.d)
    q, k, v = P.to_dev(x["q"]), P.to_dev(x["k"]), P.to_dev(x["v"])
    b = fv.LayerBuffers.allocate(g)
    fv.fvattn_block_pool(g, q, k, b.q_pool, b.k_pool)
    fv.fvattn_route(g, b.q_pool, b.k_pool, wl.p, wl.k_floor, sc, b.mask, b.counts)
    cg = g.c()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        st = fv.lib().fvattn_testing_attn_stall(
            ctypes.byref(cg), q.data_ptr(), k.data_ptr(), v.data_ptr(), b.mask.data_ptr(), ctypes.c_float(sc),
            b.out.data_ptr(), b.lse.data_ptr(), b.workspace.data_ptr(), b.workspace.numel(),
            ctypes.c_ulonglong(1_000_000), ctypes.c_void_p(stream))
        assert st == 0, fv.fvattn_status_string(st)
        assert fv.STATUS_NAMES[fv.fvattn_device_status(b.workspace)] == "FVATTN_ERR_DEVICE_TIMEOUT"
    # the context is intact and the workspace starts clean on the next call
    b.out.fill_(float("nan"))
    b.lse.fill_(float("nan"))
    fv.fvattn_block_sparse_attn(g, q, k, v, b.mask, sc, b.out, b.lse, b.workspace, b.sm_busy_ns)
    torch.cuda.synchronize()
    assert fv.fvattn_device_status(b.workspace) == 0
    keep = O.unpack_mask(b.mask.cpu().numpy().view(np.uint32), wl.nB)
    res = dict(out=P.bf16_to_np(b.out), lse=b.lse.cpu().numpy())
    qbs = None if wl.nB <= 32 else W.sample_qblocks(wl, 8)
    P.check_attn(wl, x, keep, res, qbs)


def test_stall_hook_argument_checks():
    """Rejected on the host, before any CUDA call (no GPU needed)."""
    import free_adaptive_block_b200 as fv
    g = P.geometry(W.SMALL_RAGGED)
    cg = g.c()
    L = fv.lib()
    args = (ctypes.byref(cg), 16, 16, 16, 16, ctypes.c_float(0.1), 16, 16, 16, 1 << 20)
    E = {v: k for k, v in fv.STATUS_NAMES.items()}
    assert L.fvattn_testing_attn_stall(*args, ctypes.c_ulonglong(0), None) == E["FVATTN_ERR_INVALID_ARG"]
    assert L.fvattn_testing_attn_stall(*args, ctypes.c_ulonglong(10**9), None) == E["FVATTN_ERR_INVALID_ARG"]
