"""The C ABI without a GPU: the library loads, exports every entry point the header
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

import free_adaptive_block_b200 as fv
from free_adaptive_block_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return fv.lib()


def header_functions():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(fvattn_[a-z_]+)\s*\(", src))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n


G480 = fv.Geometry(B=1, H=12, T=21, Hs=30, Ws=52, d=128, bt=1, bh=8, bw=16)


def test_geometry_queries(L):
    assert fv.fvattn_num_blocks(G480) == (336, 11)
    assert fv.fvattn_num_blocks(fv.Geometry(1, 2, 4, 8, 8, 64, 2, 4, 4)) == (8, 1)
    ws = fv.fvattn_attn_workspace_size(G480)
    assert ws >= 256 + 8 * 12 * 336 and ws % 256 == 0


def call_route(L, g, qp=0x1000, kp=0x2000, p=0.9, k=4, scale=0.088, mask=0x3000, counts=0x4000):
    cg = g.c()
    return L.fvattn_route(ctypes.byref(cg), qp, kp, p, k, scale, mask, counts, None)


def test_host_side_argument_checks(L):
    E = {v: k for k, v in fv.STATUS_NAMES.items()}
    assert call_route(L, G480, qp=None) == E["FVATTN_ERR_INVALID_ARG"]
    assert call_route(L, G480, p=float("nan")) == E["FVATTN_ERR_INVALID_ARG"]
    assert call_route(L, G480, p=-0.1) == E["FVATTN_ERR_INVALID_ARG"]
    assert call_route(L, G480, k=-1) == E["FVATTN_ERR_INVALID_ARG"]
    assert call_route(L, G480, scale=0.0) == E["FVATTN_ERR_INVALID_ARG"]
    assert call_route(L, G480, mask=0x3002) == E["FVATTN_ERR_UNSUPPORTED"]     # misaligned word
    assert call_route(L, G480, qp=0x1004) == E["FVATTN_ERR_UNSUPPORTED"]       # pooled rows need 16 B
    bad_d = fv.Geometry(1, 12, 21, 30, 52, 96, 1, 8, 16)
    assert call_route(L, bad_d) == E["FVATTN_ERR_UNSUPPORTED"]
    big_block = fv.Geometry(1, 1, 4, 16, 16, 128, 2, 8, 16)        # 256 tokens per block
    assert call_route(L, big_block) == E["FVATTN_ERR_UNSUPPORTED"]
    zero = fv.Geometry(1, 0, 4, 16, 16, 128, 1, 8, 16)
    assert call_route(L, zero) == E["FVATTN_ERR_INVALID_ARG"]
    # every empty extent is an argument error, for every entry point's geometry check
    for i in range(9):
        ext = [1, 12, 21, 30, 52, 128, 1, 8, 16]
        ext[i] = 0
        assert call_route(L, fv.Geometry(*ext)) == E["FVATTN_ERR_INVALID_ARG"], i
        ext[i] = -3
        assert call_route(L, fv.Geometry(*ext)) == E["FVATTN_ERR_INVALID_ARG"], i
    # limits of the tensor maps and index types
    assert call_route(L, fv.Geometry(1, 1, 1, 8, 65536, 128, 1, 8, 16)) == E["FVATTN_ERR_UNSUPPORTED"]
    assert call_route(L, fv.Geometry(1, 1, 32768, 1, 16, 128, 1, 1, 16)) == E["FVATTN_ERR_UNSUPPORTED"]
    assert call_route(L, fv.Geometry(1, 1, 16, 65535, 2049, 128, 16, 8, 1)) == E["FVATTN_ERR_UNSUPPORTED"]
    assert call_route(L, fv.Geometry(1, 1, 1, 2, 2049 * 64, 64, 1, 2, 64)) == E["FVATTN_ERR_UNSUPPORTED"]
    assert L.fvattn_route(None, 0x1000, 0x2000, 0.9, 4, 0.1, 0x3000, 0x4000, None) == E["FVATTN_ERR_INVALID_ARG"]
    cg = G480.c()
    # attention: missing mask, missing / short workspace
    assert L.fvattn_block_sparse_attn(ctypes.byref(cg), 0x1000, 0x2000, 0x3000, None, 0.1, 0x4000,
                                      0x5000, 0x6000, 1 << 20, None, None) == E["FVATTN_ERR_INVALID_ARG"]
    assert L.fvattn_dense_attn(ctypes.byref(cg), 0x1000, 0x2000, 0x3000, 0.1, 0x4000, 0x5000,
                               None, 1 << 20, None, None) == E["FVATTN_ERR_WORKSPACE"]
    assert L.fvattn_dense_attn(ctypes.byref(cg), 0x1000, 0x2000, 0x3000, 0.1, 0x4000, 0x5000,
                               0x6000, 64, None, None) == E["FVATTN_ERR_WORKSPACE"]
    assert L.fvattn_block_pool(ctypes.byref(cg), 0x1000, None, 0x3000, 0x4000, None) == E["FVATTN_ERR_INVALID_ARG"]
    assert L.fvattn_device_status(None, None) == E["FVATTN_ERR_INVALID_ARG"]
    # two-kernel route: the route checks, then a missing / short / misaligned workspace
    need = fv.fvattn_route_workspace_size(G480)
    assert need == 256 + 12 * 336 * 11 * 32 * 4 + 4 * 12 * 336 * 128 * 4   # header, logits, split rows
    args = (ctypes.byref(cg), 0x1000, 0x2000, 0.9, 4, 0.088, 0x3000, 0x4000)
    assert L.fvattn_route_ws(*args, None, need, None) == E["FVATTN_ERR_WORKSPACE"]
    assert L.fvattn_route_ws(*args, 0x10000, need - 1, None) == E["FVATTN_ERR_WORKSPACE"]
    assert L.fvattn_route_ws(*args, 0x10008, need, None) == E["FVATTN_ERR_UNSUPPORTED"]
    assert L.fvattn_route_ws(ctypes.byref(cg), 0x1000, 0x2000, -1.0, 4, 0.088, 0x3000, 0x4000,
                             0x10000, need, None) == E["FVATTN_ERR_INVALID_ARG"]
    # pool and route in one call: the route workspace
    need_pr = fv.fvattn_pool_route_workspace_size(G480)
    assert need_pr == need
    pr = lambda p=0.9, kf=4, qp=0x5000, ws=0x10000, n=need_pr: L.fvattn_pool_route(
        ctypes.byref(cg), 0x1000, 0x2000, p, kf, 0.088, qp, 0x6000, 0x3000, 0x4000, ws, n, None)
    assert pr(qp=None) == E["FVATTN_ERR_INVALID_ARG"]
    assert pr(p=float("nan")) == E["FVATTN_ERR_INVALID_ARG"]
    assert pr(kf=-2) == E["FVATTN_ERR_INVALID_ARG"]
    assert pr(ws=None) == E["FVATTN_ERR_WORKSPACE"]
    assert pr(n=need_pr - 1) == E["FVATTN_ERR_WORKSPACE"]
    assert pr(ws=0x10008) == E["FVATTN_ERR_UNSUPPORTED"]


def test_route_ex_and_repair_argument_checks(L):
    E = {v: k for k, v in fv.STATUS_NAMES.items()}
    cg = G480.c()
    need = fv.fvattn_route_workspace_size(G480)

    def ex(ws=0x10000, n=need, mask=0x3000, **kw):
        o = fv.RouteOpts(**{**dict(p=0.9, k_floor=4, scale=0.088), **kw})
        return L.fvattn_route_ex(ctypes.byref(cg), 0x1000, 0x2000, ctypes.byref(o), mask, 0x4000, ws, n, None)
    assert L.fvattn_route_ex(ctypes.byref(cg), 0x1000, 0x2000, None, 0x3000, 0x4000, 0x10000, need,
                             None) == E["FVATTN_ERR_INVALID_ARG"]
    assert ex(p=-1.0) == E["FVATTN_ERR_INVALID_ARG"]
    assert ex(k_floor=-1) == E["FVATTN_ERR_INVALID_ARG"]
    assert ex(scale=0.0) == E["FVATTN_ERR_INVALID_ARG"]
    assert ex(token_mass=2) == E["FVATTN_ERR_INVALID_ARG"]
    assert ex(repair=-1) == E["FVATTN_ERR_INVALID_ARG"]
    assert ex(kf_stride=-3) == E["FVATTN_ERR_INVALID_ARG"]
    assert ex(ws=None) == E["FVATTN_ERR_WORKSPACE"]
    assert ex(n=need - 1) == E["FVATTN_ERR_WORKSPACE"]
    assert ex(ws=0x10008) == E["FVATTN_ERR_UNSUPPORTED"]
    assert ex(mask=0x3001) == E["FVATTN_ERR_UNSUPPORTED"]
    assert L.fvattn_mask_repair(None, 0x1000, 0x1000, 0x2000, None) == E["FVATTN_ERR_INVALID_ARG"]
    assert L.fvattn_mask_repair(ctypes.byref(cg), None, 0x1000, 0x2000, None) == E["FVATTN_ERR_INVALID_ARG"]
    assert L.fvattn_mask_repair(ctypes.byref(cg), 0x1000, 0x1002, 0x2000, None) == E["FVATTN_ERR_UNSUPPORTED"]


def test_status_strings(L):
    for code in range(7):
        assert fv.fvattn_status_string(code)
    assert fv.fvattn_status_string(99) == "unknown status"


def test_binding_raises_without_cuda_tensors(L):
    import torch
    q = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)
    g = fv.Geometry(1, 2, 4, 8, 8, 64, 2, 4, 4)
    with pytest.raises(ValueError):
        fv.fvattn_block_pool(g, q, q, torch.zeros(1, 2, 8, 64), torch.zeros(1, 2, 8, 64), stream=0)
