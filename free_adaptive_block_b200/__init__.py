"""Python binding of libfvattn: adaptive block-sparse attention for video DiTs on B200.

Argument marshalling only: every step of the path runs in the library's CUDA kernels
(sm_100a).  PyTorch provides device memory and streams.  There is no CPU fallback:
if ``libfvattn.so`` is missing or cannot be loaded, every call raises.

Entry points mirror the C ABI in ``include/fvattn.h``:

* ``fvattn_block_pool``   3D block mean-pooling of Q and K
* ``fvattn_route``        per-head Top-p routing with a Top-k floor -> packed mask, counts
* ``fvattn_route_ws``     the same routing in two kernels through a caller-owned workspace
* ``fvattn_block_sparse_attn``  attention over the kept key blocks -> out, lse
* ``fvattn_dense_attn``   the same kernel with every key block kept

and ``attention_layer`` strings the three steps together for one layer; ``LayerGraph``
captures that layer once in a CUDA graph and replays it.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

__all__ = [
    "Geometry", "FvattnError", "lib", "fvattn_num_blocks", "fvattn_block_pool", "fvattn_route",
    "fvattn_attn_workspace_size", "fvattn_num_sms", "fvattn_block_sparse_attn",
    "fvattn_route_workspace_size", "fvattn_route_ws", "fvattn_pool_route_workspace_size",
    "fvattn_pool_route", "RouteOpts", "fvattn_route_ex", "fvattn_mask_repair", "fvattn_slack_augment",
    "fvattn_dense_attn", "fvattn_block_sparse_attn_noalloc", "fvattn_noalloc_device_status", "fvattn_device_status", "fvattn_status_string", "attention_layer",
    "LayerBuffers", "LayerGraph", "HostPipeline",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfvattn.so")

FVATTN_OK = 0
STATUS_NAMES = {0: "FVATTN_OK", 1: "FVATTN_ERR_INVALID_ARG", 2: "FVATTN_ERR_UNSUPPORTED",
                3: "FVATTN_ERR_WORKSPACE", 4: "FVATTN_ERR_CUDA", 5: "FVATTN_ERR_DEVICE_TIMEOUT",
                6: "FVATTN_ERR_DEVICE"}


class FvattnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        detail = fvattn_status_string(status)
        if status == 4:
            detail += ": " + lib().fvattn_last_cuda_error().decode()
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)} ({detail})")


class _CGeom(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "T", "Hs", "Ws", "d", "bt", "bh", "bw")]


class RouteOpts(ctypes.Structure):
    """fvattn_route_opts_t: Top-p mass, floor and scale, plus the optional frontend steps
    (token-level Top-p masses, keyframe blocks, runtime mask repair)."""
    _fields_ = [("p", ctypes.c_float), ("k_floor", ctypes.c_int), ("scale", ctypes.c_float),
                ("token_mass", ctypes.c_int), ("kf_stride", ctypes.c_int), ("kf_phase", ctypes.c_int),
                ("repair", ctypes.c_int)]


@dataclasses.dataclass(frozen=True)
class Geometry:
    B: int
    H: int
    T: int
    Hs: int
    Ws: int
    d: int
    bt: int
    bh: int
    bw: int

    @property
    def N(self) -> int:
        return self.T * self.Hs * self.Ws

    @property
    def nB(self) -> int:
        return (-(-self.T // self.bt)) * (-(-self.Hs // self.bh)) * (-(-self.Ws // self.bw))

    @property
    def words(self) -> int:
        return -(-self.nB // 32)

    def c(self) -> _CGeom:
        return _CGeom(self.B, self.H, self.T, self.Hs, self.Ws, self.d, self.bt, self.bh, self.bw)


_lib = None

_SIGS = {
    "fvattn_num_blocks": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "fvattn_block_pool": (ctypes.c_int, [ctypes.c_void_p] * 6),
    "fvattn_route": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                    ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p]),
    "fvattn_attn_workspace_size": (ctypes.c_size_t, [ctypes.c_void_p]),
    "fvattn_route_workspace_size": (ctypes.c_size_t, [ctypes.c_void_p]),
    "fvattn_route_ws": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                       ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "fvattn_num_sms": (ctypes.c_int, []),
    "fvattn_pool_route_workspace_size": (ctypes.c_size_t, [ctypes.c_void_p]),
    "fvattn_pool_route": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                         ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                         ctypes.c_void_p]),
    "fvattn_block_sparse_attn": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]),
    "fvattn_dense_attn": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                         ctypes.c_void_p, ctypes.c_void_p]),
    "fvattn_block_sparse_attn_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                        ctypes.c_void_p]),
    "fvattn_device_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "fvattn_noalloc_device_status": (ctypes.c_int, [ctypes.c_void_p]),
    "fvattn_route_ex": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                       ctypes.c_void_p]),
    "fvattn_mask_repair": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p]),
    "fvattn_slack_augment": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float,
                                            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_size_t, ctypes.c_void_p]),
    "fvattn_testing_attn_stall": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_size_t, ctypes.c_ulonglong, ctypes.c_void_p]),
    "fvattn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fvattn_last_cuda_error": (ctypes.c_char_p, []),
}


def lib() -> ctypes.CDLL:
    """Load libfvattn.so (built in-tree by ``_build.py`` / ``__graft_entry__.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m free_adaptive_block_b200._build` (nvcc, sm_100a)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = args
        _lib = handle
    return _lib


def fvattn_status_string(status: int) -> str:
    return lib().fvattn_status_string(int(status)).decode()


def _ok(fn: str, status: int) -> None:
    if status != FVATTN_OK:
        raise FvattnError(fn, status)


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _current_device() -> int:
    import torch
    return torch.cuda.current_device()


def _ptr(t, dtype, shape, name):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    dev = _current_device()
    if t.device.index != dev:
        # the kernels run on the current device and would fault on another GPU's memory
        raise ValueError(f"{name} is on cuda:{t.device.index}, but the current device is cuda:{dev}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def fvattn_num_blocks(g: Geometry):
    nB, words = ctypes.c_int(), ctypes.c_int()
    cg = g.c()
    _ok("fvattn_num_blocks", lib().fvattn_num_blocks(ctypes.byref(cg), ctypes.byref(nB), ctypes.byref(words)))
    return nB.value, words.value


def fvattn_block_pool(g: Geometry, q, k, q_pool, k_pool, stream=None) -> None:
    import torch
    tok = (g.B, g.H, g.N, g.d)
    pooled = (g.B, g.H, g.nB, g.d)
    cg = g.c()
    _ok("fvattn_block_pool", lib().fvattn_block_pool(
        ctypes.byref(cg), _ptr(q, torch.bfloat16, tok, "q"), _ptr(k, torch.bfloat16, tok, "k"),
        _ptr(q_pool, torch.float32, pooled, "q_pool"), _ptr(k_pool, torch.float32, pooled, "k_pool"),
        _stream(stream)))


def fvattn_route(g: Geometry, q_pool, k_pool, p: float, k_floor: int, scale: float, mask, counts,
                 stream=None) -> None:
    import torch
    pooled = (g.B, g.H, g.nB, g.d)
    cg = g.c()
    _ok("fvattn_route", lib().fvattn_route(
        ctypes.byref(cg), _ptr(q_pool, torch.float32, pooled, "q_pool"),
        _ptr(k_pool, torch.float32, pooled, "k_pool"), float(p), int(k_floor), float(scale),
        _ptr(mask, torch.int32, (g.B, g.H, g.nB, g.words), "mask"),
        _ptr(counts, torch.int32, (g.B, g.H, g.nB), "counts"), _stream(stream)))


def fvattn_route_workspace_size(g: Geometry) -> int:
    cg = g.c()
    return int(lib().fvattn_route_workspace_size(ctypes.byref(cg)))


def fvattn_route_ws(g: Geometry, q_pool, k_pool, p: float, k_floor: int, scale: float, mask, counts,
                    workspace, stream=None) -> None:
    import torch
    pooled = (g.B, g.H, g.nB, g.d)
    cg = g.c()
    _ok("fvattn_route_ws", lib().fvattn_route_ws(
        ctypes.byref(cg), _ptr(q_pool, torch.float32, pooled, "q_pool"),
        _ptr(k_pool, torch.float32, pooled, "k_pool"), float(p), int(k_floor), float(scale),
        _ptr(mask, torch.int32, (g.B, g.H, g.nB, g.words), "mask"),
        _ptr(counts, torch.int32, (g.B, g.H, g.nB), "counts"),
        _ptr(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream)))


def fvattn_route_ex(g: Geometry, q_pool, k_pool, opts: RouteOpts, mask, counts, workspace,
                    stream=None) -> None:
    """fvattn_route_ws with the options of ``RouteOpts`` (token-level Top-p, keyframes,
    mask repair)."""
    import torch
    pooled = (g.B, g.H, g.nB, g.d)
    cg = g.c()
    _ok("fvattn_route_ex", lib().fvattn_route_ex(
        ctypes.byref(cg), _ptr(q_pool, torch.float32, pooled, "q_pool"),
        _ptr(k_pool, torch.float32, pooled, "k_pool"), ctypes.byref(opts),
        _ptr(mask, torch.int32, (g.B, g.H, g.nB, g.words), "mask"),
        _ptr(counts, torch.int32, (g.B, g.H, g.nB), "counts"),
        _ptr(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream)))


def fvattn_mask_repair(g: Geometry, mask_in, mask_out, counts, stream=None) -> None:
    """Runtime mask repair: one-block holes of every row filled (mask_out may be mask_in)."""
    import torch
    shape = (g.B, g.H, g.nB, g.words)
    cg = g.c()
    _ok("fvattn_mask_repair", lib().fvattn_mask_repair(
        ctypes.byref(cg), _ptr(mask_in, torch.int32, shape, "mask_in"), _ptr(mask_out, torch.int32, shape, "mask_out"),
        _ptr(counts, torch.int32, (g.B, g.H, g.nB), "counts"), _stream(stream)))


def fvattn_slack_augment(g: Geometry, route_workspace, tau: float, mask, counts, scratch, n_sm: int = 0,
                         stream=None) -> None:
    """Slack-aware augmentation of the final wave of tiles, in place on mask and counts;
    route_workspace holds the logits of the route call that wrote the mask."""
    import torch
    cg = g.c()
    _ok("fvattn_slack_augment", lib().fvattn_slack_augment(
        ctypes.byref(cg), _ptr(route_workspace, torch.uint8, None, "route_workspace"), route_workspace.numel(),
        float(tau), int(n_sm), _ptr(mask, torch.int32, (g.B, g.H, g.nB, g.words), "mask"),
        _ptr(counts, torch.int32, (g.B, g.H, g.nB), "counts"), _ptr(scratch, torch.uint8, None, "scratch"),
        scratch.numel(), _stream(stream)))


def fvattn_pool_route_workspace_size(g: Geometry) -> int:
    cg = g.c()
    return int(lib().fvattn_pool_route_workspace_size(ctypes.byref(cg)))


def fvattn_pool_route(g: Geometry, q, k, p: float, k_floor: int, scale: float, q_pool, k_pool, mask,
                      counts, workspace, stream=None) -> None:
    """fvattn_block_pool then fvattn_route_ws in one call (the same kernels); same results."""
    import torch
    tok = (g.B, g.H, g.N, g.d)
    pooled = (g.B, g.H, g.nB, g.d)
    cg = g.c()
    _ok("fvattn_pool_route", lib().fvattn_pool_route(
        ctypes.byref(cg), _ptr(q, torch.bfloat16, tok, "q"), _ptr(k, torch.bfloat16, tok, "k"),
        float(p), int(k_floor), float(scale), _ptr(q_pool, torch.float32, pooled, "q_pool"),
        _ptr(k_pool, torch.float32, pooled, "k_pool"),
        _ptr(mask, torch.int32, (g.B, g.H, g.nB, g.words), "mask"),
        _ptr(counts, torch.int32, (g.B, g.H, g.nB), "counts"),
        _ptr(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream)))


def fvattn_attn_workspace_size(g: Geometry) -> int:
    cg = g.c()
    return int(lib().fvattn_attn_workspace_size(ctypes.byref(cg)))


def fvattn_num_sms() -> int:
    return int(lib().fvattn_num_sms())


def _check_busy(sm_busy_ns) -> None:
    """The kernel writes one entry per CTA, up to one per SM."""
    if sm_busy_ns is not None and sm_busy_ns.numel() < fvattn_num_sms():
        raise ValueError(f"sm_busy_ns needs fvattn_num_sms() = {fvattn_num_sms()} entries, "
                         f"got {sm_busy_ns.numel()}")


def fvattn_block_sparse_attn(g: Geometry, q, k, v, mask, scale: float, out, lse, workspace,
                             sm_busy_ns=None, stream=None) -> None:
    import torch
    _check_busy(sm_busy_ns)
    tok = (g.B, g.H, g.N, g.d)
    cg = g.c()
    _ok("fvattn_block_sparse_attn", lib().fvattn_block_sparse_attn(
        ctypes.byref(cg), _ptr(q, torch.bfloat16, tok, "q"), _ptr(k, torch.bfloat16, tok, "k"),
        _ptr(v, torch.bfloat16, tok, "v"), _ptr(mask, torch.int32, (g.B, g.H, g.nB, g.words), "mask"),
        float(scale), _ptr(out, torch.bfloat16, tok, "out"), _ptr(lse, torch.float32, tok[:3], "lse"),
        _ptr(workspace, torch.uint8, None, "workspace"), workspace.numel(),
        _ptr(sm_busy_ns, torch.int64, None, "sm_busy_ns"), _stream(stream)))


def fvattn_dense_attn(g: Geometry, q, k, v, scale: float, out, lse, workspace, sm_busy_ns=None,
                      stream=None) -> None:
    import torch
    _check_busy(sm_busy_ns)
    tok = (g.B, g.H, g.N, g.d)
    cg = g.c()
    _ok("fvattn_dense_attn", lib().fvattn_dense_attn(
        ctypes.byref(cg), _ptr(q, torch.bfloat16, tok, "q"), _ptr(k, torch.bfloat16, tok, "k"),
        _ptr(v, torch.bfloat16, tok, "v"), float(scale), _ptr(out, torch.bfloat16, tok, "out"),
        _ptr(lse, torch.float32, tok[:3], "lse"), _ptr(workspace, torch.uint8, None, "workspace"),
        workspace.numel(), _ptr(sm_busy_ns, torch.int64, None, "sm_busy_ns"), _stream(stream)))


def fvattn_block_sparse_attn_noalloc(g: Geometry, q, k, v, mask, scale: float, out, lse,
                                     sm_busy_ns=None, stream=None) -> None:
    """fvattn_block_sparse_attn without a workspace argument: for callers that cannot
    allocate device memory; the library uses its own static scratch area instead."""
    import torch
    _check_busy(sm_busy_ns)
    tok = (g.B, g.H, g.N, g.d)
    cg = g.c()
    _ok("fvattn_block_sparse_attn_noalloc", lib().fvattn_block_sparse_attn_noalloc(
        ctypes.byref(cg), _ptr(q, torch.bfloat16, tok, "q"), _ptr(k, torch.bfloat16, tok, "k"),
        _ptr(v, torch.bfloat16, tok, "v"), _ptr(mask, torch.int32, (g.B, g.H, g.nB, g.words), "mask"),
        float(scale), _ptr(out, torch.bfloat16, tok, "out"), _ptr(lse, torch.float32, tok[:3], "lse"),
        _ptr(sm_busy_ns, torch.int64, None, "sm_busy_ns"), _stream(stream)))


def fvattn_noalloc_device_status(stream=None) -> int:
    """Status of the last fvattn_block_sparse_attn_noalloc call on the current device."""
    return int(lib().fvattn_noalloc_device_status(_stream(stream)))


def fvattn_device_status(workspace, stream=None) -> int:
    import torch
    return int(lib().fvattn_device_status(_ptr(workspace, torch.uint8, None, "workspace"),
                                          _stream(stream)))


@dataclasses.dataclass
class LayerBuffers:
    """Device buffers of one layer (allocated with torch)."""
    q_pool: "object"
    k_pool: "object"
    mask: "object"
    counts: "object"
    out: "object"
    lse: "object"
    workspace: "object"
    sm_busy_ns: "object"
    route_ws: "object" = None   # workspace of fvattn_route_ws (None: the one-kernel route)
    pool_route_ws: "object" = None   # workspace of fvattn_pool_route (used when present)

    @classmethod
    def allocate(cls, g: Geometry, device="cuda") -> "LayerBuffers":
        import torch
        ws = torch.empty(fvattn_attn_workspace_size(g), dtype=torch.uint8, device=device)
        return cls(q_pool=torch.empty(g.B, g.H, g.nB, g.d, dtype=torch.float32, device=device),
                   k_pool=torch.empty(g.B, g.H, g.nB, g.d, dtype=torch.float32, device=device),
                   mask=torch.empty(g.B, g.H, g.nB, g.words, dtype=torch.int32, device=device),
                   counts=torch.empty(g.B, g.H, g.nB, dtype=torch.int32, device=device),
                   out=torch.empty(g.B, g.H, g.N, g.d, dtype=torch.bfloat16, device=device),
                   lse=torch.empty(g.B, g.H, g.N, dtype=torch.float32, device=device),
                   workspace=ws,
                   sm_busy_ns=torch.zeros(max(1, fvattn_num_sms()), dtype=torch.int64, device=device),
                   route_ws=torch.empty(fvattn_route_workspace_size(g), dtype=torch.uint8, device=device),
                   pool_route_ws=torch.empty(fvattn_pool_route_workspace_size(g), dtype=torch.uint8,
                                             device=device))


def attention_layer(g: Geometry, q, k, v, p: float, k_floor: int, scale: Optional[float] = None,
                    buffers: Optional[LayerBuffers] = None, stream=None) -> LayerBuffers:
    """One adaptive block-sparse attention layer: pool -> route -> block-sparse attention.
    Returns the buffers holding mask, counts, out and lse (asynchronous on `stream`)."""
    if scale is None:
        scale = 1.0 / math.sqrt(g.d)
    b = buffers if buffers is not None else LayerBuffers.allocate(g, q.device)
    if b.pool_route_ws is not None:
        fvattn_pool_route(g, q, k, p, k_floor, scale, b.q_pool, b.k_pool, b.mask, b.counts, b.pool_route_ws,
                          stream)
    else:
        fvattn_block_pool(g, q, k, b.q_pool, b.k_pool, stream)
        if b.route_ws is not None:
            fvattn_route_ws(g, b.q_pool, b.k_pool, p, k_floor, scale, b.mask, b.counts, b.route_ws, stream)
        else:
            fvattn_route(g, b.q_pool, b.k_pool, p, k_floor, scale, b.mask, b.counts, stream)
    fvattn_block_sparse_attn(g, q, k, v, b.mask, scale, b.out, b.lse, b.workspace, b.sm_busy_ns, stream)
    return b


class LayerGraph:
    """One attention layer (pool -> route -> block-sparse attention) captured once in a
    CUDA graph and replayed.

    A replay launches the layer's kernels (pool, route, the two schedule-prep kernels and
    attention) with no host work in between: argument checks, tensor-map encoding and the
    launch configuration happen once, at capture.  Everything the calls were given is
    fixed in the graph: q, k, v and the buffers must stay allocated, at the same
    addresses, with the same shapes; to run on new inputs, copy them into ``q``, ``k``,
    ``v`` (for instance from pinned host memory on the same stream) before ``replay``.
    p, k_floor and scale are fixed as well."""

    def __init__(self, g: Geometry, q, k, v, p: float, k_floor: int, scale: Optional[float] = None,
                 buffers: Optional[LayerBuffers] = None):
        import torch
        self.g, self.q, self.k, self.v = g, q, k, v
        self.p, self.k_floor = float(p), int(k_floor)
        self.scale = 1.0 / math.sqrt(g.d) if scale is None else float(scale)
        self.buffers = buffers if buffers is not None else LayerBuffers.allocate(g, q.device)
        # one uncaptured run on a side stream first (module loading, kernel attributes)
        side = torch.cuda.Stream(q.device)
        side.wait_stream(torch.cuda.current_stream(q.device))
        with torch.cuda.stream(side):
            attention_layer(g, q, k, v, self.p, self.k_floor, self.scale, self.buffers)
        torch.cuda.current_stream(q.device).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            attention_layer(g, q, k, v, self.p, self.k_floor, self.scale, self.buffers)

    def replay(self) -> LayerBuffers:
        """Launches the captured layer on the current stream; returns its buffers."""
        self.graph.replay()
        return self.buffers


class HostPipeline:
    """One attention layer on inputs in (pinned) host memory, with the transfers overlapped
    with the kernels.

    The (b, h) slices run in ``chunks`` groups of consecutive slices.  A copy stream sends
    every group's Q, K and V to the device in turn; the current stream runs pool, route and
    attention on group c as soon as its inputs have arrived, while group c + 1 is still in
    transit; a second copy stream brings group c's out and lse back while group c + 1
    computes.  Pooling, routing and attention of a slice depend on that slice alone, so
    the results equal one ``attention_layer`` call on the whole layer, bit for bit.

    ``run`` is asynchronous on the current stream: the host inputs must stay unchanged, and
    the host outputs are valid, once the current stream has passed the call (for instance
    after ``torch.cuda.current_stream().synchronize()``)."""

    def __init__(self, g: Geometry, p: float, k_floor: int, scale: Optional[float] = None,
                 chunks: int = 4, device=None):
        import torch
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.g = g
        self.p, self.k_floor = float(p), int(k_floor)
        self.scale = 1.0 / math.sqrt(g.d) if scale is None else float(scale)
        S = g.B * g.H
        n = max(1, min(int(chunks), S))
        edges = [round(i * S / n) for i in range(n + 1)]
        self.ranges = [(a, b) for a, b in zip(edges[:-1], edges[1:]) if b > a]
        tok = (g.B, g.H, g.N, g.d)
        self.q = torch.empty(tok, dtype=torch.bfloat16, device=dev)
        self.k = torch.empty(tok, dtype=torch.bfloat16, device=dev)
        self.v = torch.empty(tok, dtype=torch.bfloat16, device=dev)
        full = LayerBuffers.allocate(g, dev)
        self.buffers = full
        widest = max(b - a for a, b in self.ranges)
        gw = dataclasses.replace(g, B=1, H=widest)
        ws = torch.empty(fvattn_attn_workspace_size(gw), dtype=torch.uint8, device=dev)
        rws = torch.empty(fvattn_route_workspace_size(gw), dtype=torch.uint8, device=dev)
        prws = torch.empty(fvattn_pool_route_workspace_size(gw), dtype=torch.uint8, device=dev)
        self.workspace = ws
        self.pool_route_ws = prws

        def rows(t, a, b):
            # slices [a, b) of a [B][H][...] tensor as a [1][b - a][...] view
            flat = t.reshape((S,) + tuple(t.shape[2:]))
            return flat[a:b].reshape((1, b - a) + tuple(t.shape[2:]))

        self._rows = rows
        self.sub = []
        for a, b in self.ranges:
            gc = dataclasses.replace(g, B=1, H=b - a)
            bc = LayerBuffers(q_pool=rows(full.q_pool, a, b), k_pool=rows(full.k_pool, a, b),
                              mask=rows(full.mask, a, b), counts=rows(full.counts, a, b),
                              out=rows(full.out, a, b), lse=rows(full.lse, a, b), workspace=ws,
                              sm_busy_ns=full.sm_busy_ns, route_ws=rws, pool_route_ws=prws)
            self.sub.append((gc, bc, rows(self.q, a, b), rows(self.k, a, b), rows(self.v, a, b)))
        self.s_in = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.ev_in = [torch.cuda.Event() for _ in self.ranges]
        self.ev_done = [torch.cuda.Event() for _ in self.ranges]

    def run(self, q_h, k_h, v_h, out_h, lse_h) -> LayerBuffers:
        """q_h, k_h, v_h: bf16 [B][H][N][d] host tensors (pinned for overlap); out_h: bf16
        [B][H][N][d] and lse_h: fp32 [B][H][N] host tensors that receive the results.
        Returns the device buffers (mask, counts, pooled rows, out, lse)."""
        import torch
        g = self.g
        tok = (g.B, g.H, g.N, g.d)
        for t, name, dt, shape in ((q_h, "q", torch.bfloat16, tok), (k_h, "k", torch.bfloat16, tok),
                                   (v_h, "v", torch.bfloat16, tok), (out_h, "out", torch.bfloat16, tok),
                                   (lse_h, "lse", torch.float32, tok[:3])):
            if t.is_cuda or t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous host tensor of {dt} and shape {shape}")
        cur = torch.cuda.current_stream(self.q.device)
        # the previous run's kernels read q, k, v and wrote out, lse: wait for them
        self.s_in.wait_stream(cur)
        self.s_out.wait_stream(cur)
        with torch.cuda.stream(self.s_in):
            for (a, b), (gc, bc, qd, kd, vd), ev in zip(self.ranges, self.sub, self.ev_in):
                qd.copy_(self._rows(q_h, a, b), non_blocking=True)
                kd.copy_(self._rows(k_h, a, b), non_blocking=True)
                vd.copy_(self._rows(v_h, a, b), non_blocking=True)
                ev.record(self.s_in)
        for (a, b), (gc, bc, qd, kd, vd), e_in, e_done in zip(self.ranges, self.sub, self.ev_in, self.ev_done):
            cur.wait_event(e_in)
            attention_layer(gc, qd, kd, vd, self.p, self.k_floor, self.scale, bc, cur)
            e_done.record(cur)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(e_done)
                self._rows(out_h, a, b).copy_(bc.out, non_blocking=True)
                self._rows(lse_h, a, b).copy_(bc.lse, non_blocking=True)
        cur.wait_stream(self.s_out)
        cur.wait_stream(self.s_in)
        return self.buffers

