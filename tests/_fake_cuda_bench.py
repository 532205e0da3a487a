"""Runs bench.py's GPU arm on the CPU, for tests of its control flow and of its JSON
line: CUDA events, streams, graphs and devices are replaced by stand-ins, the library
calls by no-ops (the route keeps every block), and the NCCL process group by gloo.
Timings are therefore constant (4 ms per event pair); only the bench's bookkeeping is
under test.  Usage: python tests/_fake_cuda_bench.py <bench arguments>."""
import contextlib
import importlib.util
import itertools
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import free_adaptive_block_b200 as fv  # noqa: E402

_ctr = itertools.count()


class FakeEvent:
    def __init__(self, enable_timing=False, **kw):
        self.t = None

    def record(self, stream=None):
        self.t = next(_ctr)

    def elapsed_time(self, other):
        return 4.0


class FakeStream:
    cuda_stream = 0

    def wait_stream(self, other):
        pass

    def wait_event(self, event):
        pass


class FakeGraph:
    def replay(self):
        pass


_real_device = torch.device


def fake_device(*a, **k):
    if a and a[0] == "cuda":
        return _real_device("cpu")
    return _real_device(*a, **k)


torch.cuda.set_device = lambda d: None
torch.cuda.current_device = lambda: 0
torch.cuda.synchronize = lambda d=None: None
torch.cuda.Event = FakeEvent
torch.cuda.current_stream = lambda d=None: FakeStream()
torch.cuda.Stream = lambda d=None: FakeStream()
torch.cuda.stream = lambda s: contextlib.nullcontext()
torch.cuda.CUDAGraph = FakeGraph
torch.cuda.graph = lambda g: contextlib.nullcontext()
torch.device = fake_device
torch.Tensor.pin_memory = lambda self: self
_real_init = dist.init_process_group
dist.init_process_group = lambda backend, **kw: _real_init("gloo", **kw)


def keep_all(g, qp, kp, p, kf, sc, mask, counts, *rest, **kw):
    mask.fill_(-1)


fv.fvattn_attn_workspace_size = lambda g: 1024
fv.fvattn_route_workspace_size = lambda g: 1024
fv.fvattn_num_sms = lambda: 148
fv.fvattn_block_pool = lambda *a, **k: None
fv.fvattn_route = keep_all
fv.fvattn_route_ws = keep_all
fv.fvattn_block_sparse_attn = lambda *a, **k: None
fv.fvattn_dense_attn = lambda *a, **k: None
fv.fvattn_device_status = lambda *a, **k: 0
fv.fvattn_pool_route_workspace_size = lambda g: 1024
fv.fvattn_pool_route = lambda g, q, k, p, kf, sc, qp, kp, mask, counts, ws, stream=None: mask.fill_(-1)
fv.fvattn_route_ex = lambda g, qp, kp, opts, mask, counts, ws, stream=None: mask.fill_(-1)
fv.fvattn_slack_augment = lambda *a, **k: None


class FakeLayerGraph:
    def __init__(self, g, q, k, v, p, kf, scale, buf):
        keep_all(g, None, None, p, kf, scale, buf.mask, buf.counts)

    def replay(self):
        pass


fv.LayerGraph = FakeLayerGraph

spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(spec)
spec.loader.exec_module(bench)
sys.argv = ["bench.py"] + sys.argv[1:]
bench.main()
