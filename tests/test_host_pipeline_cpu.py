"""HostPipeline's chunking on the CPU: its slice ranges, views and copies, with a stand-in
for the layer that computes a different result for every (b, h) slice.  The chunked run
must write exactly what the stand-in gives on the whole layer, for every chunk count;
CUDA streams and events are replaced by no-op stand-ins, device tensors by CPU ones."""
import contextlib

import pytest
import torch

import free_adaptive_block_b200 as fv


class FakeStream:
    def wait_stream(self, other):
        pass

    def wait_event(self, event):
        pass


class FakeEvent:
    def record(self, stream=None):
        pass


def stand_in_layer(g, q, k, v, p, k_floor, scale, b, stream=None):
    """A per-slice function of the slice's own inputs (and of nothing else)."""
    tok = (g.B, g.H, g.N, g.d)
    assert tuple(q.shape) == tok and tuple(b.out.shape) == tok and tuple(b.lse.shape) == tok[:3]
    assert tuple(b.mask.shape) == (g.B, g.H, g.nB, g.words)
    b.out.copy_((q.float() * 2 - k.float() + v.float() * 0.5).to(torch.bfloat16))
    b.lse.copy_(q.float().sum(-1) - k.float().amax(-1))
    b.mask.copy_(k.float()[..., : g.nB * 0 + 1, :1].to(torch.int32).expand(b.mask.shape))
    b.counts.copy_(v.float()[..., :1, 0].to(torch.int32).expand(b.counts.shape))
    return b


@pytest.fixture
def cpu_cuda(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "Stream", lambda *a, **k: FakeStream())
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: FakeEvent())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: FakeStream())
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(fv, "fvattn_attn_workspace_size", lambda g: 64)
    monkeypatch.setattr(fv, "fvattn_route_workspace_size", lambda g: 64)
    monkeypatch.setattr(fv, "fvattn_pool_route_workspace_size", lambda g: 64)
    monkeypatch.setattr(fv, "fvattn_num_sms", lambda: 4)
    monkeypatch.setattr(fv, "attention_layer", stand_in_layer)


@pytest.mark.parametrize("B,H,chunks", [(1, 3, 1), (1, 3, 2), (1, 3, 3), (2, 2, 3), (2, 3, 4), (1, 5, 9)])
def test_chunked_run_equals_whole_layer(cpu_cuda, B, H, chunks):
    g = fv.Geometry(B=B, H=H, T=2, Hs=8, Ws=12, d=16, bt=1, bh=4, bw=8)
    gen = torch.Generator().manual_seed(7)
    tok = (B, H, g.N, g.d)
    q, k, v = (torch.randn(tok, generator=gen).to(torch.bfloat16) for _ in range(3))
    want = fv.LayerBuffers.allocate(g, "cpu")
    stand_in_layer(g, q, k, v, 0.9, 2, 0.25, want)

    pipe = fv.HostPipeline(g, 0.9, 2, 0.25, chunks=chunks, device="cpu")
    assert pipe.ranges[0][0] == 0 and pipe.ranges[-1][1] == B * H
    assert all(a < b for a, b in pipe.ranges)
    assert all(r0[1] == r1[0] for r0, r1 in zip(pipe.ranges, pipe.ranges[1:]))
    out_h = torch.full(tok, float("nan"), dtype=torch.bfloat16)
    lse_h = torch.full(tok[:3], float("nan"))
    b = pipe.run(q, k, v, out_h, lse_h)
    assert torch.equal(out_h.view(torch.int16), want.out.view(torch.int16))
    assert torch.equal(lse_h, want.lse)
    assert torch.equal(b.mask, want.mask) and torch.equal(b.counts, want.counts)


def test_run_refuses_device_or_misshaped_host_tensors(cpu_cuda):
    g = fv.Geometry(B=1, H=2, T=1, Hs=4, Ws=8, d=16, bt=1, bh=4, bw=8)
    pipe = fv.HostPipeline(g, 0.9, 1, device="cpu")
    tok = (1, 2, g.N, g.d)
    good = torch.zeros(tok, dtype=torch.bfloat16)
    lse = torch.zeros(tok[:3])
    with pytest.raises(ValueError, match="q must be"):
        pipe.run(torch.zeros((1, 2, g.N, 8), dtype=torch.bfloat16), good, good, good, lse)
    with pytest.raises(ValueError, match="lse must be"):
        pipe.run(good, good, good, good, torch.zeros(tok[:3], dtype=torch.float64))
