"""HostPipeline (the layer on host-resident inputs, transfers overlapped with the
kernels in chunks of (b, h) slices) against one attention_layer call on the same inputs,
already on the device: every slice is computed on its own, so out, lse, mask and counts
must be equal bit for bit, for any chunking, and on a second run through the same
streams and buffers."""
import numpy as np
import pytest

from free_adaptive_block_b200 import workloads as W

from tests._parity import geometry, scale_of

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl,chunks", [(W.SMALL_RAGGED, 1), (W.SMALL_RAGGED, 2), (W.SMALL_RAGGED, 3),
                                       (W.SMALL_RAGGED_T, 3), (W.WAN21_480P, 4)],
                         ids=lambda v: v.name if hasattr(v, "name") else str(v))
def test_pipeline_equals_layer(wl, chunks):
    import torch
    import free_adaptive_block_b200 as fv
    x = W.generate(wl)
    g = geometry(wl)
    sc = scale_of(wl.d)
    host = {n: torch.from_numpy(W.bf16_bits(x[n])).view(torch.bfloat16).pin_memory() for n in ("q", "k", "v")}
    ref = fv.attention_layer(g, host["q"].cuda(), host["k"].cuda(), host["v"].cuda(), wl.p, wl.k_floor, sc)
    torch.cuda.synchronize()
    want = {n: getattr(ref, n).cpu() for n in ("out", "lse", "mask", "counts")}
    pipe = fv.HostPipeline(g, wl.p, wl.k_floor, sc, chunks=chunks)
    out_h = torch.empty(want["out"].shape, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty(want["lse"].shape, dtype=torch.float32).pin_memory()
    for _ in range(2):
        out_h.fill_(float("nan"))
        lse_h.fill_(float("nan"))
        b = pipe.run(host["q"], host["k"], host["v"], out_h, lse_h)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(out_h.view(torch.int16), want["out"].view(torch.int16))
        assert np.array_equal(lse_h.numpy().view(np.uint32), want["lse"].numpy().view(np.uint32))
        assert torch.equal(b.mask.cpu(), want["mask"])
        assert torch.equal(b.counts.cpu(), want["counts"])
        assert fv.fvattn_device_status(pipe.workspace) == 0
        assert fv.fvattn_device_status(pipe.pool_route_ws) == 0
