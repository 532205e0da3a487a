"""A layer captured in a CUDA graph (LayerGraph) replays to exactly the outputs of the
direct calls, including after its inputs are overwritten in place between replays."""
import dataclasses

import pytest

from free_adaptive_block_b200 import workloads as W
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl", [W.SMALL_RAGGED, W.WAN21_480P], ids=lambda w: w.name)
def test_graph_replay_matches_direct_calls(wl):
    import torch
    import free_adaptive_block_b200 as fv
    g = P.geometry(wl)
    sc = P.scale_of(wl.d)
    x = W.generate(wl)
    q, k, v = P.to_dev(x["q"]), P.to_dev(x["k"]), P.to_dev(x["v"])
    direct = fv.attention_layer(g, q, k, v, wl.p, wl.k_floor, sc)
    torch.cuda.synchronize()
    lg = fv.LayerGraph(g, q, k, v, wl.p, wl.k_floor, sc)
    for _ in range(2):
        b = lg.replay()
        torch.cuda.synchronize()
        assert fv.fvattn_device_status(b.workspace) == 0
        assert torch.equal(b.mask, direct.mask) and torch.equal(b.counts, direct.counts)
        assert torch.equal(b.out.view(torch.int16), direct.out.view(torch.int16))
        assert torch.equal(b.lse, direct.lse)

    # new inputs copied into the captured buffers: the replay follows them
    x2 = W.generate(dataclasses.replace(wl, seed=wl.seed + 1000))
    q.copy_(P.to_dev(x2["q"]))
    k.copy_(P.to_dev(x2["k"]))
    v.copy_(P.to_dev(x2["v"]))
    direct2 = fv.attention_layer(g, q, k, v, wl.p, wl.k_floor, sc)
    b = lg.replay()
    torch.cuda.synchronize()
    assert torch.equal(b.mask, direct2.mask)
    assert torch.equal(b.out.view(torch.int16), direct2.out.view(torch.int16))
    assert torch.equal(b.lse, direct2.lse)
