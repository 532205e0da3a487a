"""The seeded generator: shapes, determinism, bf16-exact values, block structure."""
import numpy as np

from free_adaptive_block_b200 import workloads as W


def test_shapes_and_geometry_of_the_named_workloads():
    assert (W.WAN21_480P.N, W.WAN21_480P.nB, W.WAN21_480P.words) == (32760, 336, 11)
    assert (W.WAN22_720P.N, W.WAN22_720P.nB, W.WAN22_720P.words) == (75600, 630, 20)
    assert (W.WAN21_6X.N, W.WAN21_6X.nB, W.WAN21_6X.words) == (188760, 1936, 61)
    assert (W.TINY.N, W.TINY.nB, W.TINY.words) == (256, 8, 1)
    assert len(W.sweep()) == 15


def test_deterministic_and_bf16_exact():
    a = W.generate(W.SMALL_RAGGED)
    b = W.generate(W.SMALL_RAGGED)
    for name in "qkv":
        assert a[name].shape == (1, 3, 3 * 20 * 40, 128)
        assert np.array_equal(a[name], b[name])
        bits = a[name].view(np.uint32)
        assert not (bits & 0xFFFF).any(), "values must be exactly bf16"
    assert np.all((a["qscale"] >= 0.5) & (a["qscale"] <= 4.0))


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -9, -3.0], np.float32)
    want = np.array([1.0, 1.0, 1 + 2 ** -6, 1.0, -3.0], np.float32)
    assert np.array_equal(W.bf16_round(x.copy()), want)
    assert W.bf16_bits(np.array([1.0], np.float32))[0] == 0x3F80


def test_block_component_gives_spatial_locality():
    # tokens of one block share a component, so their K rows correlate more than
    # tokens of different blocks
    w = W.SMALL_RAGGED
    x = W.generate(w)
    bid = W.token_block_ids(w)
    k = x["k"][0, 0].astype(np.float64)
    means = np.stack([k[bid == j].mean(0) for j in range(w.nB)])
    assert np.linalg.norm(means, axis=1).mean() > 2.0   # block means stand out of the noise


def test_sample_contains_every_size_class():
    s = W.sample_qblocks(W.WAN21_480P, 64)
    assert len(s) == 64 and len(set(s.tolist())) == 64
    nBx = 4
    nBy = 4
    assert any(j % nBx == nBx - 1 and (j // nBx) % nBy == nBy - 1 for j in s)   # corner
    assert any(j % nBx == nBx - 1 and (j // nBx) % nBy != nBy - 1 for j in s)   # W edge
    assert any(j % nBx != nBx - 1 and (j // nBx) % nBy == nBy - 1 for j in s)   # H edge
