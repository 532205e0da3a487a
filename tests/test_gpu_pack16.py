"""GPU parity for 16-row narrow key blocks, packed eight to a K/V slot.

With 1 x 8 x 16 blocks and a latent width of 16 n + 2, the W-edge blocks are 2 tokens
wide, so their boxes have 16 rows and the attention kernel packs up to eight of them
into one 128-row K/V slot, one S and one P.V product.  This geometry has nine narrow key
blocks per head (three per frame): one full group of eight and a group of one.  Pool,
mask and attention are compared with the oracle as in the other small parity cases."""
import numpy as np
import pytest

import oracle as O
from free_adaptive_block_b200 import workloads as W
from tests import _parity as P

pytestmark = pytest.mark.gpu

PACK16 = [
    W.Workload("pack16_h2_3x20x50", B=1, H=2, d=128, T=3, Hs=20, Ws=50, bt=1, bh=8, bw=16,
               p=0.9, k_floor=4, seed=2003, kind="block"),
    W.Workload("pack16_b2_h2_d64_2x16x34", B=2, H=2, d=64, T=2, Hs=16, Ws=34, bt=1, bh=8, bw=16,
               p=0.8, k_floor=2, seed=2004, kind="block"),
]


def test_geometry_packs_sixteen_row_blocks():
    for wl in PACK16:
        rx_e = wl.Ws - (-(-wl.Ws // wl.bw) - 1) * wl.bw
        assert wl.bt * wl.bh * rx_e == 16


@pytest.mark.parametrize("wl", PACK16, ids=lambda w: w.name)
def test_pack16_parity(wl):
    x = W.generate(wl)
    res = P.gpu_layer(wl, x, wl.p, wl.k_floor)
    qp, kp = P.check_pool(wl, x, res)
    P.check_route(wl, qp, kp, res, wl.p, wl.k_floor)
    keep = O.unpack_mask(res["mask"], wl.nB)
    P.check_attn(wl, x, keep, res)


@pytest.mark.parametrize("wl", PACK16, ids=lambda w: w.name)
def test_pack16_dense_parity(wl):
    x = W.generate(wl)
    res = P.gpu_layer(wl, x, wl.p, wl.k_floor, dense=True)
    keep = np.ones((wl.B, wl.H, wl.nB, wl.nB), bool)
    P.check_attn(wl, x, keep, res)
