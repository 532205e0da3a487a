"""The bench's accounting (free_adaptive_block_b200.metrics), pinned on the CPU.

The throughput the bench reports is effective FLOPs over measured time, so the FLOP
count is checked against brute force: every (query token, key token) pair whose key
block is kept for the query's block contributes 4*d FLOPs (a multiply-add in Q K^T and
one in P V).  Block real sizes come from per-token block assignment, mask bits from
an explicit bit loop."""
import itertools

import numpy as np
import pytest

from free_adaptive_block_b200 import metrics as MX

GEOMS = [
    # T, Hs, Ws, bt, bh, bw
    (4, 8, 8, 2, 4, 4),        # divides evenly
    (3, 20, 40, 1, 8, 16),     # ragged in H and W
    (5, 12, 20, 2, 4, 8),      # ragged in T, H and W
    (21, 30, 52, 1, 8, 16),    # the Wan2.1-480p latent
]


def token_blocks(T, Hs, Ws, bt, bh, bw):
    """Block id of every token, T-major tokens and blocks, by explicit loops."""
    nBy, nBx = -(-Hs // bh), -(-Ws // bw)
    ids = []
    for t, y, x in itertools.product(range(T), range(Hs), range(Ws)):
        ids.append(((t // bt) * nBy + y // bh) * nBx + x // bw)
    return np.array(ids)


@pytest.mark.parametrize("geom", GEOMS)
def test_real_counts_match_per_token_assignment(geom):
    T, Hs, Ws, bt, bh, bw = geom
    nB = -(-T // bt) * -(-Hs // bh) * -(-Ws // bw)
    brute = np.bincount(token_blocks(*geom), minlength=nB)
    got = MX.real_counts(*geom)
    assert got.shape == (nB,)
    assert np.array_equal(got, brute)
    assert got.sum() == T * Hs * Ws


def test_unpack_words_bit_order():
    rng = np.random.default_rng(3)
    for nB in (1, 31, 32, 33, 64, 336):
        words = -(-nB // 32)
        w = rng.integers(0, 2**32, size=(2, 3, 5, words), dtype=np.uint64).astype(np.uint32)
        got = MX.unpack_words(w.view(np.int32), nB)
        assert got.shape == (2, 3, 5, nB)
        for idx in itertools.product(range(2), range(3), range(5)):
            for j in range(nB):
                assert got[idx + (j,)] == bool((int(w[idx + (j // 32,)]) >> (j % 32)) & 1)


@pytest.mark.parametrize("geom", GEOMS[:3])
def test_effective_flops_against_token_pairs(geom):
    T, Hs, Ws, bt, bh, bw = geom
    d, B, H = 64, 1, 2
    blk = token_blocks(*geom)
    nB = int(blk.max()) + 1
    rng = np.random.default_rng(11)
    keep = rng.random((B, H, nB, nB)) < 0.4
    pairs = 0
    for b, h in itertools.product(range(B), range(H)):
        # keep[b, h, block of query token, block of key token], summed over all token pairs
        pairs += int(keep[b, h][blk[:, None], blk[None, :]].sum())
    assert MX.effective_flops(keep, MX.real_counts(*geom), d) == 4.0 * d * pairs


@pytest.mark.parametrize("geom", GEOMS)
def test_all_kept_equals_dense(geom):
    T, Hs, Ws, bt, bh, bw = geom
    real = MX.real_counts(*geom)
    nB = real.size
    B, H, d = 1, 3, 128
    keep = np.ones((B, H, nB, nB), dtype=bool)
    N = T * Hs * Ws
    assert MX.effective_flops(keep, real, d) == MX.dense_flops(B, H, N, d) == 4.0 * d * N * N * B * H


def test_pool_route_bytes_480p():
    B, H, N, nB, d, words = 1, 12, 32760, 336, 128, 11
    q_k_read = 2 * B * H * N * d * 2                 # Q and K, bf16
    pooled = 2 * (B * H * nB * d * 4) * 2            # pooled Q and K, fp32, written then read
    mask_counts = B * H * nB * (words + 1) * 4
    assert MX.pool_route_bytes(B, H, N, nB, d, words) == q_k_read + pooled + mask_counts
    assert 209e6 < MX.pool_route_bytes(B, H, N, nB, d, words) < 211e6
