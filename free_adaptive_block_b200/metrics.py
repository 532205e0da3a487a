"""Host-side bookkeeping for benchmarks: real block sizes, effective FLOPs and bytes.

Effective attention FLOPs count only real tokens: 4 * d * sum over (b, h, query block)
of q_real(qb) * sum over kept key blocks of k_real(kb)  (2 flops per multiply-add,
two products: Q K^T and P V).
"""
from __future__ import annotations

import numpy as np


def real_counts(T: int, Hs: int, Ws: int, bt: int, bh: int, bw: int) -> np.ndarray:
    """Real token count of every 3D block, T-major block order."""
    nBt, nBy, nBx = -(-T // bt), -(-Hs // bh), -(-Ws // bw)
    rt = np.minimum(bt, T - np.arange(nBt) * bt)
    ry = np.minimum(bh, Hs - np.arange(nBy) * bh)
    rx = np.minimum(bw, Ws - np.arange(nBx) * bw)
    return (rt[:, None, None] * ry[None, :, None] * rx[None, None, :]).reshape(-1).astype(np.int64)


def unpack_words(words: np.ndarray, nB: int) -> np.ndarray:
    w = words.astype(np.uint32).view(np.uint8)
    bits = np.unpackbits(w.reshape(words.shape[:-1] + (-1,)), axis=-1, bitorder="little")
    return bits[..., :nB].astype(bool)


def effective_flops(keep: np.ndarray, real: np.ndarray, d: int) -> float:
    """keep: bool [B, H, nB, nB]."""
    kreal = keep.astype(np.int64) @ real            # [B, H, nB] kept real keys per query block
    return float(4.0 * d * (kreal * real[None, None, :]).sum())


def dense_flops(B: int, H: int, N: int, d: int) -> float:
    return 4.0 * d * float(N) * float(N) * B * H


def pool_route_bytes(B: int, H: int, N: int, nB: int, d: int, words: int) -> float:
    """Algorithmic HBM bytes of pool + route: read Q and K (bf16), write and read the
    pooled Q and K (fp32), write the mask and the counts."""
    return float(2 * B * H * N * d * 2 + 2 * 2 * B * H * nB * d * 4 + B * H * nB * words * 4 + B * H * nB * 4)
