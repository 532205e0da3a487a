"""Seeded synthetic workloads shaped like the Wan-family video DiT attention layers.

This module only draws random tensors and describes shapes.  It holds none of the
method's arithmetic (no pooling, no scores, no selection, no attention): both the
CUDA path and the fp64 oracle take their inputs from here, and nothing else is
shared between them.

Shapes follow the FVAttn explainer (arXiv 2607.16190, "Step-distilled Wan2.2 I2V"
workload) and the LVSA Long-Video Showcase README ("Results" table: Wan 2.1 1.3B,
horizons 1x..6x; "Configuration": Wan uses 21 reference latent frames).  A 480x832
video maps to a 30x52 latent per frame and 720x1280 to 45x80 (8x VAE, 2x2 patch).

Token order is T-major: token n of a (b, h) slice sits at latent position
(t, y, x) with n = (t * Hs + y) * Ws + x.  A 3D block is bt x bh x bw latent
positions; edge blocks are partial.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    T: int
    Hs: int
    Ws: int
    bt: int
    bh: int
    bw: int
    p: float
    k_floor: int
    seed: int
    kind: str                       # "plain" | "block" | "block_keyframe"
    qscale: Optional[Tuple[float, ...]] = None   # fixed per-head Q scales ("plain")
    keyframe_period: int = 20

    @property
    def N(self) -> int:
        return self.T * self.Hs * self.Ws

    @property
    def nblocks_3d(self) -> Tuple[int, int, int]:
        return (-(-self.T // self.bt), -(-self.Hs // self.bh), -(-self.Ws // self.bw))

    @property
    def nB(self) -> int:
        a, b, c = self.nblocks_3d
        return a * b * c

    @property
    def words(self) -> int:
        return -(-self.nB // 32)

    def geom(self) -> Dict[str, int]:
        return dict(B=self.B, H=self.H, T=self.T, Hs=self.Hs, Ws=self.Ws, d=self.d,
                    bt=self.bt, bh=self.bh, bw=self.bw)

    def with_pk(self, p: float, k_floor: int) -> "Workload":
        return dataclasses.replace(self, p=p, k_floor=k_floor,
                                   name=f"{self.name}_p{p:g}_k{k_floor}")


# The five workloads.  Seeds are 1234 + the workload's index; the sweep reuses the
# 480p inputs (same generator, same seed) and only varies p and k_floor.
TINY = Workload("tiny_h2_d64_4x8x8", B=1, H=2, d=64, T=4, Hs=8, Ws=8, bt=2, bh=4, bw=4,
                p=0.9, k_floor=2, seed=1235, kind="plain", qscale=(0.5, 3.0))
WAN21_480P = Workload("wan21_1.3b_480p_h12_21x30x52", B=1, H=12, d=128, T=21, Hs=30, Ws=52,
                      bt=1, bh=8, bw=16, p=0.9, k_floor=4, seed=1236, kind="block")
WAN22_720P = Workload("wan22_14b_720p_h40_21x45x80", B=1, H=40, d=128, T=21, Hs=45, Ws=80,
                      bt=1, bh=8, bw=16, p=0.9, k_floor=8, seed=1237, kind="block")
WAN21_6X = Workload("wan21_1.3b_6x_h12_121x30x52", B=1, H=12, d=128, T=121, Hs=30, Ws=52,
                    bt=1, bh=8, bw=16, p=0.85, k_floor=8, seed=1238, kind="block_keyframe")
SWEEP_P = (0.5, 0.7, 0.9, 0.95, 1.0)
SWEEP_K = (1, 4, 16)


def sweep() -> List[Workload]:
    return [WAN21_480P.with_pk(p, k) for p in SWEEP_P for k in SWEEP_K]


# Small ragged cases the oracle finishes in seconds: several KV blocks, partial
# blocks on the H and W edges (and on the T edge for the last one).
SMALL_RAGGED = Workload("small_ragged_h3_3x20x40", B=1, H=3, d=128, T=3, Hs=20, Ws=40,
                        bt=1, bh=8, bw=16, p=0.9, k_floor=4, seed=2001, kind="block")
SMALL_RAGGED_T = Workload("small_ragged_t_b2_h2_5x12x20", B=2, H=2, d=64, T=5, Hs=12, Ws=20,
                          bt=2, bh=4, bw=8, p=0.8, k_floor=3, seed=2002, kind="block")

ALL = {w.name: w for w in [TINY, WAN21_480P, WAN22_720P, WAN21_6X, SMALL_RAGGED, SMALL_RAGGED_T]}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32.
    Works in place on a float32 array that it owns (a copy is made otherwise)."""
    x = np.require(x, dtype=np.float32, requirements=["C", "W", "O"])
    u = x.view(np.uint32)
    lsb = (u >> 16) & 1
    lsb += 0x7FFF
    u += lsb
    u &= np.uint32(0xFFFF0000)
    return x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Raw uint16 bfloat16 bit patterns of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def token_block_ids(w: Workload) -> np.ndarray:
    """Block id of every token in T-major order (block ids are T-major over the block grid)."""
    nBt, nBy, nBx = w.nblocks_3d
    t = np.arange(w.T)[:, None, None] // w.bt
    y = np.arange(w.Hs)[None, :, None] // w.bh
    x = np.arange(w.Ws)[None, None, :] // w.bw
    return ((t * nBy + y) * nBx + x).reshape(-1)


def _orthonormal_rows(rng: np.random.Generator, r: int, d: int) -> np.ndarray:
    g = rng.standard_normal((d, r))
    qm, _ = np.linalg.qr(g)
    return qm.T.astype(np.float64)          # r x d, orthonormal rows


def generate(w: Workload) -> Dict[str, np.ndarray]:
    """Draw Q, K, V for one workload.

    Returns float32 arrays [B, H, N, d] whose values are exactly bf16, plus the
    per-head Q scales.  Recipe:

    * "plain": Q, K, V ~ N(0, 1); Q of head h is multiplied by qscale[h].
    * "block": per head an orthonormal 4 x d basis U_h; per 3D block c ~ N(0, I_4)
      and u = 1.5 * sqrt(d / 64) * c @ U_h.  Q = s_h * (z + u[block]),
      K = z' + u[block], V = z'' with z, z', z'' ~ N(0, 1) per token, and
      s_h = exp(Uniform(ln 0.5, ln 4)).
    * "block_keyframe": "block" plus, per head, a second orthonormal basis W_h and
      per spatial block position a component w = 1.5 * sqrt(d / 64) * g @ W_h,
      g ~ N(0, I_4).  w is added to K of the blocks of every keyframe (latent frames
      t = 0 mod keyframe_period) and to Q of every block at that spatial position.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed))
    B, H, N, d = w.B, w.H, w.N, w.d
    shape = (B, H, N, d)
    if w.kind == "plain":
        s = np.asarray(w.qscale, dtype=np.float64)
        assert s.shape == (H,)
        q = rng.standard_normal(shape, dtype=np.float32)
        k = rng.standard_normal(shape, dtype=np.float32)
        v = rng.standard_normal(shape, dtype=np.float32)
        q *= s.astype(np.float32)[None, :, None, None]
        return dict(q=bf16_round(q), k=bf16_round(k), v=bf16_round(v), qscale=s)

    s = np.exp(rng.uniform(math.log(0.5), math.log(4.0), size=H))
    amp = 1.5 * math.sqrt(d / 64.0)
    bid = token_block_ids(w)
    nB = w.nB
    comp_q = np.empty((B, H, nB, d), dtype=np.float32)
    comp_k = np.empty((B, H, nB, d), dtype=np.float32)
    U = [_orthonormal_rows(rng, 4, d) for _ in range(H)]
    c = rng.standard_normal((B, H, nB, 4))
    for b in range(B):
        for h in range(H):
            u = amp * (c[b, h] @ U[h])
            comp_q[b, h] = u
            comp_k[b, h] = u
    if w.kind == "block_keyframe":
        nBt, nBy, nBx = w.nblocks_3d
        Wb = [_orthonormal_rows(rng, 4, d) for _ in range(H)]
        g = rng.standard_normal((B, H, nBy * nBx, 4))
        blk = np.arange(nB)
        tb = blk // (nBy * nBx)
        pos = blk % (nBy * nBx)
        # a block is a keyframe block when its first latent frame is a keyframe
        key_blk = ((tb * w.bt) % w.keyframe_period) == 0
        for b in range(B):
            for h in range(H):
                wv = amp * (g[b, h] @ Wb[h])          # [positions, d]
                comp_q[b, h] += wv[pos]
                comp_k[b, h][key_blk] += wv[pos[key_blk]]
    elif w.kind != "block":
        raise ValueError(f"unknown workload kind {w.kind!r}")

    out = {}
    for name in ("q", "k", "v"):
        z = np.empty(shape, dtype=np.float32)
        for b in range(B):
            for h in range(H):
                zs = rng.standard_normal((N, d), dtype=np.float32)
                if name == "q":
                    zs += comp_q[b, h][bid]
                    zs *= np.float32(s[h])
                elif name == "k":
                    zs += comp_k[b, h][bid]
                z[b, h] = bf16_round(zs)
        out[name] = z
    out["qscale"] = s
    return out


def sample_qblocks(w: Workload, per_head: int, seed: int = 77) -> np.ndarray:
    """Seeded sample of query-block ids (shared by all heads) that always contains one
    block of every real-size class (interior, H edge, W edge, T edge and corners)."""
    nBt, nBy, nBx = w.nblocks_3d
    nB = w.nB
    if per_head >= nB:
        return np.arange(nB)
    rng = np.random.Generator(np.random.PCG64(seed))
    classes = {}
    for j in range(nB):
        tb, yb, xb = j // (nBy * nBx), (j // nBx) % nBy, j % nBx
        key = (tb == nBt - 1 and w.T % w.bt != 0, yb == nBy - 1 and w.Hs % w.bh != 0,
               xb == nBx - 1 and w.Ws % w.bw != 0)
        classes.setdefault(key, []).append(j)
    must = sorted({int(rng.choice(v)) for v in classes.values()})
    rest = np.setdiff1d(np.arange(nB), must)
    extra = rng.choice(rest, size=max(0, per_head - len(must)), replace=False)
    return np.sort(np.concatenate([np.asarray(must, dtype=np.int64), extra.astype(np.int64)]))
