"""Plain fp64 CPU oracle for adaptive block-sparse attention (pool -> route -> attention).

TEST INFRASTRUCTURE ONLY.  This module defines what the CUDA path must compute and is
used by the tests, by ``__graft_entry__.smoke()`` and by the CPU-baseline legs of
``bench.py``.  The library itself never imports it, and it imports nothing from the
library: it shares no code, table or constant with the CUDA kernels.

It follows the FVAttn explainer (papers.ananclaw.com, arXiv 2607.16190,
"Adaptive Sparse Attention with Runtime Load Balancing for Video Generation"),
section 核心方法 §1 稀疏路由前端 (sparse-routing frontend):

* Video-aware block organisation: spatio-temporal tokens are regrouped into 3D
  blocks and routing decides per block  -> :func:`block_geometry`, :func:`pool`.
* Top-p routing: keep the minimal set whose cumulative similarity mass reaches p
  -> :func:`route`.
* Top-k safety floor: every head keeps at least k KV blocks however aggressive p is
  -> :func:`route`.
* Attention then runs only over the selected KV blocks (the kernel that replaces
  FlashAttention, 核心方法 §2, ``attn_kernel.run()``) -> :func:`masked_attn`; the
  all-blocks case is plain softmax attention -> :func:`dense_attn`.

The pages give no formula for the routing score, no block size and no p or k.  The
readings used here (each also listed in the design notes):

* routing score of key block j for query block i: softmax over all key blocks of
  (mean-pooled q_i) . (mean-pooled k_j) / sqrt(d); blocks are not size-weighted;
* a block's mean is over its real tokens only (edge blocks are partial);
* order by score descending, ties by lower block index; "reaches p" means >= p;
  p >= 1 keeps every block; the floor counts blocks and takes the first k of the
  same order; the query's own block is always added after the prefix rule;
* attention over the real tokens of the kept blocks, lse = natural log of the
  softmax denominator (the FlashAttention convention).

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed forms,
brute force on tiny inputs, hand-derived golden cases and a library routine.
"""
from __future__ import annotations

import dataclasses
import itertools
from fractions import Fraction
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np


# ----------------------------------------------------------------------------------
# 3D blocks (video-aware block organisation)
# ----------------------------------------------------------------------------------
@dataclasses.dataclass
class BlockGeometry:
    T: int
    Hs: int
    Ws: int
    bt: int
    bh: int
    bw: int
    nBt: int
    nBy: int
    nBx: int
    nB: int
    block_of_token: np.ndarray        # [N] block id of each token (T-major tokens)
    tokens_of_block: List[np.ndarray]  # ascending token indices of each block
    real_count: np.ndarray            # [nB] number of real tokens per block


def block_geometry(T: int, Hs: int, Ws: int, bt: int, bh: int, bw: int) -> BlockGeometry:
    """Map every latent position (t, y, x) -- token n = (t*Hs + y)*Ws + x -- to the 3D
    block (t//bt, y//bh, x//bw), numbered T-major: id = (tb*nBy + yb)*nBx + xb.
    Blocks on the far T/H/W edges are partial: only positions inside the latent exist."""
    nBt, nBy, nBx = -(-T // bt), -(-Hs // bh), -(-Ws // bw)
    nB = nBt * nBy * nBx
    tt, yy, xx = np.meshgrid(np.arange(T), np.arange(Hs), np.arange(Ws), indexing="ij")
    blk = ((tt // bt) * nBy + (yy // bh)) * nBx + (xx // bw)
    blk = blk.reshape(-1)
    by_block = np.argsort(blk, kind="stable")             # token ids grouped by block
    bounds = np.cumsum(np.bincount(blk, minlength=nB))[:-1]
    tokens = [t.astype(np.int64) for t in np.split(by_block, bounds)]
    real = np.asarray([len(t) for t in tokens], dtype=np.int64)
    return BlockGeometry(T, Hs, Ws, bt, bh, bw, nBt, nBy, nBx, nB, blk, tokens, real)


# ----------------------------------------------------------------------------------
# Pooling
# ----------------------------------------------------------------------------------
def pool(X: np.ndarray, g: BlockGeometry) -> np.ndarray:
    """Mean of X over the real tokens of each 3D block.  X: [B, H, N, d] -> [B, H, nB, d]."""
    B, H, N, d = X.shape
    out = np.empty((B, H, g.nB, d), dtype=np.float64)
    for j, toks in enumerate(g.tokens_of_block):
        out[:, :, j, :] = X[:, :, toks, :].astype(np.float64).sum(axis=2) / len(toks)
    return out


# ----------------------------------------------------------------------------------
# Routing: Top-p with a Top-k floor, own block always kept
# ----------------------------------------------------------------------------------
@dataclasses.dataclass
class RouteResult:
    keep: np.ndarray      # bool [B, H, nB(query), nB(key)]
    counts: np.ndarray    # int  [B, H, nB]
    scores: np.ndarray    # fp64 [B, H, nB, nB] routing scores (rows sum to 1)
    order: np.ndarray     # int  [B, H, nB, nB] key blocks sorted by (score desc, index asc)
    csum: np.ndarray      # fp64 [B, H, nB, nB] cumulative mass along `order`
    m_p: np.ndarray       # int  [B, H, nB] Top-p prefix length
    m_keep: np.ndarray    # int  [B, H, nB] prefix length after the Top-k floor
    mass: Optional[np.ndarray] = None   # fp64 [B, H, nB, nB] mass of each block (= scores
                                        # unless the Top-p runs over tokens)


def routing_scores(Qp: np.ndarray, Kp: np.ndarray, scale: float) -> np.ndarray:
    """s[i, j] = softmax over key blocks j of (Qp[i] . Kp[j]) * scale, in fp64."""
    logits = np.einsum("bhid,bhjd->bhij", Qp.astype(np.float64), Kp.astype(np.float64)) * scale
    e = np.exp(logits - logits.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def token_scores(Qp: np.ndarray, Kp: np.ndarray, scale: float, real_count: np.ndarray) -> np.ndarray:
    """Top-p over tokens, decided per block: every real token of key block j takes the
    block's pooled logit l_j = (Qp[i] . Kp[j]) * scale, and the softmax runs over all real
    tokens.  Returns the score of one token of block j, exp(l_j) / sum_k n_k exp(l_k)
    (n_k = real token count of block k); the block's mass is n_j times it."""
    logits = np.einsum("bhid,bhjd->bhij", Qp.astype(np.float64), Kp.astype(np.float64)) * scale
    e = np.exp(logits - logits.max(axis=-1, keepdims=True))
    return e / (e * np.asarray(real_count, np.float64)).sum(axis=-1, keepdims=True)


def route(Qp: np.ndarray, Kp: np.ndarray, p: float, k_floor: int, scale: float,
          real_count: Optional[np.ndarray] = None) -> RouteResult:
    """Per (batch, head, query block): sort key blocks by score (desc, ties by lower
    index); m_p = the shortest prefix whose cumulative mass is >= p (every block when
    p >= 1, capped at nB); m = max(m_p, min(k_floor, nB)); keep that prefix plus the
    query's own block.

    With `real_count` (the real token count of every block) the Top-p runs over tokens
    (:func:`token_scores`): the blocks keep the order of their routing scores (the order
    of their pooled logits, which every token of the block takes), and `mass`, what the
    prefix accumulates, is a block's share of the token mass, n_j times its token score."""
    s = routing_scores(Qp, Kp, scale)
    if real_count is None:
        mass = s
    else:
        mass = token_scores(Qp, Kp, scale, real_count) * np.asarray(real_count, np.float64)
    B, H, nB, _ = s.shape
    order = np.argsort(-s, axis=-1, kind="stable")
    csum = np.cumsum(np.take_along_axis(mass, order, axis=-1), axis=-1)
    if p >= 1.0:
        m_p = np.full((B, H, nB), nB, dtype=np.int64)
    else:
        m_p = np.minimum(1 + (csum < p).sum(axis=-1), nB)
    m_keep = np.maximum(m_p, min(int(k_floor), nB))
    rank = np.empty_like(order)
    np.put_along_axis(rank, order, np.broadcast_to(np.arange(nB), order.shape), axis=-1)
    keep = rank < m_keep[..., None]
    own = np.arange(nB)
    keep[..., own, own] = True
    return RouteResult(keep=keep, counts=keep.sum(axis=-1), scores=s, order=order,
                       csum=csum, m_p=m_p, m_keep=m_keep, mass=mass)


def pack_mask(keep: np.ndarray) -> np.ndarray:
    """Pack a boolean [..., nB] keep matrix as uint32 words: bit j%32 of word j//32."""
    nB = keep.shape[-1]
    words = -(-nB // 32)
    padded = np.zeros(keep.shape[:-1] + (words * 32,), dtype=np.uint64)
    padded[..., :nB] = keep
    padded = padded.reshape(keep.shape[:-1] + (words, 32))
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (padded * weights).sum(axis=-1).astype(np.uint32)


def unpack_mask(words: np.ndarray, nB: int) -> np.ndarray:
    """Inverse of :func:`pack_mask`."""
    w = words.astype(np.uint64)[..., None]
    bits = (w >> np.arange(32, dtype=np.uint64)) & np.uint64(1)
    return bits.reshape(words.shape[:-1] + (words.shape[-1] * 32,))[..., :nB].astype(bool)


def keyframe_blocks(g: BlockGeometry, stride: int, phase: int) -> np.ndarray:
    """Key blocks that hold a keyframe (LVSA README, rotating keyframes): latent frame t is
    a keyframe when (t - phase) mod stride == 0, and a block is a keyframe block when one
    of its real frames is.  bool [nB]; all False when stride <= 0."""
    kf = np.zeros(g.nB, dtype=bool)
    if stride <= 0:
        return kf
    frames = np.arange(g.T)
    key_t = ((frames - phase) % stride) == 0
    for j in range(g.nB):
        tb = j // (g.nBy * g.nBx)
        kf[j] = key_t[tb * g.bt:min(g.T, tb * g.bt + g.bt)].any()
    return kf


def add_keyframes(keep: np.ndarray, kf: np.ndarray) -> np.ndarray:
    """Every query block also keeps every keyframe block (added after the prefix rule, like
    the own block; they do not count toward Top-p or the floor)."""
    return keep | kf[None, None, None, :]


def repair_mask(keep: np.ndarray, g: BlockGeometry) -> np.ndarray:
    """Runtime mask repair on the materialized mask, without scores (FVAttn explainer,
    核心方法 §1, 运行时修补): in each row, a dropped key block whose two neighbours along
    the time, height or width axis of the 3D block grid both exist and are both kept is a
    one-block hole, and is restored.  One pass: every decision reads the mask as given."""
    nB = g.nB
    out = keep.copy()
    tb, rem = np.divmod(np.arange(nB), g.nBy * g.nBx)
    yb, xb = np.divmod(rem, g.nBx)
    for coord, ext, step in ((tb, g.nBt, g.nBy * g.nBx), (yb, g.nBy, g.nBx), (xb, g.nBx, 1)):
        inner = np.nonzero((coord > 0) & (coord < ext - 1))[0]
        hole = keep[..., inner - step] & keep[..., inner + step]
        out[..., inner] |= hole
    return out


def tile_costs(keep: np.ndarray, real_count: np.ndarray) -> np.ndarray:
    """Attention work of every (b, h, query block) tile: its real query tokens times the
    real key tokens of its kept blocks.  int [B, H, nB]."""
    rc = np.asarray(real_count, np.int64)
    return rc[None, None, :] * (keep.astype(np.int64) @ rc)


def slack_augment(keep: np.ndarray, scores: np.ndarray, real_count: np.ndarray, n_sm: int,
                  tau: float) -> np.ndarray:
    """Slack-aware sparse augmentation on one GPU (FVAttn explainer, 核心方法 §3: the slack
    that idle workers leave before the critical path ends is filled with high-value blocks,
    filtered by a score threshold).

    The tiles run longest first (cost descending, ties by tile index).  The last n_sm
    tiles of that order form the final wave, where workers fall idle: its largest tile
    sets the end, cost c*.  Every tile of the wave takes its dropped blocks of routing
    score >= tau, in score order (descending, ties by lower index), each while the tile's
    cost stays <= c*, stopping at the first that does not fit."""
    B, H, nB, _ = keep.shape
    rc = np.asarray(real_count, np.int64)
    cost = tile_costs(keep, rc).reshape(-1)
    T = cost.size
    order = np.lexsort((np.arange(T), -cost))          # cost desc, then index asc
    wave = order[max(0, T - int(n_sm)):]
    out = keep.copy()
    if wave.size == 0:
        return out
    cap = cost[wave].max()
    flat_keep = out.reshape(T, nB)
    flat_s = scores.reshape(T, nB)
    for t in wave:
        qb = t % nB
        c = cost[t]
        cand = [j for j in np.lexsort((np.arange(nB), -flat_s[t]))
                if not flat_keep[t, j] and flat_s[t, j] >= tau]
        for j in cand:
            add = rc[qb] * rc[j]
            if c + add > cap:
                break
            flat_keep[t, j] = True
            c += add
    return out


def keep_for_cut(r: RouteResult, m: np.ndarray) -> np.ndarray:
    """The keep matrix for prefix lengths m [B,H,nB] (instead of r.m_keep): the first m
    key blocks of each row's order, plus the query's own block."""
    nB = r.order.shape[-1]
    rank = np.empty_like(r.order)
    np.put_along_axis(rank, r.order, np.broadcast_to(np.arange(nB), r.order.shape), axis=-1)
    keep = rank < m[..., None]
    own = np.arange(nB)
    keep[..., own, own] = True
    return keep


def band_for_cut(r: RouteResult, m: np.ndarray, band: float = 1e-5) -> np.ndarray:
    """Key blocks whose kept/dropped state rounding may flip when the prefix has length m.

    The cutoff is the score c of the m-th block in the order.  Blocks whose score lies
    within `band` of c can change places in an fp32 order, but that changes the kept set
    only when they sit on both sides of the cut; so a row's near-cutoff blocks are
    excluded when some of them are inside the prefix and some outside, and none are
    excluded otherwise.  The own block is kept either way and is never excluded."""
    nB = r.order.shape[-1]
    s_sorted = np.take_along_axis(r.scores, r.order, axis=-1)
    cutoff = np.take_along_axis(s_sorted, (np.maximum(m, 1) - 1)[..., None], axis=-1)
    near = np.abs(r.scores - cutoff) < band
    rank = np.empty_like(r.order)
    np.put_along_axis(rank, r.order, np.broadcast_to(np.arange(nB), r.order.shape), axis=-1)
    inside = rank < m[..., None]
    straddles = (near & inside).any(-1) & (near & ~inside).any(-1)
    excluded = near & straddles[..., None]
    own = np.arange(nB)
    excluded[..., own, own] = False
    return excluded


def candidate_cuts(r: RouteResult, p: float, k_floor: int, band: float = 1e-5) -> np.ndarray:
    """Prefix lengths an fp32 implementation may legitimately reach, per row: int
    [B,H,nB,3] holding m_keep and, where a cumulative sum next to the Top-p cut lies
    within `band` of p, the prefix length after the floor with the cut moved one block
    later (the sum at m_p may round below p) or one block earlier (the sum at m_p - 1
    may round up to p); m_keep again where no such sum is near p."""
    B, H, nB, _ = r.scores.shape
    out = np.repeat(r.m_keep[..., None], 3, axis=-1)
    if p < 1.0:
        floor = min(int(k_floor), nB)
        cs, m_p = r.csum, r.m_p
        near_at = np.abs(np.take_along_axis(cs, (m_p - 1)[..., None], -1)[..., 0] - p) < band
        prev = np.take_along_axis(cs, np.maximum(m_p - 2, 0)[..., None], -1)[..., 0]
        near_prev = (m_p >= 2) & (np.abs(prev - p) < band)
        alt_up = np.maximum(np.minimum(m_p + 1, nB), floor)
        alt_dn = np.maximum(np.maximum(m_p - 1, 1), floor)
        out[..., 1] = np.where(near_at, alt_up, r.m_keep)
        out[..., 2] = np.where(near_prev, alt_dn, r.m_keep)
    return out


def comparison_band(r: RouteResult, p: float, k_floor: int, band: float = 1e-5
                    ) -> Tuple[np.ndarray, np.ndarray]:
    """Where a GPU mask computed in fp32 may legitimately differ from this fp64 one.

    Returns (excluded [B,H,nB,nB] bool, ambiguous [B,H,nB] bool):
    * excluded: key blocks whose score lies within `band` of the cutoff score (the
      score of the last block of the kept prefix, after the floor), in rows where such
      blocks lie on both sides of the cut (:func:`band_for_cut`); the own block is
      never excluded;
    * ambiguous: rows where a cumulative sum next to the Top-p cut lies within `band`
      of p, so that rounding can move the cut by one block and change the prefix
      length after the floor (:func:`candidate_cuts`).  Such rows are compared with
      the keep set of each candidate cut."""
    excluded = band_for_cut(r, r.m_keep, band)
    amb = (candidate_cuts(r, p, k_floor, band) != r.m_keep[..., None]).any(-1)
    return excluded, amb


def check_route_invariants(keep_row: np.ndarray, s_row: np.ndarray, own: int, p: float,
                           k_floor: int, tol: float = 0.0,
                           mass_row: Optional[np.ndarray] = None) -> Optional[str]:
    """Check that a keep vector is a valid Top-p/Top-k/own-block selection for one row
    of scores, up to `tol` on scores and masses.  Returns None when valid, else why.

    Valid means: the own block is kept, and for P = the kept set (or the kept set
    without the own block, when the own block was added after the prefix):
    every block of P scores >= every block outside P (minus tol); |P| >= min(k, nB);
    mass(P) >= p - tol unless P is everything; and P is minimal: when |P| exceeds
    the floor, dropping its lowest-scoring block leaves mass < p + tol.  Masses are
    `mass_row` when given (Top-p over tokens), else the scores."""
    nB = s_row.shape[0]
    m_row = s_row if mass_row is None else mass_row
    if not keep_row[own]:
        return "own block not kept"
    floor = min(int(k_floor), nB)
    cands = [keep_row.copy()]
    alt = keep_row.copy()
    alt[own] = False
    if alt.any():
        cands.append(alt)
    reasons = []
    for P in cands:
        inside, outside = s_row[P], s_row[~P]
        n = int(P.sum())
        if outside.size and inside.min() < outside.max() - tol:
            reasons.append("not a top set"); continue
        if n < floor:
            reasons.append("below the Top-k floor"); continue
        mass = m_row[P].sum()
        if p >= 1.0:
            if n != nB:
                reasons.append("p >= 1 must keep every block"); continue
            return None
        if n < nB and mass < p - tol:
            reasons.append("mass below p"); continue
        last = np.nonzero(P)[0][np.argmin(s_row[P])]
        if n > floor and n > 1 and mass - m_row[last] >= p + tol:
            reasons.append("not minimal"); continue
        return None
    return "; ".join(reasons)


def brute_force_route_row(s_row: np.ndarray, own: int, p: float, k_floor: int) -> np.ndarray:
    """Exhaustive reference for one row (tiny nB only): the smallest cardinality c* of
    any subset with mass >= p (nB if none, or if p >= 1); then among all subsets of size
    max(c*, min(k, nB)) the one of largest mass, ties to the lexicographically smallest
    index tuple; plus the own block.  Subset masses are exact rational sums of the fp64
    scores, so subsets of exactly equal mass tie and fall to the index rule, whatever
    order a floating-point sum would take them in."""
    nB = s_row.shape[0]
    assert nB <= 12, "brute force is for tiny rows only"
    exact = [Fraction(float(v)) for v in s_row]
    mass_of = lambda S: sum((exact[j] for j in S), Fraction(0))   # noqa: E731
    if p >= 1.0:
        c_star = nB
    else:
        target = Fraction(float(p))
        c_star = nB
        for c in range(1, nB + 1):
            if any(mass_of(S) >= target for S in itertools.combinations(range(nB), c)):
                c_star = c
                break
    m = max(c_star, min(int(k_floor), nB))
    best, best_mass = None, Fraction(-1)
    for S in itertools.combinations(range(nB), m):      # lexicographic order
        mass = mass_of(S)
        if mass > best_mass:
            best, best_mass = S, mass
    keep = np.zeros(nB, dtype=bool)
    keep[list(best)] = True
    keep[own] = True
    return keep


def brute_force_token_route_row(tok_score_row: np.ndarray, real_count: np.ndarray, own: int,
                                p: float, k_floor: int) -> np.ndarray:
    """Token-level reference for one row of the Top-p over tokens (tiny inputs only).  The
    row is expanded into real tokens, n_j tokens of score tok_score_row[j] for block j,
    ordered by score (ties by block index); the shortest token prefix whose exact
    (rational) mass reaches p selects tokens, and a block is kept when it holds a selected
    token.  The floor then lengthens the kept blocks, in the same block order, to
    min(k, nB); the own block is added."""
    nB = tok_score_row.shape[0]
    blocks = sorted(range(nB), key=lambda j: (-float(tok_score_row[j]), j))
    tokens = [j for j in blocks for _ in range(int(real_count[j]))]
    if p >= 1.0:
        chosen = set(range(nB))
    else:
        target, acc, chosen = Fraction(float(p)), Fraction(0), set()
        for j in tokens:
            chosen.add(j)
            acc += Fraction(float(tok_score_row[j]))
            if acc >= target:
                break
        else:
            chosen = set(range(nB))
    floor = min(int(k_floor), nB)
    for j in blocks:
        if len(chosen) >= floor:
            break
        chosen.add(j)
    keep = np.zeros(nB, dtype=bool)
    keep[sorted(chosen)] = True
    keep[own] = True
    return keep


# ----------------------------------------------------------------------------------
# Attention over the kept blocks, and plain dense attention
# ----------------------------------------------------------------------------------
def masked_attn(Q: np.ndarray, K: np.ndarray, V: np.ndarray, keep: np.ndarray,
                g: BlockGeometry, scale: float, qblocks: Optional[Sequence[int]] = None
                ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """For each real query token i of each listed query block qb, over the real tokens j
    of the key blocks kept for (b, h, qb):  lse_i = ln sum_j exp(q_i . k_j * scale) and
    out_i = sum_j exp(q_i . k_j * scale - lse_i) v_j.  Computed directly (no online
    softmax), in fp64.

    Returns (tokens, out, lse): `tokens` lists the token indices covered (the listed
    blocks' tokens, block by block); out is [B, H, len(tokens), d], lse [B, H, len(tokens)]."""
    B, H, N, d = Q.shape
    if qblocks is None:
        qblocks = range(g.nB)
    qblocks = list(qblocks)
    tokens = np.concatenate([g.tokens_of_block[qb] for qb in qblocks])
    out = np.empty((B, H, tokens.size, d), dtype=np.float64)
    lse = np.empty((B, H, tokens.size), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            Kh = K[b, h].astype(np.float64)
            Vh = V[b, h].astype(np.float64)
            pos = 0
            for qb in qblocks:
                qt = g.tokens_of_block[qb]
                kept = np.nonzero(keep[b, h, qb])[0]
                kt = np.concatenate([g.tokens_of_block[j] for j in kept])
                S = (Q[b, h, qt].astype(np.float64) @ Kh[kt].T) * scale
                mx = S.max(axis=1, keepdims=True)
                l = mx[:, 0] + np.log(np.exp(S - mx).sum(axis=1))
                out[b, h, pos:pos + qt.size] = np.exp(S - l[:, None]) @ Vh[kt]
                lse[b, h, pos:pos + qt.size] = l
                pos += qt.size
    return tokens, out, lse


def dense_attn(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float,
               tokens: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of the listed query tokens (all by default) over every token."""
    B, H, N, d = Q.shape
    if tokens is None:
        tokens = np.arange(N)
    out = np.empty((B, H, len(tokens), d), dtype=np.float64)
    lse = np.empty((B, H, len(tokens)), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            S = (Q[b, h, tokens].astype(np.float64) @ K[b, h].astype(np.float64).T) * scale
            mx = S.max(axis=1, keepdims=True)
            l = mx[:, 0] + np.log(np.exp(S - mx).sum(axis=1))
            out[b, h] = np.exp(S - l[:, None]) @ V[b, h].astype(np.float64)
            lse[b, h] = l
    return out, lse


def layer(Q: np.ndarray, K: np.ndarray, V: np.ndarray, g: BlockGeometry, p: float,
          k_floor: int, scale: float, qblocks: Optional[Sequence[int]] = None) -> Dict:
    """The whole path for one attention layer: pool -> route -> masked attention."""
    Qp, Kp = pool(Q, g), pool(K, g)
    r = route(Qp, Kp, p, k_floor, scale)
    tokens, out, lse = masked_attn(Q, K, V, r.keep, g, scale, qblocks)
    return dict(Qp=Qp, Kp=Kp, route=r, tokens=tokens, out=out, lse=lse)
