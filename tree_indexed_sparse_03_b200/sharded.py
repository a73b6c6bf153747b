"""Sequence-sharded decode over several ranks: the exchange steps.

A context too long for one GPU is split into contiguous token ranges, one per
rank, on boundaries of the top-level nodes, so that every rank holds whole
subtrees and builds them exactly as a single tree would (a node's planes depend
only on the keys it covers: "Zyphra Hierarchical Attention", Zyphra blog,
section "Building the tree"; the summaries are merged recursively and exactly).
The tokens after the last complete top-level node (partial subtrees and the
tail) belong to the last rank.

Routing stays one global top-p descent per query head (blog, section "Routing
in the tree"; tanhow.com summary, section "How does top-p routing choose
tokens?"): at every step each rank scores its own candidates, and the softmax
over the candidates and the cut that keeps the smallest prefix reaching mass p
are taken over the candidates of all ranks.  The exchange is one all-gather per
step of (estimate, start token) per candidate.  Masses are compared as 2^-40
fixed-point integers relative to the step's largest estimate, so their sums are
exact and independent of which rank holds which candidate: the kept set is the
same for any number of ranks.  Candidates are ordered by (estimate descending,
start token ascending), as in the single-GPU routing.  Each rank then expands
its own kept nodes.

Attention runs on each rank over its own attended keys (its kept blocks, the
sink token 0 on the rank holding it, the tail on the last rank) and produces a
partial (m, l, o): running max, softmax denominator relative to m, and the
numerator vector.  One all-gather of the partials and the merge
o = sum_r e^(m_r - M) o_r / sum_r e^(m_r - M) l_r, with M = max_r m_r, give the
attention over the union of the attended sets.

The local work (the estimates of a list of nodes, the partial attention over a
token list) comes in as callbacks: on GPUs it is the routing and attention
kernels' work on each rank's tree, here the exchange logic alone.  The
collectives run on any torch.distributed backend (NCCL between GPUs, gloo on
the host); every rank takes the same collective steps in the same order, since
the loop ends when the global candidate count is zero.
"""
from __future__ import annotations

import math
from fractions import Fraction
from typing import Callable, List, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist

Node = Tuple[int, int]  # (level, index within the level); level 1 = leaf blocks

FIXED_ONE = 1 << 40  # fixed-point unit of the masses


def shard_ranges(n_tokens: int, block: int, levels: int, world: int) -> List[Tuple[int, int]]:
    """Token range [lo, hi) of every rank: whole top-level nodes (block**levels tokens each) split as evenly
    as possible; the tokens after the last complete top-level node go to the last rank."""
    top = block ** levels
    n_top = n_tokens // top
    bounds = [(n_top * r // world) * top for r in range(world)] + [n_tokens]
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def local_roots(n_tokens: int, block: int, levels: int, lo: int, hi: int) -> List[Node]:
    """The first candidates a rank holds: the complete top-level nodes in [lo, hi), then the roots of the
    partial subtrees there (the largest complete nodes not covered by a complete node one level up)."""
    n = [n_tokens // block ** l for l in range(levels + 1)]
    roots: List[Node] = []
    for level in range(levels, 0, -1):
        first = 0 if level == levels else block * n[level + 1]
        w = block ** level
        for i in range(first, n[level]):
            if lo <= i * w and (i + 1) * w <= hi:
                roots.append((level, i))
    return roots


def _gather(x: torch.Tensor, group=None) -> List[torch.Tensor]:
    """All-gather of 1-D tensors whose lengths differ between ranks (sizes first, then padded values)."""
    world = dist.get_world_size(group)
    n = torch.tensor([x.numel()], dtype=torch.int64, device=x.device)
    sizes = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(sizes, n, group=group)
    cap = max(1, max(int(s) for s in sizes))
    pad = torch.zeros(cap, dtype=x.dtype, device=x.device)
    pad[: x.numel()] = x
    out = [torch.zeros_like(pad) for _ in range(world)]
    dist.all_gather(out, pad, group=group)
    return [o[: int(s)] for o, s in zip(out, sizes)]


def top_p_keep(est: np.ndarray, start: np.ndarray, p: float) -> np.ndarray:
    """Indices of the kept candidates of one step: the shortest prefix in (estimate desc, start asc) order
    whose fixed-point mass reaches p of the total (p >= 1: all)."""
    n = est.size
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    order = np.lexsort((start, -est))
    if p >= 1.0:
        return order
    m = float(est.max())
    w = [int(round(math.exp(float(e) - m) * FIXED_ONE)) for e in est[order]]
    total = sum(w)
    frac = Fraction(p)
    thr = -(-(frac.numerator * total) // frac.denominator)  # ceil(p * total), exactly
    run = 0
    for k, wk in enumerate(w):
        run += wk
        if run >= thr:
            return order[: k + 1]
    return order


def route_sharded(score: Callable[[Sequence[Node]], np.ndarray], p, n_tokens: int, block: int, levels: int,
                  lo: int, hi: int, group=None) -> List[int]:
    """The kept level-1 blocks of this rank for one query head.

    ``score(nodes)`` returns the estimates of this rank's nodes; ``p`` is one threshold or one per step
    (later steps take the last).  Every rank must call it with the same query and thresholds.
    """
    rank = dist.get_rank(group)
    cand = local_roots(n_tokens, block, levels, lo, hi)
    leaves: List[int] = []
    s = 0
    while True:
        est = np.asarray(score(cand), dtype=np.float64) if cand else np.zeros(0)
        start = np.array([i * block ** l for l, i in cand], dtype=np.int64)
        g_est = _gather(torch.from_numpy(est), group)
        g_start = _gather(torch.from_numpy(start), group)
        if sum(t.numel() for t in g_est) == 0:
            break
        owner = np.concatenate([np.full(t.numel(), r, dtype=np.int64) for r, t in enumerate(g_est)])
        local = np.concatenate([np.arange(t.numel(), dtype=np.int64) for t in g_est])
        ps = float(p) if np.ndim(p) == 0 else float(p[min(s, len(p) - 1)])
        kept = top_p_keep(torch.cat(g_est).numpy(), torch.cat(g_start).numpy(), ps)
        nxt: List[Node] = []
        for j in kept:
            if owner[j] != rank:
                continue
            level, idx = cand[local[j]]
            if level == 1:
                leaves.append(idx)
            else:
                nxt += [(level - 1, block * idx + c) for c in range(block)]
        cand = nxt
        s += 1
    return sorted(leaves)


def attended_local(leaves: Sequence[int], n_tokens: int, block: int, lo: int, hi: int) -> np.ndarray:
    """This rank's attended tokens: its kept blocks, the sink token 0 if it holds it, the tail if it is the
    last rank (the tokens after the last complete block)."""
    parts = [np.arange(i * block, (i + 1) * block) for i in leaves]
    if lo == 0 and n_tokens > 0:
        parts.append(np.array([0]))
    if hi == n_tokens:
        parts.append(np.arange((n_tokens // block) * block, n_tokens))
    if not parts:
        return np.zeros(0, dtype=np.int64)
    return np.unique(np.concatenate(parts).astype(np.int64))


def combine_partials(parts: Sequence[Tuple[float, float, np.ndarray]]) -> np.ndarray:
    """Merge of partial softmax attentions (m, l, o): o = sum e^(m_r - M) o_r / sum e^(m_r - M) l_r."""
    live = [(m, l, o) for m, l, o in parts if np.isfinite(m)]
    M = max(m for m, _, _ in live)
    L = sum(math.exp(m - M) * l for m, l, _ in live)
    return sum(math.exp(m - M) * o for m, _, o in live) / L


def attend_sharded(partial: Callable[[np.ndarray], Tuple[float, float, np.ndarray]], tokens: np.ndarray, d: int,
                   group=None) -> np.ndarray:
    """Attention over the union of every rank's attended tokens: ``partial(tokens)`` gives this rank's
    (m, l, o) (m = -inf, l = 0, o = 0 for no tokens); one all-gather of the partials, then the merge."""
    if tokens.size:
        m, l, o = partial(tokens)
    else:
        m, l, o = -math.inf, 0.0, np.zeros(d)
    mine = torch.tensor(np.concatenate([[m, l], np.asarray(o, dtype=np.float64)]), dtype=torch.float64)
    world = dist.get_world_size(group)
    out = [torch.zeros_like(mine) for _ in range(world)]
    dist.all_gather(out, mine, group=group)
    return combine_partials([(float(t[0]), float(t[1]), t[2:].numpy()) for t in out])
