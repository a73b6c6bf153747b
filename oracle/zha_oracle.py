"""Plain fp64 restatement of Zyphra Hierarchical Attention (ZHA) decode.

TEST INFRASTRUCTURE ONLY (see the package docstring): slow, obviously correct,
numpy fp64, no blocking or fusion beyond what the method's definition states.

Sources (web pages about the method):
  [blog]    "Zyphra Hierarchical Attention" (translation of the Zyphra blog post,
            news.farwalk.ai), sections "Building the tree" (构建树), "Routing in
            the tree" (在树中路由), "How does this give subquadratic scaling?".
  [summary] "Zyphra发布ZHA稀疏注意力方法，可改造冻结大模型" (tanhow.com), sections
            "How does ZHA's tree indexer work? / Building the tree" and
            "How does top-p routing choose tokens?".
  [abstract] "Subquadratic Attention with a Hierarchical Tree-Structured
            Indexer" (arXiv 2610.42112 listing), abstract.

The pages state the method in words only.  The formulas used here are the
plain reading of those words, written out:

  * a block B of contiguous raw keys has log attention mass
    f_B(q) = log sum_{k in B} exp(q.k / sqrt(d));
  * at each reference query r_j the node stores the tangent plane of f_B:
    its value f_B(r_j), its slope mu_j / sqrt(d) with
    mu_j = sum_k softmax_k(r_j.k / sqrt(d)) k, and the intercept
    b_j = f_B(r_j) - r_j.mu_j / sqrt(d)   ([summary] "Building the tree": each
    reference query gives a tangent-plane estimate of the block's log mass);
  * the estimate for a new query is the maximum over the planes,
    e(q) = max_j (b_j + q.mu_j / sqrt(d))  (same passage: the max over the
    planes approximates the attention any future query gives the block);
  * summaries are merged recursively, b children per parent
    ([blog] "Building the tree": with block size four, one level covers 4 keys,
    two levels 16, six levels 4,096 tokens).  The merge is exact: parent
    f = logsumexp of the children's f, parent mu_j = children's mu_j weighted by
    the softmax of the children's f(r_j);
  * routing is top-down top-p: softmax the candidate estimates, keep the
    smallest set reaching mass p, expand only its children, repeat down to
    raw keys ([blog] "Routing in the tree"; [summary] "How does top-p routing
    choose tokens?"); order ties go to the lower start token;
  * final attention is ordinary softmax attention over the kept raw keys, with
    the first token always kept as the attention sink ([summary], same
    section) and the tail tokens not yet in a complete block always kept.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, Dict, List, Sequence, Tuple

import numpy as np

Node = Tuple[int, int]  # (level, index within level); level 1 = leaf blocks


# --------------------------------------------------------------------------- geometry
def level_counts(n_tokens: int, block: int, levels: int) -> List[int]:
    """Complete nodes per level: entry l is floor(n_tokens / block**l), l = 0..levels.

    A level-l node covers block**l contiguous tokens ([blog] "Building the
    tree": each level summarises block-times more keys).  Only complete nodes
    exist; tokens past the last complete leaf block form the tail.
    """
    return [n_tokens // block ** l for l in range(levels + 1)]


def node_span(node: Node, block: int) -> Tuple[int, int]:
    """Token range [start, end) covered by a node."""
    level, idx = node
    width = block ** level
    return idx * width, (idx + 1) * width


def forest_roots(n_tokens: int, block: int, levels: int) -> List[Node]:
    """First routing candidates: the complete top nodes plus the roots of partial subtrees.

    Reading: a partial subtree's root is the largest complete node not covered
    by a complete node one level up.  Listed by start token, these roots tile
    [0, block * n_1) exactly once (the base-``block`` digits of n_1).
    """
    n = level_counts(n_tokens, block, levels)
    roots: List[Node] = [(levels, i) for i in range(n[levels])]
    for level in range(levels - 1, 0, -1):
        roots += [(level, i) for i in range(block * n[level + 1], n[level])]
    return roots


def children(node: Node, block: int) -> List[Node]:
    level, idx = node
    return [(level - 1, block * idx + c) for c in range(block)]


# --------------------------------------------------------------------------- planes
@dataclass
class Planes:
    """Tangent planes of the nodes of one level: f [n, R], mu [n, R, d], bias [n, R]."""

    f: np.ndarray
    mu: np.ndarray
    bias: np.ndarray


def _logsumexp(x: np.ndarray, axis: int) -> np.ndarray:
    m = np.max(x, axis=axis, keepdims=True)
    return np.squeeze(m, axis) + np.log(np.sum(np.exp(x - m), axis=axis))


def leaf_planes(blocks: np.ndarray, refs: np.ndarray) -> Planes:
    """Planes of blocks of raw keys.

    blocks [n, b, d] (fp64), refs [R, d] (fp64).  For each block and each
    reference query r_j: scores s_k = r_j.k / sqrt(d); f = logsumexp_k s_k;
    w = softmax(s); mu_j = sum_k w_k k; b_j = f - r_j.mu_j / sqrt(d).
    ([summary] "Building the tree"; tangent plane of the log attention mass.)
    """
    d = blocks.shape[-1]
    s = np.einsum("nkd,rd->nrk", blocks, refs) / math.sqrt(d)        # [n, R, b]
    f = _logsumexp(s, axis=2)                                         # [n, R]
    w = np.exp(s - f[:, :, None])                                     # softmax over the block
    mu = np.einsum("nrk,nkd->nrd", w, blocks)                         # [n, R, d]
    bias = f - np.einsum("nrd,rd->nr", mu, refs) / math.sqrt(d)
    return Planes(f, mu, bias)


def merge_planes(child: Planes, refs: np.ndarray, block: int) -> Planes:
    """Planes of the complete parents of one level from their ``block`` children.

    Exact recursive merge ([blog] "Building the tree": summaries are grouped
    and compressed again, recursively): parent f(r_j) = logsumexp over the
    children of f_c(r_j); parent mu_j = sum_c softmax_c(f_c(r_j)) mu_{c,j};
    b_j = f - r_j.mu_j / sqrt(d).
    """
    d = refs.shape[-1]
    n_par = child.f.shape[0] // block
    R = refs.shape[0]
    fc = child.f[: n_par * block].reshape(n_par, block, R)
    muc = child.mu[: n_par * block].reshape(n_par, block, R, d)
    f = _logsumexp(fc, axis=1)                                        # [n_par, R]
    a = np.exp(fc - f[:, None, :])                                    # softmax over children
    mu = np.einsum("pcr,pcrd->prd", a, muc)
    bias = f - np.einsum("prd,rd->pr", mu, refs) / math.sqrt(d)
    return Planes(f, mu, bias)


def build_tree(K: np.ndarray, refs: np.ndarray, n_tokens: int, block: int,
               levels: int) -> Dict[int, Planes]:
    """All complete nodes of one KV head's tree: level -> Planes.

    K [>= n_tokens, d] raw keys (fp64), refs [R, d].  Level 1 from raw blocks,
    levels 2..L by the exact merge.  The full raw cache stays available; the
    tree is for search only ([blog] "Building the tree", last paragraph).
    """
    n = level_counts(n_tokens, block, levels)
    d = K.shape[-1]
    tree = {1: leaf_planes(K[: n[1] * block].reshape(n[1], block, d), refs)}
    for level in range(2, levels + 1):
        tree[level] = merge_planes(tree[level - 1], refs, block)
    return tree


def node_planes_direct(K: np.ndarray, refs: np.ndarray, node: Node, block: int) -> Planes:
    """Planes of one node computed straight from the raw keys it covers (one block of b**level keys)."""
    s, e = node_span(node, block)
    return leaf_planes(K[s:e][None], refs)


def estimate(mu: np.ndarray, bias: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Max-of-planes estimate e(q) = max_j (b_j + q.mu_j / sqrt(d)) for a batch of nodes.

    mu [n, R, d], bias [n, R], q [d] -> [n].  ([summary] "Building the tree":
    the maximum over the planes approximates the attention any future query
    gives the block.)
    """
    d = mu.shape[-1]
    return np.max(bias + np.einsum("nrd,d->nr", mu, q) / math.sqrt(d), axis=1)


def log_mass(K: np.ndarray, node: Node, q: np.ndarray, block: int) -> float:
    """True log attention mass f_node(q) = logsumexp over the node's keys of q.k / sqrt(d)."""
    s, e = node_span(node, block)
    z = K[s:e] @ q / math.sqrt(K.shape[-1])
    m = z.max()
    return float(m + np.log(np.exp(z - m).sum()))


# --------------------------------------------------------------------------- FP4 router planes
# [summary] TL;DR: an FP4 router variant was also tested (no details given).  Reading: the router
# reads each slope row as 4-bit e2m1 codes with one
# e4m3 scale per 16 dimensions (the OCP microscaling element and scale formats), quantised from the
# stored slopes by round-to-nearest; the intercepts stay fp32.  The decisions (scale, codes) are taken in
# fp32 arithmetic, as the stored slopes are fp32-representable; the values are then exact.
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e4m3_nearest(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Nearest e4m3 value (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, largest finite 448) of
    each x >= 0, ties to the even mantissa, at most 448: (values, encodings)."""
    x = np.asarray(x, dtype=np.float64)
    vals = np.zeros_like(x)
    bits = np.zeros(x.shape, dtype=np.uint8)
    for i in np.ndindex(x.shape):
        v = float(x[i])
        if not v > 0:
            continue
        if v >= 448.0:
            vals[i], bits[i] = 448.0, 0x7E
            continue
        E = math.frexp(v)[1] - 1                  # v in [2^E, 2^(E+1))
        if E < -6:                                # subnormals: multiples of 2^-9
            m = float(np.rint(v * 2.0 ** 9))
            vals[i], bits[i] = m * 2.0 ** -9, int(m)
            continue
        m = float(np.rint(v * 2.0 ** (3 - E)))   # in [8, 16]
        if m == 16.0:
            m, E = 8.0, E + 1
        val = m * 2.0 ** (E - 3)
        if val > 448.0:
            vals[i], bits[i] = 448.0, 0x7E
        else:
            vals[i], bits[i] = val, ((E + 7) << 3) | (int(m) - 8)
    return vals, bits


def e4m3_decode(bits: np.ndarray) -> np.ndarray:
    """Values of e4m3 encodings (finite ones)."""
    b = np.asarray(bits).astype(np.int64)
    e, m = (b >> 3) & 15, (b & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    return np.where((b & 128) != 0, -mag, mag)


def e2m1_code(y: np.ndarray) -> np.ndarray:
    """e2m1 code (bit 3 the sign, bits 0-2 the index into E2M1_VALUES) of the nearest representable value
    of each y, ties to the even mantissa, magnitude at most 6; magnitude 0 is coded +0."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    # index i has mantissa bit i & 1 (i >= 1): a tie between i and i+1 goes to the even one
    idx = np.zeros(a.shape, dtype=np.uint8)
    for i in range(1, 8):
        lo, hi = E2M1_VALUES[i - 1], E2M1_VALUES[i]
        mid = (lo + hi) / 2
        up = (a > mid) | ((a == mid) & (i % 2 == 0))   # above the midpoint, or at it with i even
        idx = np.where(up, np.uint8(i), idx)
    return np.where(idx == 0, 0, idx | np.where(y < 0, 8, 0)).astype(np.uint8)


def quantize_fp4(mu: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Codes [..., d] and scale encodings [..., d/16] of slope rows mu [..., d] (fp32-representable)."""
    m32 = np.asarray(mu, dtype=np.float32)
    g = m32.reshape(*m32.shape[:-1], m32.shape[-1] // 16, 16)
    amax = np.abs(g).max(axis=-1)
    sval, sbits = e4m3_nearest((amax / np.float32(6)).astype(np.float32))   # fp32 division
    s32 = sval.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (g / s32[..., None]).astype(np.float32)                            # fp32 division
    codes = np.where(s32[..., None] > 0, e2m1_code(y), 0).astype(np.uint8)
    return codes.reshape(m32.shape), sbits


def dequantize_fp4(codes: np.ndarray, sbits: np.ndarray) -> np.ndarray:
    """Slopes code * scale (exact) from codes [..., d] and scale encodings [..., d/16]."""
    c = np.asarray(codes).astype(np.int64)
    v = E2M1_VALUES[c & 7] * np.where((c & 8) != 0, -1.0, 1.0)
    return v * np.repeat(e4m3_decode(sbits), 16, axis=-1)


# --------------------------------------------------------------------------- routing
@dataclass
class RouteStep:
    """One top-p step: candidates, their estimates, the order and the cut."""

    cand: List[Node]
    ehat: np.ndarray          # estimate of each candidate (candidate order)
    order: np.ndarray         # candidate indices in (ehat desc, start asc) order
    cum: np.ndarray           # cumulative softmax mass along ``order``
    k: int                    # number kept (a prefix of ``order``)
    p: float = 1.0            # the step's threshold


@dataclass
class RouteTrace:
    leaves: List[int] = field(default_factory=list)     # kept level-1 block indices
    steps: List[RouteStep] = field(default_factory=list)


PlanesFn = Callable[[int, np.ndarray], Tuple[np.ndarray, np.ndarray]]


def top_p_count(ehat: np.ndarray, order: np.ndarray, p: float) -> Tuple[int, np.ndarray]:
    """Size of the smallest prefix of ``order`` whose softmax mass reaches p.

    "Reaching p" reads as cumulative mass >= p.  p >= 1 keeps every candidate
    (so that rounding can never drop one and p = 1 is dense attention).
    """
    m = ehat.max()
    pi = np.exp(ehat - m)
    pi = pi / pi.sum()
    cum = np.cumsum(pi[order])
    if p >= 1.0:
        return len(order), cum
    hit = np.nonzero(cum >= p)[0]
    k = int(hit[0]) + 1 if hit.size else len(order)
    return k, cum


def step_threshold(p, s: int) -> float:
    """Threshold of routing step s (s = 0 scores the roots).

    ``p`` is one value for every step, or a sequence with one value per step
    (later steps take the last one): the blog's closing section ("matching the
    degree of compression to the predictive information") and the review's
    section on thresholds that follow depth and content say a fixed top-p at
    every level is not enough and the threshold should change with tree depth
    and context length; they give no schedule, so the schedule is an input.
    """
    if np.ndim(p) == 0:
        return float(p)
    return float(p[min(s, len(p) - 1)])


def route(planes: PlanesFn, q: np.ndarray, p, n_tokens: int, block: int,
          levels: int) -> RouteTrace:
    """Top-down top-p routing of one query head ([blog] "Routing in the tree").

    ``planes(level, idx_array)`` returns (mu [n, R, d], bias [n, R]) of the
    requested nodes - the oracle's own tree or planes read back from the GPU.
    Start: the forest roots.  Each step softmaxes the candidate estimates,
    keeps the smallest prefix (ehat descending, lower start token first on
    ties) reaching mass p (``step_threshold(p, s)`` at step s); kept level-1
    nodes are final, kept higher nodes contribute their ``block`` children to
    the next candidate set.
    """
    trace = RouteTrace()
    cand = forest_roots(n_tokens, block, levels)
    s = 0
    while cand:
        ehat = np.empty(len(cand))
        lv = np.array([c[0] for c in cand])
        ix = np.array([c[1] for c in cand])
        for level in np.unique(lv):
            sel = np.nonzero(lv == level)[0]
            mu, bias = planes(int(level), ix[sel])
            ehat[sel] = estimate(mu, bias, q)
        start = ix * np.array([block ** int(v) for v in lv])
        order = np.lexsort((start, -ehat))        # primary: ehat desc; secondary: start asc
        ps = step_threshold(p, s)
        k, cum = top_p_count(ehat, order, ps)
        trace.steps.append(RouteStep(cand, ehat, order, cum, k, ps))
        s += 1
        nxt: List[Node] = []
        for j in order[:k]:
            node = cand[j]
            if node[0] == 1:
                trace.leaves.append(node[1])
            else:
                nxt += children(node, block)
        cand = nxt
    trace.leaves.sort()
    return trace


def retained_mass(trace: RouteTrace) -> float:
    """Estimated attention mass a route keeps: the product over its steps of the
    share of the step's candidate mass (the softmax of their estimates) that the
    step keeps.  The blog's section on attention becoming too sparse notes that
    keeping a fixed share of the probability at every level keeps, after the
    whole descent, a share of the original mass that shrinks with depth; each
    step keeps at least its threshold, so the product is at least the product
    of the thresholds of the steps taken (1 when every step keeps everything).
    """
    return float(np.prod([st.cum[st.k - 1] if st.k > 0 else 0.0 for st in trace.steps]))


def route_multi(planes: PlanesFn, Qm: np.ndarray, p, n_tokens: int, block: int,
                levels: int) -> List[RouteTrace]:
    """Routing of m queries of one context (e.g. the queries of a prefill chunk): each query head is routed
    on its own, exactly as a decode query ([blog] "Routing in the tree"); the queries share only the tree.
    The pages model decode only ([summary] "ZHA 有多快？"); sharing the first step's scoring between the
    queries is a question of how it is computed, not of what."""
    return [route(planes, q, p, n_tokens, block, levels) for q in Qm]


def tree_planes_fn(tree: Dict[int, Planes]) -> PlanesFn:
    return lambda level, idx: (tree[level].mu[idx], tree[level].bias[idx])


# --------------------------------------------------------------------------- attention
def attended_tokens(leaves: Sequence[int], n_tokens: int, block: int) -> np.ndarray:
    """Sorted unique token set a query attends to: kept blocks + sink + tail.

    Token 0 is always kept as the attention sink ([summary] "How does top-p
    routing choose tokens?").  Tokens after the last complete block are not
    in any node and are always attended (plain reading for causal decode).
    """
    n1 = n_tokens // block
    parts = [np.arange(i * block, (i + 1) * block) for i in leaves]
    if n_tokens > 0:
        parts.append(np.array([0]))
    parts.append(np.arange(n1 * block, n_tokens))
    return np.unique(np.concatenate(parts).astype(np.int64))


def attend(K: np.ndarray, V: np.ndarray, q: np.ndarray, tokens: np.ndarray) -> np.ndarray:
    """Ordinary softmax attention of q over the given token subset (max-subtracted, fp64)."""
    s = K[tokens] @ q / math.sqrt(K.shape[-1])
    w = np.exp(s - s.max())
    return (w / w.sum()) @ V[tokens]


def dense(K: np.ndarray, V: np.ndarray, q: np.ndarray, n_tokens: int) -> np.ndarray:
    """Dense decode attention over all n_tokens cached keys."""
    return attend(K, V, q, np.arange(n_tokens))


def decode_head(K: np.ndarray, V: np.ndarray, planes: PlanesFn, q: np.ndarray, p,
                n_tokens: int, block: int, levels: int) -> Tuple[np.ndarray, RouteTrace]:
    """Route + attend for one query head of one sequence."""
    trace = route(planes, q, p, n_tokens, block, levels)
    tokens = attended_tokens(trace.leaves, n_tokens, block)
    return attend(K, V, q, tokens), trace
