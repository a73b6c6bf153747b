"""Pins of the fp64 oracle to facts other than itself.

Each ``pin_*`` function raises AssertionError when the oracle module it is
given disagrees with a closed form, a brute-force computation, the calculus
of tangent planes or the pages' printed coverage arithmetic.  The same
functions run against the real oracle (tests/test_oracle_pins.py) and against
copies with planted mistakes (tests/test_oracle_mutations.py), so that every
plausible slip in the oracle is caught by at least one of them.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _rng(seed):
    return np.random.default_rng(seed)


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(1e-300, float(np.max(np.abs(b))) + 1e-30))


# ------------------------------------------------------------------ geometry pins
def pin_coverage_golden(zo):
    """Keys per node at a depth equal the pages' coverage figures (4, 16, 4096 at block 4)."""
    for block, levels, keys in _read_table("coverage.txt"):
        block, levels, keys = int(block), int(levels), int(keys)
        s, e = zo.node_span((levels, 0), block)
        assert e - s == keys, (block, levels, e - s, keys)
        s, e = zo.node_span((levels, 3), block)
        assert (s, e) == (3 * keys, 4 * keys)
        # a context of exactly one top node has exactly one root, covering all keys
        roots = zo.forest_roots(keys, block, levels)
        assert roots == [(levels, 0)], roots


def pin_top_counts(zo):
    """64 top nodes for 4,096 keys at (b=4, L=3) and for 262,144 keys at (b=4, L=6)."""
    assert zo.level_counts(4096, 4, 3)[3] == 64
    assert zo.level_counts(262144, 4, 6)[6] == 64
    assert zo.level_counts(262144, 256, 1)[1] == 1024
    assert len(zo.forest_roots(262144, 4, 6)) == 64


def pin_forest_tiles(zo):
    """Roots are disjoint complete nodes, sorted by start, tiling [0, b*n_1) exactly."""
    rng = _rng(1)
    for _ in range(200):
        b = int(rng.integers(2, 6))
        L = int(rng.integers(1, 5))
        n = int(rng.integers(0, 3 * b ** (L + 1)))
        roots = zo.forest_roots(n, b, L)
        n1 = n // b
        pos = 0
        for node in roots:
            s, e = zo.node_span(node, b)
            assert s == pos, (n, b, L, roots)
            assert 1 <= node[0] <= L
            pos = e
        assert pos == b * n1, (n, b, L, pos)
        # brute force: the number of roots is the digit sum of n1 in base b above level L
        top = n1 // b ** (L - 1)
        rest = n1 % b ** (L - 1)
        digits = 0
        while rest:
            digits += rest % b
            rest //= b
        assert len(roots) == top + digits


# ------------------------------------------------------------------ plane pins
def pin_zero_ref_is_mean(zo):
    """r = 0: the plane is flat at log(n); mu is the plain mean of the covered keys."""
    rng = _rng(2)
    K = rng.normal(size=(64, 8))
    refs = np.zeros((1, 8))
    tree = zo.build_tree(K, refs, 64, 4, 3)
    for level, pl in tree.items():
        n = 4 ** level
        for i in range(pl.f.shape[0]):
            s, e = i * n, (i + 1) * n
            assert abs(pl.f[i, 0] - math.log(n)) < 1e-12
            assert abs(pl.bias[i, 0] - math.log(n)) < 1e-12
            assert np.allclose(pl.mu[i, 0], K[s:e].mean(0), atol=1e-12, rtol=1e-12)


def pin_identical_keys_exact(zo):
    """All keys of a node equal k: e(q) = log n + q.k/sqrt(d) exactly, at every level."""
    rng = _rng(3)
    d = 16
    k = rng.normal(size=d)
    K = np.tile(k, (64, 1))
    refs = rng.normal(size=(3, d))
    tree = zo.build_tree(K, refs, 64, 4, 3)
    for _ in range(5):
        q = rng.normal(size=d) * 2
        for level, pl in tree.items():
            e = zo.estimate(pl.mu, pl.bias, q)
            want = math.log(4 ** level) + q @ k / math.sqrt(d)
            assert np.allclose(e, want, atol=1e-10), (level, e, want)


def pin_bias_is_entropy(zo):
    """b_j equals the entropy of softmax(r_j.k/sqrt(d)) over the covered keys; 0 <= b_j <= log n."""
    rng = _rng(4)
    d = 12
    K = rng.normal(size=(48, d)) * 1.3
    refs = rng.normal(size=(4, d))
    tree = zo.build_tree(K, refs, 48, 3, 2)
    for level, pl in tree.items():
        n = 3 ** level
        for i in range(pl.f.shape[0]):
            keys = K[i * n:(i + 1) * n]
            for j in range(refs.shape[0]):
                s = keys @ refs[j] / math.sqrt(d)
                w = np.exp(s - s.max())
                w /= w.sum()
                H = -float(np.sum(w * np.log(w)))
                assert abs(pl.bias[i, j] - H) < 1e-10, (level, i, j, pl.bias[i, j], H)
                assert -1e-12 <= pl.bias[i, j] <= math.log(n) + 1e-12


def pin_value_and_slope(zo):
    """f_j is the log mass at r_j; mu_j/sqrt(d) is its gradient there (central differences)."""
    rng = _rng(5)
    d = 10
    K = rng.normal(size=(32, d))
    refs = rng.normal(size=(3, d)) * 0.7
    tree = zo.build_tree(K, refs, 32, 2, 4)
    eps = 1e-5
    for level, pl in tree.items():
        for i in range(pl.f.shape[0]):
            node = (level, i)
            for j in range(refs.shape[0]):
                r = refs[j]
                assert abs(pl.f[i, j] - zo.log_mass(K, node, r, 2)) < 1e-11
                for _ in range(2):
                    u = rng.normal(size=d)
                    fd = (zo.log_mass(K, node, r + eps * u, 2) - zo.log_mass(K, node, r - eps * u, 2)) / (2 * eps)
                    assert abs(fd - u @ pl.mu[i, j] / math.sqrt(d)) < 1e-6, (level, i, j)


def pin_merge_exact(zo):
    """Every merged node equals the planes computed directly from its covered raw keys."""
    rng = _rng(6)
    d = 8
    for b, L, n in [(4, 3, 70), (2, 5, 45), (3, 3, 81)]:
        K = rng.normal(size=(n, d)) * 1.5
        refs = rng.normal(size=(5, d))
        tree = zo.build_tree(K, refs, n, b, L)
        for level, pl in tree.items():
            assert pl.f.shape[0] == n // b ** level
            for i in range(pl.f.shape[0]):
                direct = zo.node_planes_direct(K, refs, (level, i), b)
                assert _rel(pl.f[i], direct.f[0]) < 1e-12
                assert _rel(pl.mu[i], direct.mu[0]) < 1e-12
                assert _rel(pl.bias[i], direct.bias[0]) < 1e-10


def pin_convexity_bound(zo):
    """Tangent planes of a convex function lie below it: e(q) <= f_node(q), with equality at each r_j."""
    rng = _rng(7)
    d = 16
    K = rng.normal(size=(96, d)) * 1.2
    refs = rng.normal(size=(4, d))
    tree = zo.build_tree(K, refs, 96, 4, 3)
    for _ in range(10):
        q = rng.normal(size=d) * 2
        for level, pl in tree.items():
            e = zo.estimate(pl.mu, pl.bias, q)
            for i in range(pl.f.shape[0]):
                assert e[i] <= zo.log_mass(K, (level, i), q, 4) + 1e-10
    for level, pl in tree.items():
        for j in range(refs.shape[0]):
            e = zo.estimate(pl.mu, pl.bias, refs[j])
            for i in range(pl.f.shape[0]):
                assert abs(e[i] - zo.log_mass(K, (level, i), refs[j], 4)) < 1e-10


# ------------------------------------------------------------------ routing pins
def _brute_top_p(ehat, start, p):
    """Smallest subset reaching mass p (brute force over all subsets), then the canonical choice."""
    pi = np.exp(ehat - ehat.max())
    pi /= pi.sum()
    n = len(ehat)
    if p >= 1:
        return n
    for k in range(1, n + 1):
        if any(pi[list(c)].sum() >= p for c in itertools.combinations(range(n), k)):
            return k
    return n


def pin_minimal_prefix(zo):
    """Each step keeps a minimum-cardinality set reaching p, namely the first k by (e desc, start asc)."""
    rng = _rng(8)
    d = 8
    for trial in range(12):
        b = int(rng.integers(2, 5))
        L = int(rng.integers(1, 3))
        n = int(rng.integers(b, min(b ** (L + 1) * 3, 60)))
        K = rng.normal(size=(n, d)) * 2
        refs = rng.normal(size=(2, d))
        tree = zo.build_tree(K, refs, n, b, L)
        q = rng.normal(size=d) * 2
        p = float(rng.choice([0.3, 0.6, 0.9, 0.97]))
        trace = zo.route(zo.tree_planes_fn(tree), q, p, n, b, L)
        for step in trace.steps:
            if len(step.cand) > 14:
                continue
            start = np.array([zo.node_span(c, b)[0] for c in step.cand])
            assert step.k == _brute_top_p(step.ehat, start, p), (trial, step.k)
            want = sorted(range(len(step.cand)), key=lambda i: (-step.ehat[i], start[i]))[: step.k]
            assert sorted(step.order[: step.k].tolist()) == sorted(want)


def pin_step_thresholds(zo):
    """Per-step thresholds: a constant schedule equals the single p; every step keeps a minimum-cardinality
    set reaching its own threshold (brute force); a threshold of 1 at a step keeps all of that step."""
    rng = _rng(21)
    d = 8
    for trial in range(10):
        b = int(rng.integers(2, 5))
        L = int(rng.integers(2, 4))
        n = int(rng.integers(b ** 2, min(b ** (L + 1) * 2, 60)))
        K = rng.normal(size=(n, d)) * 2
        refs = rng.normal(size=(2, d))
        tree = zo.build_tree(K, refs, n, b, L)
        pf = zo.tree_planes_fn(tree)
        q = rng.normal(size=d) * 2
        p = float(rng.choice([0.4, 0.8, 0.95]))
        assert zo.route(pf, q, [p] * L, n, b, L).leaves == zo.route(pf, q, p, n, b, L).leaves
        sched = [float(x) for x in rng.choice([0.3, 0.6, 0.9, 1.0], size=int(rng.integers(1, L + 1)))]
        trace = zo.route(pf, q, sched, n, b, L)
        for s, step in enumerate(trace.steps):
            ps = sched[min(s, len(sched) - 1)]
            assert step.p == ps
            if ps >= 1:
                assert step.k == len(step.cand)
            if len(step.cand) <= 14:
                start = np.array([zo.node_span(c, b)[0] for c in step.cand])
                assert step.k == _brute_top_p(step.ehat, start, ps), (trial, s, step.k)


def pin_retained_mass(zo):
    """The retained estimated mass of a route: every step keeps at least its threshold of its candidates'
    softmax mass, so the product is at least the product of the thresholds and at most 1; a route with every
    threshold 1 keeps all of it (up to rounding); with threshold 1 at the roots and x at the next step the retained
    mass is that second step's kept share, summed here directly over the kept candidates' estimates."""
    rng = _rng(23)
    d = 8
    for trial in range(12):
        b = int(rng.integers(2, 5))
        L = int(rng.integers(2, 4))
        n = int(rng.integers(b ** 2, min(b ** (L + 1) * 2, 60)))
        K = rng.normal(size=(n, d)) * 2
        refs = rng.normal(size=(2, d))
        tree = zo.build_tree(K, refs, n, b, L)
        pf = zo.tree_planes_fn(tree)
        q = rng.normal(size=d) * 2
        sched = [float(x) for x in rng.choice([0.3, 0.6, 0.9, 0.99], size=L)]
        trace = zo.route(pf, q, sched, n, b, L)
        r = zo.retained_mass(trace)
        bound = float(np.prod([st.p for st in trace.steps]))
        assert bound - 1e-12 <= r <= 1 + 1e-12, (trial, r, bound)
        assert abs(zo.retained_mass(zo.route(pf, q, 1.0, n, b, L)) - 1.0) <= 1e-12
        x = float(rng.choice([0.5, 0.8]))
        tr2 = zo.route(pf, q, [1.0, x], n, b, L)
        if len(tr2.steps) == 2:  # (two levels: the roots, then the children of the kept top nodes)
            st = tr2.steps[1]
            kept = st.order[: st.k]
            w = np.exp(st.ehat - st.ehat.max())
            share = w[kept].sum() / w.sum()
            assert abs(zo.retained_mass(tr2) - share) <= 1e-12, (trial, zo.retained_mass(tr2), share)
            assert share >= x - 1e-12


def pin_e4m3_grid(zo):
    """Every finite non-negative e4m3 encoding decodes to its value and rounds back to itself; the values
    rise strictly from 0 through 2^-9 (smallest subnormal) and 2^-6 (smallest normal) to 448."""
    bits = np.arange(0, 127, dtype=np.uint8)          # 0x7F would be NaN
    vals = zo.e4m3_decode(bits)
    assert vals[0] == 0 and vals[1] == 2.0 ** -9 and vals[8] == 2.0 ** -6 and vals[-1] == 448.0
    assert np.all(np.diff(vals) > 0)
    v2, b2 = zo.e4m3_nearest(vals)
    assert np.array_equal(v2, vals) and np.array_equal(b2, bits)
    # midpoints go to the neighbour with the even mantissa, points off them to the nearer neighbour
    mids = (vals[1:] + vals[:-1]) / 2
    got, _ = zo.e4m3_nearest(mids)
    even = np.where(bits[:-1] % 2 == 0, vals[:-1], vals[1:])
    assert np.array_equal(got, even)
    below, _ = zo.e4m3_nearest(mids * (1 - 1e-9))
    above, _ = zo.e4m3_nearest(mids * (1 + 1e-9))
    assert np.array_equal(below, vals[:-1]) and np.array_equal(above, vals[1:])
    assert zo.e4m3_nearest(np.array([1e6]))[0][0] == 448.0


def pin_e2m1_codes(zo):
    """The eight e2m1 magnitudes code to themselves with either sign; midpoints go to the even mantissa
    (0, 1, 2, 4 are even); beyond 6 saturates."""
    vals = zo.E2M1_VALUES
    assert np.array_equal(zo.E2M1_VALUES[zo.e2m1_code(vals) & 7], vals)
    assert np.array_equal(zo.E2M1_VALUES[zo.e2m1_code(-vals) & 7], vals)
    assert np.all((zo.e2m1_code(-vals[1:]) & 8) == 8) and zo.e2m1_code(np.array([-0.1]))[0] == 0
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    assert np.array_equal(zo.E2M1_VALUES[zo.e2m1_code(ties)], [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0])
    assert zo.E2M1_VALUES[zo.e2m1_code(np.array([7.0, 100.0])) & 7].tolist() == [6.0, 6.0]


def pin_fp4_quantize(zo):
    """A group whose largest magnitude is 6 * (an e4m3 value) gets exactly that scale and codes it as +-6;
    every slope is within one scale step (the widest e2m1 gap is 4 to 6) of its value, within a quarter
    step where |v| / scale <= 2; an all-zero group has scale 0 and zero codes."""
    rng = _rng(31)
    mu = rng.normal(size=(6, 64)).astype(np.float32)
    mu[0, :16] = 0.0
    mu[1, 16:32] = np.float32(0.75) * rng.uniform(-1, 1, 16).astype(np.float32)
    mu[1, 16] = np.float32(6 * 0.125)                   # amax = 6 * 0.125, 0.125 is an e4m3 value
    codes, sb = zo.quantize_fp4(mu)
    dq = zo.dequantize_fp4(codes, sb)
    sc = np.repeat(zo.e4m3_decode(sb), 16, axis=-1)
    assert np.all(np.abs(dq - mu) <= sc + 1e-12)
    small = np.abs(mu) <= 2 * sc
    assert np.all(np.abs(dq - mu)[small] <= 0.25 * sc[small] + 1e-12)
    assert sb[0, 0] == 0 and np.all(codes[0, :16] == 0)
    assert zo.e4m3_decode(sb[1, 1]) == 0.125 and dq[1, 16] == 0.75
    # symmetric: negating the slopes negates the values
    c2, s2 = zo.quantize_fp4(-mu)
    assert np.array_equal(zo.dequantize_fp4(c2, s2), -dq)


def pin_cut_reaches_p_exactly(zo):
    """Four equal estimates at p = 0.5: mass 0.25 + 0.25 reaches p, so exactly two are kept."""
    e = np.zeros(4)
    order = np.arange(4)
    k, cum = zo.top_p_count(e, order, 0.5)
    assert k == 2, k
    k, _ = zo.top_p_count(e, order, 0.25)
    assert k == 1
    k, _ = zo.top_p_count(e, order, 1.0)
    assert k == 4


def pin_ties_lower_start(zo):
    """Identical blocks tie exactly; the lower start token is kept first."""
    d = 4
    k = np.array([1.0, -0.5, 0.25, 2.0])
    K = np.tile(k, (16, 1))              # four identical leaf blocks at b=4
    refs = np.eye(d)[:2]
    tree = zo.build_tree(K, refs, 16, 4, 1)
    for p, want in [(0.2, [0]), (0.3, [0, 1]), (0.6, [0, 1, 2]), (0.99, [0, 1, 2, 3])]:
        trace = zo.route(zo.tree_planes_fn(tree), np.ones(d), p, 16, 4, 1)
        assert trace.leaves == want, (p, trace.leaves)


def pin_children_expand(zo):
    """A kept non-leaf node hands exactly its b children (covering its span) to the next step."""
    rng = _rng(9)
    d = 8
    n, b, L = 64, 4, 3
    K = rng.normal(size=(n, d))
    refs = rng.normal(size=(2, d))
    tree = zo.build_tree(K, refs, n, b, L)
    trace = zo.route(zo.tree_planes_fn(tree), rng.normal(size=d), 0.8, n, b, L)
    for prev, nxt in zip(trace.steps[:-1], trace.steps[1:]):
        kept = [prev.cand[j] for j in prev.order[: prev.k] if prev.cand[j][0] > 1]
        spans = sorted(zo.node_span(c, b) for c in nxt.cand)
        want = sorted(s for node in kept for s in
                      [(zo.node_span(node, b)[0] + c * b ** (node[0] - 1),
                        zo.node_span(node, b)[0] + (c + 1) * b ** (node[0] - 1)) for c in range(b)])
        assert spans == want


def pin_single_key_blocks_exact(zo):
    """b = 1: every plane is exact, so routing is exact top-p over the true key masses."""
    rng = _rng(10)
    d = 8
    n = 13
    K = rng.normal(size=(n, d)) * 1.5
    refs = rng.normal(size=(2, d))
    tree = zo.build_tree(K, refs, n, 1, 1)
    for _ in range(5):
        q = rng.normal(size=d) * 2
        e = zo.estimate(tree[1].mu, tree[1].bias, q)
        assert np.allclose(e, K @ q / math.sqrt(d), atol=1e-12)
        for p in (0.5, 0.9):
            trace = zo.route(zo.tree_planes_fn(tree), q, p, n, 1, 1)
            s = K @ q / math.sqrt(d)
            pi = np.exp(s - s.max())
            pi /= pi.sum()
            order = np.argsort(-s, kind="stable")
            k = int(np.argmax(np.cumsum(pi[order]) >= p)) + 1
            assert trace.leaves == sorted(order[:k].tolist())


# ------------------------------------------------------------------ attention pins
def pin_attended_tokens(zo):
    """Sink and tail always attended, no token twice, kept blocks' tokens present."""
    assert zo.attended_tokens([2, 0], 13, 4).tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 12]
    assert zo.attended_tokens([], 13, 4).tolist() == [0, 12]
    assert zo.attended_tokens([], 3, 4).tolist() == [0, 1, 2]      # no complete block
    assert zo.attended_tokens([1], 8, 4).tolist() == [0, 4, 5, 6, 7]
    assert zo.attended_tokens([], 1, 4).tolist() == [0]


def pin_attend_bruteforce(zo):
    """Attention matches a pure-Python loop on a tiny case."""
    rng = _rng(11)
    K = rng.normal(size=(7, 3))
    V = rng.normal(size=(7, 3))
    q = rng.normal(size=3)
    toks = np.array([0, 2, 5, 6])
    num = [0.0, 0.0, 0.0]
    den = 0.0
    for t in toks.tolist():
        s = sum(q[i] * K[t, i] for i in range(3)) / math.sqrt(3)
        w = math.exp(s)
        den += w
        for i in range(3):
            num[i] += w * V[t, i]
    want = np.array(num) / den
    assert np.allclose(zo.attend(K, V, q, toks), want, atol=1e-13)


def pin_dense_vs_sdpa(zo):
    """Dense decode equals torch's scaled_dot_product_attention (fp64, CPU)."""
    import torch
    rng = _rng(12)
    K = rng.normal(size=(50, 16))
    V = rng.normal(size=(50, 16))
    q = rng.normal(size=16) * 3
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, None, None], torch.tensor(K)[None, None], torch.tensor(V)[None, None]
    )[0, 0, 0].numpy()
    assert np.allclose(zo.dense(K, V, q, 50), want, atol=1e-12)


def pin_p1_is_dense(zo):
    """p = 1 keeps every node, so ZHA decode equals dense decode."""
    rng = _rng(13)
    d = 8
    for n, b, L in [(45, 4, 2), (64, 4, 3), (10, 3, 2), (3, 4, 2), (130, 2, 6)]:
        K = rng.normal(size=(n, d))
        V = rng.normal(size=(n, d))
        refs = rng.normal(size=(3, d))
        tree = zo.build_tree(K, refs, n, b, L)
        q = rng.normal(size=d) * 2
        o, trace = zo.decode_head(K, V, zo.tree_planes_fn(tree), q, 1.0, n, b, L)
        assert trace.leaves == list(range(n // b))
        assert np.allclose(o, zo.dense(K, V, q, n), atol=1e-12)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
