"""Sequence-sharded decode (tree_indexed_sparse_03_b200/sharded.py) on CPU ranks with gloo, world size 2.

Each rank holds a contiguous token range aligned to top-level nodes.  Its local work (node estimates,
partial attention) is done here with the oracle on the rank's own tree; the exchange steps (one all-gather
per routing step, one for the attention partials) are the module's.  Checked against the single tree:
  - a rank's own tree, built from its token range alone, has the planes of the global tree's nodes there;
  - the kept blocks of the two ranks together equal the single-rank route (exact integer masses make the
    cut independent of the sharding) and the oracle's route on the whole tree;
  - the merged attention equals the oracle's attention over the union of the attended tokens (fp64).
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    # n_tokens, block, levels, n_refs, d, p
    (3001, 4, 3, 4, 64, 0.9),
    (2500, 3, 4, 2, 64, [0.99, 0.8, 0.7]),
    (700, 8, 2, 3, 128, 0.75),
]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case_inputs(ci):
    sys.path.insert(0, ROOT)
    from synth.workloads import small_topics, generate
    n, block, levels, R, d, p = CASES[ci]
    w = small_topics(n, d=d, n_q_heads=4, n_kv_heads=1, block=block, levels=levels, n_refs=R, p=0.9, batch=1)
    inp = generate(w)
    return inp, n, block, levels, R, d, p


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle.zha_oracle as zo
    from tree_indexed_sparse_03_b200 import sharded as sh
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        selves = [dist.new_group([r]) for r in range(world)]  # single-rank groups: the unsharded run
        res = []
        for ci in range(len(CASES)):
            inp, n, block, levels, R, d, p = _case_inputs(ci)
            K = inp.K[0, :n].double().numpy()
            V = inp.V[0, :n].double().numpy()
            refs = inp.refs[0].double().numpy()
            lo, hi = sh.shard_ranges(n, block, levels, world)[rank]
            # the rank's own tree over its token range (node indices shifted to global ones)
            top = block ** levels
            own = zo.build_tree(K[lo:hi], refs, hi - lo, block, levels) if hi > lo else {}
            glob = zo.build_tree(K, refs, n, block, levels)
            plane_err = 0.0
            for level, pl in own.items():
                off = lo // block ** level
                cnt = pl.f.shape[0]
                g = glob[level]
                plane_err = max(plane_err, float(np.abs(pl.mu - g.mu[off:off + cnt]).max(initial=0.0)),
                                float(np.abs(pl.bias - g.bias[off:off + cnt]).max(initial=0.0)))
            assert lo % top == 0

            def score_fn(nodes, q):
                est = np.empty(len(nodes))
                for i, (level, idx) in enumerate(nodes):
                    pl = own[level]
                    j = idx - lo // block ** level
                    est[i] = zo.estimate(pl.mu[j:j + 1], pl.bias[j:j + 1], q)[0]
                return est

            for h in range(inp.Q.shape[2]):
                q = inp.Q[0, 0, h].double().numpy()
                leaves = sh.route_sharded(lambda nodes: score_fn(nodes, q), p, n, block, levels, lo, hi)
                toks = sh.attended_local(leaves, n, block, lo, hi)

                def partial(tokens):
                    sv = K[tokens] @ q / np.sqrt(d)
                    m = float(sv.max())
                    wv = np.exp(sv - m)
                    return m, float(wv.sum()), wv @ V[tokens]

                o = sh.attend_sharded(partial, toks, d)
                # the same on this rank alone with the whole context (single-rank group)
                one = sh.route_sharded(
                    lambda nodes: zo.estimate(np.stack([glob[l].mu[i] for l, i in nodes]),
                                              np.stack([glob[l].bias[i] for l, i in nodes]), q),
                    p, n, block, levels, 0, n, group=selves[rank])
                res.append((ci, h, rank, leaves, o.tolist(), one, plane_err))
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def sharded_results():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = dict(q.get(timeout=300) for _ in range(world))
    for pr in procs:
        pr.join(60)
        assert pr.exitcode == 0
    return got


def test_shard_ranges_tile_the_context():
    sys.path.insert(0, ROOT)
    from tree_indexed_sparse_03_b200 import sharded as sh
    import oracle.zha_oracle as zo
    for n, b, L in [(3001, 4, 3), (64, 4, 3), (5, 4, 3), (10000, 8, 2)]:
        for world in (1, 2, 3, 5):
            rs = sh.shard_ranges(n, b, L, world)
            assert rs[0][0] == 0 and rs[-1][1] == n
            assert all(a[1] == b_[0] for a, b_ in zip(rs, rs[1:]))
            roots = [r for lo, hi in rs for r in sh.local_roots(n, b, L, lo, hi)]
            assert sorted(roots) == sorted(zo.forest_roots(n, b, L))


def test_shards_reproduce_the_single_tree(sharded_results):
    sys.path.insert(0, ROOT)
    import oracle.zha_oracle as zo
    by = {}
    for rank, res in sharded_results.items():
        for ci, h, r, leaves, o, one, plane_err in res:
            assert plane_err <= 1e-12, plane_err
            by.setdefault((ci, h), []).append((r, leaves, o, one))
    assert by
    for (ci, h), parts in by.items():
        parts.sort()
        union = sorted(l for _, leaves, _, _ in parts for l in leaves)
        single = parts[0][3]
        assert parts[1][3] == single
        assert union == single, (ci, h)
        # the oracle's route and attention on the whole tree
        inp, n, block, levels, R, d, p = _case_inputs(ci)
        K = inp.K[0, :n].double().numpy()
        V = inp.V[0, :n].double().numpy()
        tree = zo.build_tree(K, inp.refs[0].double().numpy(), n, block, levels)
        q = inp.Q[0, 0, h].double().numpy()
        o_ref, trace = zo.decode_head(K, V, zo.tree_planes_fn(tree), q, p, n, block, levels)
        assert union == trace.leaves, (ci, h)
        assert parts[0][2] == parts[1][2]  # every rank holds the merged output
        assert np.abs(np.array(parts[0][2]) - o_ref).max() <= 1e-12


def test_top_p_keep_matches_the_oracle_cut():
    """The exchange's fixed-point cut keeps the same prefix of the same (estimate desc, start asc) order as the
    oracle's fp64 cut, except where the cumulative mass at the cut lies within rounding of p; p >= 1 keeps all."""
    sys.path.insert(0, ROOT)
    from tree_indexed_sparse_03_b200 import sharded as sh
    import oracle.zha_oracle as zo
    rng = np.random.default_rng(5)
    near = 0
    for trial in range(400):
        n = int(rng.integers(1, 80))
        est = rng.normal(size=n) * float(rng.choice([0.5, 2.0, 8.0]))
        if trial % 4 == 0:
            est = np.round(est)  # exact ties: the lower start goes first
        start = rng.permutation(n).astype(np.int64) * 4
        p = float(rng.choice([0.3, 0.7, 0.95, 0.999, 1.0]))
        kept = sh.top_p_keep(est, start, p)
        order = np.lexsort((start, -est))
        k, cum = zo.top_p_count(est, order, p)
        assert list(kept) == list(order[: len(kept)])
        if p >= 1.0:
            assert len(kept) == n
        elif len(kept) != k:
            near += 1
            j = min(k, len(kept)) - 1
            assert abs(cum[j] - p) <= 1e-9, (trial, k, len(kept), cum[j], p)
    assert near <= 4
