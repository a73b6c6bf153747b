"""zha_route_multi: m queries of one context routed and attended at once (the first routing step as one
tensor-core contraction of the roots' slopes with all the queries), against the fp64 oracle.

Stage-wise as for decode: the oracle's route of every query head on the GPU-stored planes must keep the GPU's
blocks (boundary cases counted), and the oracle's attention over the GPU's kept blocks must match the output.
The result must not depend on how the queries are grouped: the same queries through zha_decode give the same
kept blocks and outputs.
"""
import numpy as np
import pytest
import torch

import oracle.zha_oracle as zo
from parity_helpers import assert_close_out, compare_route, f64, oracle_attend_on_sets, p32
from synth.workloads import generate, random_queries, small_topics

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import tree_indexed_sparse_03_b200 as z


@pytest.fixture(scope="module")
def tree_case():
    n = 20011
    w = small_topics(n, d=128, n_q_heads=8, n_kv_heads=1, block=4, levels=4, n_refs=16, p=0.95, batch=1)
    inp = generate(w)
    cfg = z.make_config(d=128, n_q_heads=8, n_kv_heads=1, block=4, levels=4, n_refs=16, p=0.95, dtype="bf16",
                        capacity=n, max_batch=64)
    K, V = inp.K.cuda().contiguous(), inp.V.cuda().contiguous()
    tree = z.ZhaTree(cfg, K, V, inp.refs.cuda().contiguous())
    tree.build(n)
    torch.cuda.synchronize()
    tree.status()
    return w, inp, tree, n


@pytest.mark.parametrize("m,sample", [(16, None), (128, None), (1024, 96)])
def test_route_multi_against_oracle(tree_case, m, sample):
    w, inp, tree, n = tree_case
    Q = random_queries(40 + m, m, 8, 128, "bf16", topics_from=inp).cuda()
    O, (kept, cnt) = tree.route_multi(Q, want_kept=True)
    torch.cuda.synchronize()
    tree.status()
    heads = None
    rows = range(m)
    if sample:
        rows = sorted(np.random.default_rng(m).choice(m, sample, replace=False).tolist())
    Qs, ks, cs, Os = Q[rows].cpu(), kept[rows], cnt[rows], O[rows]
    rep = compare_route(tree, Qs, ks, cs, p32(0.95), n, 4, 4, 8, heads=heads)
    print(f"route_multi m={m}: {rep.summary()}")
    assert not rep.failures, "\n".join(rep.failures[:5])
    assert rep.flagged <= max(1, rep.heads // 64), rep.summary()
    ref = oracle_attend_on_sets(inp.K, inp.V, Qs, ks, cs, n, 4, 8)
    assert_close_out(Os.cpu().numpy(), ref, 2e-5 * float(inp.V[:, :n].abs().max()) + 1e-6, f"route_multi m={m}")


def test_route_multi_matches_decode(tree_case):
    """The same 64 queries through zha_route_multi and zha_decode: kept blocks equal, outputs equal where the
    kept blocks are (the first step's estimates are computed by different instructions, so a cut at a
    boundary may move; none does here)."""
    w, inp, tree, n = tree_case
    Q = random_queries(7, 64, 8, 128, "bf16", topics_from=inp).cuda()
    O1, (k1, c1) = tree.route_multi(Q, want_kept=True)
    O2, (k2, c2) = tree.decode(Q, want_kept=True)
    torch.cuda.synchronize()
    tree.status()
    same = (c1 == c2) & (k1 == k2).all(dim=-1)
    assert bool(same.all()), int((~same).sum())
    assert (O1 - O2).abs().max().item() <= 1e-5


def test_route_multi_errors(tree_case):
    w, inp, tree, n = tree_case
    with pytest.raises(ValueError):
        tree.route_multi(torch.zeros(4, 7, 128, dtype=torch.bfloat16, device="cuda"))
    from tree_indexed_sparse_03_b200 import zha as zb
    Q = torch.zeros(1, 8, 128, dtype=torch.bfloat16, device="cuda")
    O = torch.zeros(1, 8, 128, dtype=torch.float32, device="cuda")
    rc = zb.lib().zha_route_multi(tree._h, Q.data_ptr(), O.data_ptr(), 0, None, None, zb._stream(None))
    assert rc == zb.ZHA_ERR_INVALID
