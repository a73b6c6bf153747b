"""The oracle against its pins (closed forms, brute force, calculus, the pages' coverage figures)."""
import pytest

import oracle.zha_oracle as zo
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(zo)


def test_workload_geometries_match_pages():
    """The named workloads use the geometries the pages print (golden/geometries.txt)."""
    from oracle_pins import _read_table
    from synth.workloads import workload
    for name, block, levels, refs, p in _read_table("geometries.txt"):
        w = workload(name)
        assert w.block == int(block) and w.n_refs == int(refs) and abs(w.p - float(p)) < 1e-12
        if levels != "-":
            assert w.levels == int(levels)


def test_route_multi_is_m_single_routes():
    """The oracle's m-query route is m independent routes (the queries share the tree, nothing else)."""
    import numpy as np
    import oracle.zha_oracle as zo
    from synth.workloads import random_tree_case
    K, V, refs, Q = random_tree_case(5, n_tokens=900, d=64, n_q_heads=3, n_kv_heads=1, n_refs=4, batch=5, dtype="f32")
    tree = zo.build_tree(K[0].double().numpy(), refs[0].double().numpy(), 900, 4, 3)
    pf = zo.tree_planes_fn(tree)
    Qm = Q[:, 0].double().numpy()
    multi = zo.route_multi(pf, Qm, 0.8, 900, 4, 3)
    for q, tr in zip(Qm, multi):
        assert tr.leaves == zo.route(pf, q, 0.8, 900, 4, 3).leaves
    # and the routes differ between queries (the test would not notice a shared result otherwise)
    assert len({tuple(tr.leaves) for tr in multi}) > 1
