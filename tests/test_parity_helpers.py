"""The route comparison of the parity tests (tests/parity_helpers.py) on the CPU: the overridable route is
the oracle's route when nothing is overridden, and a kept set is excused only when it is the oracle's route
with a flagged decision taken the other way."""
import numpy as np

import oracle.zha_oracle as zo
from parity_helpers import excused, route_overridden, step_flags
from synth.workloads import random_tree_case


def _case(seed=3, n=700, block=4, levels=3, R=4, d=64):
    K, V, refs, Q = random_tree_case(seed, n_tokens=n, d=d, n_q_heads=1, n_kv_heads=1, n_refs=R, batch=4,
                                     dtype="f32")
    Kh = K[0].double().numpy()
    tree = zo.build_tree(Kh, refs[0].double().numpy(), n, block, levels)
    return zo.tree_planes_fn(tree), [Q[b, 0].double().numpy() for b in range(4)], n, block, levels


def test_no_override_is_the_oracle_route():
    planes, qs, n, block, levels = _case()
    for q in qs:
        for p in (0.5, 0.9, 1.0):
            a = zo.route(planes, q, p, n, block, levels)
            b = route_overridden(planes, q, p, n, block, levels, {})
            assert a.leaves == b.leaves
            assert [st.k for st in a.steps] == [st.k for st in b.steps]


def test_keep_more_adds_a_candidate():
    planes, qs, n, block, levels = _case()
    q = qs[0]
    a = zo.route(planes, q, 0.8, n, block, levels)
    b = route_overridden(planes, q, 0.8, n, block, levels, {len(a.steps) - 1: "keep_more"})
    assert set(a.leaves) < set(b.leaves)
    assert len(b.leaves) == len(a.leaves) + 1


def test_excuse_needs_a_flag():
    planes, qs, n, block, levels = _case()
    q = qs[1]
    a = zo.route(planes, q, 0.8, n, block, levels)
    assert excused(a.leaves, a, planes, q, 0.8, n, block, levels) == []
    # one leaf more without any boundary on the path: not excused
    flagged = [f for s, st in enumerate(a.steps) for f in step_flags(s, st, planes, q)]
    other = route_overridden(planes, q, 0.8, n, block, levels, {len(a.steps) - 1: "keep_more"})
    if not flagged:
        assert excused(other.leaves, a, planes, q, 0.8, n, block, levels) is None


def test_boundary_flag_excuses_exactly_the_flipped_cut():
    """With p set to the cumulative mass at a cut, the cut is a boundary: the route keeping one candidate
    fewer there is excused, and so is the oracle's own set; a set that differs elsewhere is not."""
    planes, qs, n, block, levels = _case()
    q = qs[2]
    base = zo.route(planes, q, 0.9, n, block, levels)
    st = base.steps[0]
    if st.k < 2:
        return
    p = float(st.cum[st.k - 2]) + 5e-6   # the (k-1)-prefix misses p by less than 1e-5
    tr = zo.route(planes, q, p, n, block, levels)
    flags = step_flags(0, tr.steps[0], planes, q)
    assert any(f.kind == "keep_less" and f.tight for f in flags)
    fewer = route_overridden(planes, q, p, n, block, levels, {0: "keep_less"})
    used = excused(fewer.leaves, tr, planes, q, p, n, block, levels)
    assert used is not None and used[0].kind == "keep_less"
    wrong = sorted(set(tr.leaves) ^ {max(tr.leaves) + 1 if tr.leaves else 0})
    assert excused(wrong, tr, planes, q, p, n, block, levels) is None
