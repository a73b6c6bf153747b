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
