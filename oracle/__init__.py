"""fp64 CPU oracle of the ZHA decode path - TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The CUDA library never links, loads or
calls it, and it shares no code with the CUDA path: both sides receive the
same seeded tensors from ``synth/`` and nothing else.

Every function here is pinned by ``tests/test_oracle_pins.py`` to something
other than itself (closed forms, brute force, the mathematics of the tangent
planes, the pages' coverage arithmetic).  The end-to-end kept sets on the
synthetic workloads are "parity unpinned" against the pages: the pages print
no worked numeric example and their trained reference queries are not
published.
"""
from .zha_oracle import *  # noqa: F401,F403
