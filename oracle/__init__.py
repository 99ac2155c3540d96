"""fp64 CPU oracle for the DeltaLog decode step -- TEST INFRASTRUCTURE ONLY.

Nothing in the product path may import, call or execute this package: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm use it.  It shares no code with the CUDA library.

* ``eager`` -- the plain per-token recurrences of GDN, KDA and RWKV6 in fp64.
  DeltaLog changes only the physical schedule of the state writes, not the
  recurrence (DeltaLog technical summary, gist.science, section "Method";
  arXiv 2608.15533 abstract), so the eager recurrence IS the definition of
  what every DeltaLog step must return.
* ``deferred`` -- a separately written fp64 run of the DeltaLog schedule
  itself (dense base + bounded log, M-1 appends then one merge).  It exists
  only to test the equivalence invariant; it is never a reference value.

Pins (see ``tests/test_oracle_pins.py``): hand-worked examples under
``tests/golden/``, the Householder product form of the delta rule, exact
storage with orthonormal keys, the beta=0/alpha=1 no-op, the RWKV6 closed-form
sum and its reduction to causal linear attention, and deferred == eager for
every M in 1..33.
"""
from .recurrences import (  # noqa: F401
    gdn_eager, kda_eager, rwkv6_eager, eager, deferred,
)
