"""CPU oracle of the FlowCache hot path (test infrastructure only).

Nothing in the ``cache_gating_kv_b200`` package imports this.  Only the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs
may use it.
"""

from .flowcache_oracle import *  # noqa: F401,F403
