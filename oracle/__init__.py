"""fp64 CPU oracle for the attention forward and the BlockKVCache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library never
calls it, and it never imports the CUDA library: the only thing the two sides
share is the seeded input generator module, which holds none of the method's
arithmetic.

Contents:
  * ``sdpa`` / ``sdpa_rows``  -- ctypes front end of ``sdpa_oracle.c`` (fp64, OpenMP)
  * ``brute``                 -- pure-Python per-element loops for tiny inputs
  * ``kvcache_model``         -- plain Python model of the BlockKVCache contract
  * ``merge``                 -- fp64 merge of results over disjoint key sets (by LSE)
  * ``dca``                   -- fp64 dual chunk attention (three query forms by chunk distance)
"""
from .sdpa import sdpa, sdpa_rows, build_oracle, oracle_threads, MASK_KINDS  # noqa: F401
from .merge import merge, MERGE_PLANTS  # noqa: F401
from .dca import dca, DCA_PLANTS  # noqa: F401
