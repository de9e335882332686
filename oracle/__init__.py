"""Plain fp64 CPU oracle for exact softmax attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA library (no kernels, headers, helpers or constants); both sides only
consume the same seeded inputs.

Everything here materialises the full score matrix S and the probabilities P,
one (sequence, query head) at a time, in float64, exactly as the definitions
on the source pages state them.  See ``oracle/attention.py`` for the
citations of each function.

Parity status: every public function is pinned by ``tests/test_oracle.py``
(pages' printed masks, torch fp64 SDPA / autograd, finite differences,
closed-form invariants).  The value of the LSE for a fully masked row
(-inf) is a convention the pages do not state: parity unpinned for that one
value (the pages only fix O = 0 for such rows).
"""

from .attention import (  # noqa: F401
    allowed_mask,
    head_forward,
    head_backward,
    mha_forward,
    mha_backward,
    varlen_forward,
    varlen_backward,
    kvcache_forward,
    kvcache_update_forward,
    logical_cache_rows,
    kv_head_of,
    merge_lse_partials,
)
