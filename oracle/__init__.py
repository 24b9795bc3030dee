"""fp64 CPU oracle of the hybrid sparse + linear decode attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  The
product path (``hybrid_sparse_linear_decode_b200``) never imports, calls or
links anything here, and this package imports nothing from the product.

Parity status of each function (what pins it) is listed in ``oracle/hybrid.py``.
"""

from .hybrid import (  # noqa: F401
    Partition,
    partition,
    linear_state,
    block_stats,
    block_scores,
    select_blocks,
    strided_blocks,
    select_blocks_strided,
    exact_mask,
    hybrid_direct,
    hybrid_subtract,
    full_softmax,
    pure_taylor,
    brute_force_hybrid,
    OracleUnit,
)
