"""fp64 CPU oracle for branch attention: test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The CUDA library never does.
"""
from .branch_attention import *  # noqa: F401,F403
from .branch_attention import (BITMASK, BLOCK, CHAIN, attend, backward_brute, backward_rows,  # noqa: F401
                               branch_part, default_scale, f64, forward_brute,
                               forward_decomposed, forward_ring, forward_rows, lse_merge,
                               main_part, row_first_keys, row_limits, visible_mask, visible_pair_count,
                               zigzag_chunks, branch_sees)
