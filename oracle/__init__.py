"""CPU oracle for Pyramid Sparse Attention (float64, NumPy).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``, never by the product
package.  It shares no code with the CUDA path."""
from .psa_oracle import *  # noqa: F401,F403
from .psa_oracle import (PRUNED, POOL, Pyramid, MaskResult, HeadResult, ForwardResult,
                         cdiv, pool_tokens, build_pyramid, block_rows, query_block_means,
                         block_logits, visible, straddles, rank_blocks, level_of,
                         apply_overrides, assign_levels, block_max_levels, correct_map, pyramid_attention, psa_head,
                         psa_forward, executed_flops)
