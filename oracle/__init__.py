"""CPU oracle of MiniMax Sparse Attention (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
and reference arms may import this package.  The library never does.
"""
from .msa_oracle import (LOCAL_BIAS, attended_rows, block_scores, boundary_scores,  # noqa: F401
                         indexer_append, local_block, logical_cache, msa_step, n_visible_blocks,
                         paged_append, pooled_scores, ranked_blocks, select_blocks, select_one,
                         sparse_attention, token_scores, dsa_token_scores, dsa_ranked_tokens,
                         dsa_select_one, dsa_select_tokens, dsa_boundary_scores, dsa_sparse_attention)
