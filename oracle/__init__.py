"""CPU oracle (test infrastructure only; see flexprefill.py's header)."""
from .flexprefill import *  # noqa: F401,F403
from .flexprefill import (PATTERN_QA, PATTERN_VS, QA_FLATTENED, QA_QUERYWISE,  # noqa: F401
                          n_blocks_of,
                          VS_BLOCKS, VS_TOKENS, pool_lines, select_head_vs_blocks,
                          vs_block_budget,
                          block_pool, cumulative_count,
                          cumulative_select, dense_attention, dense_lists, estimate,
                          estimated_block_map, flexprefill, js_distance, last_block_attention,
                          pattern, qa_budget, qa_row_budget, quantised_masses, select,
                          select_head_qa, select_head_qa_querywise,
                          select_head_vs, slash_block_distances, sparse_attention, tri_offset,
                          vs_budget)
