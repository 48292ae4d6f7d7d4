"""fp64 CPU oracle for permuted block-sparse attention prefill.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package smoke check
and by the benchmark's CPU-baseline leg, never by the product path.
"""
from .pbs_oracle import *  # noqa: F401,F403
from .pbs_oracle import (attn, attn_block, attn_blocks, attn_early_stop, attn_early_stop_block,
                         calibrate_thresholds, coverage_block, dense_lists,
                         diagonal_blocks, forced_blocks, inverse_permutation,
                         key_scores, key_tiles,
                         lists_to_array, n_candidates, natural_key_block_sums,
                         perm_for_block, permute, permute_segmented, permuted_key_block_sums,
                         proxy_query, segment_queries, select_sample, sample_pattern_scores,
                         sample_trunk_rows, cumulative_cut,
                         query_block_sums, segment_of_block, select,
                         sort_segments, tile_maxima, topk_target)
