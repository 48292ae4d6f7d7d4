"""Permuted block-sparse attention prefill on B200 (sm_100a).

The compute lives in libpbs.so (hand-written CUDA behind a C ABI, see
include/pbs.h); this package is its Python binding, a host-memory prefill
driver that overlaps copies and kernels on CUDA streams (host_pipeline), and
the seeded synthetic input generator used by the tests and the benchmark.
"""
from ._binding import (EXPORTS, LIB_PATH, PBS_OP_ATTN, PBS_OP_PERMUTE, PBS_OP_PERMUTE_SEGMENTED,  # noqa: F401
                       PBS_OP_SELECT, PBS_OP_SELECT_SAMPLE, PBS_OP_SELECT_SEGMENTED,
                       PBS_OP_PERMUTE_QUERIES, PBS_SELECT_SAMPLE, PBS_SELECT_SCORE_ORDER, PBS_SELECT_TAU, PBS_SELECT_TOPK, PbsError, PbsTensor,
                       describe, load, pbs_attn_fwd, pbs_attn_fwd_early_stop, pbs_attn_fwd_qperm, pbs_check_device,
                       pbs_permute, pbs_permute_queries, pbs_permute_segmented, pbs_select, pbs_select_qperm,
                       select_capacity, version,
                       workspace_size)
