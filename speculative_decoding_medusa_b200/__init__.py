"""Medusa decode-verify step on NVIDIA B200 (sm_100a).

The computation lives in libmedusa_b200.so (CUDA kernels behind a C ABI,
declared in include/medusa.h); this package is its thin Python binding plus
the seeded synthetic workloads used by the tests and the benchmark.
"""
from ._lib import (  # noqa: F401
    EXPORTS, LIB_PATH, MAX_BATCH, MAX_HEADS, MAX_KMAX, MAX_NODES, MEDUSA_ACCEPT_GREEDY,
    MEDUSA_ACCEPT_TYPICAL, MEDUSA_BF16, MEDUSA_F32,
    MedusaError, Tree, lib, medusa_heads_topk, medusa_heads_topk_tree,
    medusa_heads_topk_workspace_size,
    medusa_kv_compact, medusa_lmhead_verify, medusa_lmhead_verify_workspace_size,
    medusa_next_step, medusa_sample_bonus, medusa_topk_merge, medusa_tree_from_accuracies,
    medusa_verify_from_records, medusa_verify_records, medusa_verify_records_workspace_size,
    medusa_tree_attention, medusa_tree_attention_workspace_size,
    medusa_tree_build, medusa_verify_accept, medusa_verify_accept_compact,
    medusa_verify_accept_noalloc,
    medusa_verify_accept_workspace_size, medusa_wait_flag, new_status,
    workspace,
)
