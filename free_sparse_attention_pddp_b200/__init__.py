"""MC-Sparse (Meta-Cached Sparse Attention) hot path for NVIDIA B200.

The compute lives in ``libmcs.so`` (hand-written sm_100a CUDA behind the C ABI
of ``include/mcs.h``). This package only marshals arguments: torch tensors give
device pointers and the current CUDA stream. There is no CPU or PyTorch
fallback: a missing or unloadable library raises.

``free_sparse_attention_pddp_b200.ulysses`` runs the same calls on a
sequence-sharded multi-GPU layout: one all-to-all turns sequence shards into
head shards before the per-head path, and one turns the output back.
"""
from .binding import (  # noqa: F401
    MCS_GROUP_SIZE, MCS_GROUP_WHITEN, MCS_INFO_WORDS, MCS_OP_ANCHOR, MCS_OP_DENSE, MCS_OP_GROUP, MCS_OP_SPARSE,
    MCSError, Shape, lib_path, load, mcs_anchor, mcs_dense, mcs_group, mcs_group_ex, mcs_group_fast, mcs_meta_copy,
    mcs_meta_mask_bytes, mcs_meta_pack,
    mcs_meta_unpack, mcs_poll_status, mcs_sparse,
    mcs_sparse_host, mcs_sparse_noalloc, mcs_status_string, mcs_workspace_bytes, workspace,
)
