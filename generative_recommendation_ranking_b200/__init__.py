"""MTGR HSTU-block forward for NVIDIA B200 (sm_100a).

The forward pass of the HSTU block and block stack of "MTGR: Industrial-Scale
Generative Recommendation Framework in Meituan" over user-aggregated, jagged
token sequences, implemented in libmtgr.so (hand-written CUDA for sm_100a)
behind a C ABI (include/mtgr.h). This package is the Python binding.
"""

from ._lib import (  # noqa: F401
    MTGR_BF16,
    MTGR_EPI_NONE,
    MTGR_EPI_RESID,
    MTGR_EPI_SILU,
    MTGR_F16,
    MTGR_F32,
    MTGR_VARIANT_POOLED_GLN,
    MTGR_VARIANT_SILU_QKVU,
    MTGR_VARIANT_RAB,
    MTGRError,
    load,
    mtgr_block_workspace_bytes,
    mtgr_build_mask_meta,
    mtgr_candidate_heads,
    mtgr_heads_workspace_bytes,
    mtgr_gemm,
    mtgr_group_layernorm,
    mtgr_group_layernorm_pooled,
    mtgr_hstu_attention_fwd,
    mtgr_hstu_block_fwd,
    mtgr_mask_meta_workspace_bytes,
    mtgr_pack_offsets,
    mtgr_restrict_work,
    mtgr_stack_fwd,
    mtgr_stack_candidates_workspace_bytes,
    mtgr_stack_fwd_candidates,
    mtgr_stack_fwd_rows,
    mtgr_stack_rows_workspace_bytes,
    mtgr_stack_workspace_bytes,
    mtgr_tokenize,
    mtgr_tokenize_workspace_bytes,
    mtgr_version,
    status_string,
)
from .api import (  # noqa: F401
    BatchContextCache,
    BlockWeights,
    CandidateHeads,
    ContextCache,
    TokenMLPs,
    candidate_heads,
    tokenize,
    PackedBatch,
    capacities,
    gemm,
    group_layernorm_pooled,
    group_layernorm,
    hstu_attention,
    hstu_block_forward,
    hstu_block_forward_train,
    hstu_block_backward,
    hstu_stack_forward,
    stack_workspace,
)
