"""B200 (sm_100a) MoE token routing: fused softmax+top-k gating, expert align/permute,
activation permute-gather, top-k weighted combine and the expert-parallel sum of the
ranks' partial combines, as hand-written CUDA kernels behind the C ABI of
libmoe_route.so (include/moe_route.h).

The Python layer only marshals arguments (``binding``) and preallocates buffers
(``router.MoeRouter``); synthetic workloads live in ``inputs``.
"""
from .binding import (  # noqa: F401
    MOE_DTYPE_BF16, MOE_DTYPE_F32, MOE_ERR_BAD_EXPERT_ID, MOE_ERR_BAD_ROW, MOE_ERR_CUDA, MOE_ERR_INVALID_ARG,
    MOE_ERR_TIMEOUT, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_GATHER_HIDDEN_READY, MOE_GATHER_ZERO_PAD, MOE_OK,
    MOE_RENORMALIZE, MOE_DISPATCH_GIVEN_IDS, MOE_SCORING_SIGMOID,
    AlignResult, MoeError, alloc_align_outputs, alloc_workspace, load_library, moe_align_capacity,
    moe_align_num_blocks, moe_align_permute, moe_align_permute_noalloc, moe_align_workspace_bytes, moe_combine, moe_gather, moe_read_status,
    moe_reduce_partials,
    moe_route_dispatch, moe_route_dispatch_workspace_bytes, moe_topk_softmax, moe_version, moe_workspace_init,
    status_string, alloc_dispatch_workspace,
)
from .router import HostStepPipeline, MoeRouter  # noqa: F401

__all__ = [n for n in dir() if n.startswith("moe_") or n in ("MoeRouter", "HostStepPipeline", "MoeError", "AlignResult")]
