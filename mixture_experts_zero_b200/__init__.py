"""B200-native forward pass of a MoE layer with zero-computation experts, and its expert-bias
update (LongCat-Flash llm-wiki entity page, section 2.1).

The compute path is the C-ABI library ``libmoezero.so`` (hand-written sm_100a CUDA kernels);
this package only marshals torch tensors to it. The library is loaded on first use, and a
missing library raises instead of falling back to anything else.
"""
from .binding import (  # noqa: F401,E402
    LcMoeError,
    Shape,
    lc_moe_bias_update,
    lc_moe_check_wait_timeout,
    lc_moe_combine,
    lc_moe_expert_ffn,
    lc_moe_expert_hist,
    lc_moe_forward,
    lc_moe_forward_fp8,
    lc_moe_permute,
    lc_moe_quantize_e4m3,
    lc_moe_read_status,
    lc_moe_route,
    lc_moe_router_logits,
    lc_moe_set_wait_limit_ns,
    lc_moe_topk,
    lc_moe_workspace_bytes,
    library,
    new_workspace,
)
