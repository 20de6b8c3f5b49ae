"""B200 (sm_100a) routed MoE FFN with an expert-parallel band decomposition.

The compute lives in lib/libexpert_decode.so (hand-written CUDA behind the C
ABI of include/expert_decode.h).  This package only marshals torch tensors
into that ABI: every step of the path runs in the library's kernels, and
nothing here falls back to the CPU.
"""
from .api import (  # noqa: F401
    EP_OK, EP_EINVAL, EP_EDIM, EP_EBADID, EP_ENOMEM, EP_ECUDA, EP_ETIMEOUT,
    EPError, Plan, WorkspaceLayout, ep_plan, moe_route, moe_route_logits, moe_route_sigmoid,
    moe_ffn_workspace_size, moe_ffn_workspace_layout,
    moe_ffn_forward,
    moe_ffn_forward_noalloc,
    NvFp4, moe_ffn_nvfp4_workspace_size, moe_ffn_forward_nvfp4,
    ep_check_status, ep_set_dispatch, ep_set_router, ep_last_launch_count, ep_profile_events, library,
    library_path,
)
