"""B200-native sparse mixture-of-experts feed-forward layer.

The computation lives in libmoe.so (hand-written sm_100a CUDA behind the C
ABI of include/moe.h); this package is the thin Python binding over it.
"""

from .binding import (  # noqa: F401
    MOE_BF16, MOE_F32, MoEError, lib, lib_path,
    moe_workspace_size, moe_router_topk, moe_permute, moe_routing_stats, moe_expert_ffn,
    moe_layer_forward, moe_layer_forward_ex, moe_layer_forward_host, moe_layer_forward_host_wait,
    moe_layer_forward_noalloc,
    moe_stack_forward,
    moe_release_workspace,
    moe_device_errors, moe_last_error_string, moe_version,
    moe_profile_enable, moe_profile_read, moe_profile_stage_name, moe_profile_select,
    moe_set_gemm_variant, moe_set_wait_test,
)
