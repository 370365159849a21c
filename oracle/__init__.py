"""fp64 CPU oracle of the sparse MoE layer.  Test infrastructure only: the
product path never imports it."""

from .moe_oracle import (  # noqa: F401
    router_logits, logit_sum_bound, topk_lower_index, kept_softmax, route,
    silu, swiglu_expert, moe_forward, permute, routing_stats,
)
