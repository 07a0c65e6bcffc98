"""Float64 CPU oracle (test infrastructure; see moe_oracle's header)."""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import (  # noqa: F401
    ACT_RELU, ACT_SILU_GATED, RENORM_EPS, combine, expert_outputs, moe_ffn_forward,
    moe_ffn_given_routing, moe_route, parameter_count, routing_weights, softmax, top_k,
    topk_gap,
)
