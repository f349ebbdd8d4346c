"""fp64 CPU oracle of the Swimba layer -- test infrastructure, never the library's compute path."""
from .swimba_oracle import (  # noqa: F401
    block_branches,
    block_decode_step,
    block_forward,
    causal_conv1d,
    decode_step,
    expert_projections,
    layer_forward,
    round_bf16,
    route,
    router_logits,
    selective_scan,
    silu,
    softplus,
)
