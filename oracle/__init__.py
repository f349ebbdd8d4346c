"""fp64 CPU oracle of the Swimba layer -- test infrastructure, never the library's compute path."""
from .swimba_oracle import (  # noqa: F401
    decode_step,
    expert_projections,
    layer_forward,
    route,
    router_logits,
    selective_scan,
    silu,
    softplus,
)
