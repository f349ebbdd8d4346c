"""fp64 CPU oracle of the Swimba layer and its surrounding block (``swimba_oracle``) and of the scan
in the Mamba-2 SSD form (``swimba_ssd_oracle``) -- test infrastructure, never the library's
compute path."""
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
