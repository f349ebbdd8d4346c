"""Workload shapes of the Swimba (Switch Mamba) layer.

Five synthetic workloads, named by what they are. Each fixes the layer shape (batch B, sequence
length L, channels D = d_inner, state size N = d_state, low-rank dt width R = dt_rank, expert count
E, active experts k), the dtype of the activations ("io") and of the expert projection tables, and
the seed of the synthetic draw. The initialisation recipe they share is implemented in
``synth.py``.

The decode workload runs ``decode_steps`` single-token steps on a cached state of shape [B, D, N].
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class LayerConfig:
    name: str
    batch: int
    seqlen: int
    d_inner: int
    d_state: int
    dt_rank: int
    n_experts: int
    top_k: int
    io_dtype: str  # "f32" or "bf16": x, z and out
    w_dtype: str  # "f32" or "bf16": W_x and W_dt
    seed: int
    decode_steps: int = 0  # > 0: a recurrent decode workload of single-token steps
    cached_state: bool = False  # draw a starting state h0 ~ N(0, 0.1) (variance 0.1)

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    @property
    def xdbl_width(self) -> int:
        """Width of one expert's stage-1 projection: [dt_low (R) | B (N) | C (N)]."""
        return self.dt_rank + 2 * self.d_state

    def with_(self, **kw) -> "LayerConfig":
        return replace(self, **kw)


CONFIGS: dict[str, LayerConfig] = {
    # Tiny fp32 layer: B=1, L=128, D=128, N=16, R=8, E=4, top-1.
    "tiny_fp32": LayerConfig("tiny_fp32", 1, 128, 128, 16, 8, 4, 1, "f32", "f32", 0),
    # Mamba-130M-like channel width, bf16 activations, fp32 state: B=4, L=2048, D=1536, R=48,
    # E=8, top-2.
    "mamba130m_like": LayerConfig("mamba130m_like", 4, 2048, 1536, 16, 48, 8, 2, "bf16", "bf16", 1),
    # Mamba-1.4B-like: B=8, L=4096, D=4096, R=128, E=8, top-2. Also timed as the E=1 dense scan.
    "mamba1p4b_like": LayerConfig("mamba1p4b_like", 8, 4096, 4096, 16, 128, 8, 2, "bf16", "bf16", 2),
    # Long sequence: B=1, L=65536, D=2048, R=64, E=16, top-2.
    "long_seq_65536": LayerConfig("long_seq_65536", 1, 65536, 2048, 16, 64, 16, 2, "bf16", "bf16", 3),
    # Recurrent decode: 256 sequences x 1 token per step, D=4096, R=128, E=8, top-2, 1000 steps.
    "decode_b256": LayerConfig(
        "decode_b256", 256, 1, 4096, 16, 128, 8, 2, "bf16", "bf16", 4, decode_steps=1000, cached_state=True
    ),
}

CONFIG_ORDER = ["tiny_fp32", "mamba130m_like", "mamba1p4b_like", "long_seq_65536", "decode_b256"]


def dense_variant(cfg: LayerConfig) -> LayerConfig:
    """The same shape with a single expert (E=1, k=1): the dense selective scan."""
    return cfg.with_(name=cfg.name + "_dense_e1", n_experts=1, top_k=1)
