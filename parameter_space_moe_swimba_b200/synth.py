"""Seeded synthetic inputs for the Swimba layer.

This module draws random numbers and rounds them to their storage dtype. It holds no step of the
layer's computation (no routing, projection, mixing or scan), so the CPU oracle and the CUDA path
can both be fed from it without sharing any of the method's arithmetic.

Initialisation recipe (shared by every workload):

* x, z ~ N(0, 1), stored in the io dtype.
* Router W_r [D, E] ~ N(0, 1/D), fp32.
* Per expert e: W_x^e [D, R+2N] ~ N(0, 1/D) and W_dt^e [R, D] ~ N(0, 1/R), stored in the weight
  dtype; b_dt^e [D] = softplus^{-1}(dt) with dt ~ logU(1e-3, 1e-1), fp32.
* A^e[d, n] = -(n+1) * u^e_d with one u^e_d ~ U(0.5, 2) per (expert, channel), fp32
  ("structured"), or, for tests that must not see that power structure, an independent
  -logU(0.5, 32) per (e, d, n) ("random").
* D_skip [D] ~ N(0, 1), fp32.
* Cached decode state h0 [B, D, N] ~ N(0, 0.1) (variance 0.1), fp32.
* The surrounding block: u [B, L, d_model] ~ N(0, 1) in the io dtype; W_in [d_model, 2D] ~
  N(0, 1/d_model) and W_out [D, d_model] ~ N(0, 1/D) in the weight dtype; conv taps [D, W] and
  conv bias [D] ~ U(-1/sqrt(W), 1/sqrt(W)), fp32; a carried conv state [B, W-1, D] ~ N(0, 1) in
  the io dtype.

* Swimba on the Mamba-2 SSD form (heads of P channels, state N, one active expert per token):
  X [B, L, 1, H, P], B [B, L, 1, N] and the mixed readout C_mix [B, L, N] ~ N(0, 1) in bf16;
  gates 1 (top-1); step delta [B, L, H] ~ logU(1e-3, 1e-1) per (token, head); A_h = -U(1, 16) per
  head; D_skip [H] ~ N(0, 1); start state S0 [B, H, P, N] ~ N(0, 0.1), fp32.

N(m, s2) names the variance. bf16 values are rounded to nearest-even directly from the fp64 draw.

Random streams: every group of draws has its own PCG64 stream keyed by (seed, stream id, ...), so a
workload can be regenerated in pieces (one batch row, one decode step, one redrawn token) and the
pieces are identical to the whole.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .configs import LayerConfig

STREAM_WEIGHTS = 0
STREAM_ACTIVATIONS = 1
STREAM_REDRAW = 2
STREAM_STEP = 3
STREAM_H0 = 4
STREAM_BLOCK_WEIGHTS = 5
STREAM_BLOCK_INPUT = 6
STREAM_CONV_STATE = 7
STREAM_BLOCK_REDRAW = 8
STREAM_SSD = 9
STREAM_OUT_GRAD = 10

_BF16_MIN_NORMAL = 2.0 ** -126
_BF16_MAX = float.fromhex("0x1.fep127")


def rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


# --------------------------------------------------------------------------------------------
# Storage rounding
# --------------------------------------------------------------------------------------------

def round_f64_to_bf16_bits(a) -> np.ndarray:
    """Round fp64 values to bfloat16 (round to nearest, ties to even); returns the uint16 bits.

    bf16 keeps 8 significant bits, so 45 of fp64's 52 stored mantissa bits are dropped. Values
    must lie in bf16's normal range (or be 0); the draws here always do.
    """
    a = np.ascontiguousarray(a, dtype=np.float64)
    mag = np.abs(a)
    if np.any((mag != 0) & (mag < _BF16_MIN_NORMAL)) or np.any(mag > _BF16_MAX) or np.any(np.isnan(a)):
        raise ValueError("value outside the normal bf16 range")
    u = a.view(np.uint64)
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    u = (u + (np.uint64((1 << 44) - 1) + lsb)) & ~np.uint64((1 << 45) - 1)
    f32 = u.view(np.float64).astype(np.float32)  # exact: 8 significant bits, fp32 exponent range
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to(a64: np.ndarray, dtype: str) -> np.ndarray:
    """Storage form: uint16 bf16 bits for "bf16", float32 for "f32"."""
    if dtype == "bf16":
        return round_f64_to_bf16_bits(a64)
    if dtype == "f32":
        return np.asarray(a64, dtype=np.float64).astype(np.float32)
    raise ValueError(f"unknown dtype {dtype!r}")


def widen(stored: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 value of a stored array."""
    if dtype == "bf16":
        return bf16_bits_to_f32(stored).astype(np.float64)
    if dtype == "f32":
        return np.asarray(stored, dtype=np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


# --------------------------------------------------------------------------------------------
# Draws
# --------------------------------------------------------------------------------------------

@dataclass
class LayerWeights:
    W_r: np.ndarray  # [D, E] float32
    W_x: np.ndarray  # [E, D, R+2N] stored w_dtype
    W_dt: np.ndarray  # [E, R, D] stored w_dtype
    b_dt: np.ndarray  # [E, D] float32
    A: np.ndarray  # [E, D, N] float32, all < 0
    D_skip: np.ndarray  # [D] float32
    w_dtype: str


def inverse_softplus(y: np.ndarray) -> np.ndarray:
    """v with log(1 + e^v) = y, for y > 0 (the dt-bias initialisation)."""
    y = np.asarray(y, dtype=np.float64)
    return y + np.log(-np.expm1(-y))


def draw_weights(cfg: LayerConfig, a_mode: str = "structured") -> LayerWeights:
    D, N, R, E = cfg.d_inner, cfg.d_state, cfg.dt_rank, cfg.n_experts
    g = rng(cfg.seed, STREAM_WEIGHTS)
    W_r = g.standard_normal((D, E)) * np.sqrt(1.0 / D)
    W_x = g.standard_normal((E, D, R + 2 * N)) * np.sqrt(1.0 / D)
    W_dt = g.standard_normal((E, R, D)) * np.sqrt(1.0 / R)
    dt = np.exp(g.uniform(np.log(1e-3), np.log(1e-1), size=(E, D)))
    if a_mode == "structured":
        scale = g.uniform(0.5, 2.0, size=(E, D))
        A = -(np.arange(1, N + 1, dtype=np.float64)[None, None, :] * scale[:, :, None])
    elif a_mode == "random":
        A = -np.exp(g.uniform(np.log(0.5), np.log(32.0), size=(E, D, N)))
    else:
        raise ValueError(a_mode)
    D_skip = g.standard_normal(D)
    return LayerWeights(
        W_r=W_r.astype(np.float32),
        W_x=round_to(W_x, cfg.w_dtype),
        W_dt=round_to(W_dt, cfg.w_dtype),
        b_dt=inverse_softplus(dt).astype(np.float32),
        A=A.astype(np.float32),
        D_skip=D_skip.astype(np.float32),
        w_dtype=cfg.w_dtype,
    )


def draw_activations(cfg: LayerConfig, batch_rows=None) -> tuple[np.ndarray, np.ndarray]:
    """x, z [B, L, D] in storage form. Each batch row b has its own stream (seed, 1, b, which)."""
    rows = range(cfg.batch) if batch_rows is None else batch_rows
    shape = (len(rows), cfg.seqlen, cfg.d_inner)
    store = np.uint16 if cfg.io_dtype == "bf16" else np.float32
    x = np.empty(shape, dtype=store)
    z = np.empty(shape, dtype=store)
    for i, b in enumerate(rows):
        x[i] = round_to(rng(cfg.seed, STREAM_ACTIVATIONS, b, 0).standard_normal(shape[1:]), cfg.io_dtype)
        z[i] = round_to(rng(cfg.seed, STREAM_ACTIVATIONS, b, 1).standard_normal(shape[1:]), cfg.io_dtype)
    return x, z


def draw_step_activations(cfg: LayerConfig, step: int) -> tuple[np.ndarray, np.ndarray]:
    """x, z [B, 1, D] of decode step ``step`` (its own stream)."""
    g = rng(cfg.seed, STREAM_STEP, step)
    shape = (cfg.batch, 1, cfg.d_inner)
    x = round_to(g.standard_normal(shape), cfg.io_dtype)
    z = round_to(g.standard_normal(shape), cfg.io_dtype)
    return x, z


def draw_out_grad(cfg: LayerConfig) -> np.ndarray:
    """The incoming gradient dL/dout [B, L, D] ~ N(0, 1) in the io dtype's storage form (a
    backward pass's input; the loss itself is not modelled)."""
    g = rng(cfg.seed, STREAM_OUT_GRAD)
    return round_to(g.standard_normal((cfg.batch, cfg.seqlen, cfg.d_inner)), cfg.io_dtype)


def draw_h0(cfg: LayerConfig) -> np.ndarray:
    """Cached state [B, D, N] ~ N(0, 0.1), fp32."""
    g = rng(cfg.seed, STREAM_H0)
    return (g.standard_normal((cfg.batch, cfg.d_inner, cfg.d_state)) * np.sqrt(0.1)).astype(np.float32)


def redraw_x_row(cfg: LayerConfig, b: int, t: int, attempt: int, step: int = -1) -> np.ndarray:
    """A fresh x row [D] for token (b, t) in storage form, from stream (seed, 2, step+1, b, t, attempt).

    Used to move a token away from a near-tie of its router logits (the choice of which rows to
    redraw is made by the caller).
    """
    g = rng(cfg.seed, STREAM_REDRAW, step + 1, b, t, attempt)
    return round_to(g.standard_normal(cfg.d_inner), cfg.io_dtype)


# --------------------------------------------------------------------------------------------
# The surrounding block
# --------------------------------------------------------------------------------------------

@dataclass
class BlockWeights:
    W_in: np.ndarray  # [d_model, 2D] stored w_dtype
    conv_w: np.ndarray  # [D, W] float32
    conv_b: np.ndarray  # [D] float32
    W_out: np.ndarray  # [D, d_model] stored w_dtype
    layer: LayerWeights


def draw_block_weights(cfg: LayerConfig, d_model: int, d_conv: int, a_mode: str = "structured") -> BlockWeights:
    D = cfg.d_inner
    g = rng(cfg.seed, STREAM_BLOCK_WEIGHTS, d_model, d_conv)
    W_in = g.standard_normal((d_model, 2 * D)) * np.sqrt(1.0 / d_model)
    bound = 1.0 / np.sqrt(d_conv)
    conv_w = g.uniform(-bound, bound, size=(D, d_conv))
    conv_b = g.uniform(-bound, bound, size=D)
    W_out = g.standard_normal((D, d_model)) * np.sqrt(1.0 / D)
    return BlockWeights(
        W_in=round_to(W_in, cfg.w_dtype),
        conv_w=conv_w.astype(np.float32),
        conv_b=conv_b.astype(np.float32),
        W_out=round_to(W_out, cfg.w_dtype),
        layer=draw_weights(cfg, a_mode=a_mode),
    )


def draw_block_input(cfg: LayerConfig, d_model: int, batch_rows=None) -> np.ndarray:
    """u [B, L, d_model] in storage form; batch row b from stream (seed, 6, b)."""
    rows = range(cfg.batch) if batch_rows is None else batch_rows
    u = np.empty((len(rows), cfg.seqlen, d_model), dtype=np.uint16 if cfg.io_dtype == "bf16" else np.float32)
    for i, b in enumerate(rows):
        u[i] = round_to(rng(cfg.seed, STREAM_BLOCK_INPUT, b).standard_normal((cfg.seqlen, d_model)), cfg.io_dtype)
    return u


def draw_conv_state(cfg: LayerConfig, d_conv: int) -> np.ndarray:
    """A carried conv state [B, W-1, D] ~ N(0, 1) in storage form."""
    g = rng(cfg.seed, STREAM_CONV_STATE, d_conv)
    return round_to(g.standard_normal((cfg.batch, d_conv - 1, cfg.d_inner)), cfg.io_dtype)


def redraw_u_row(cfg: LayerConfig, d_model: int, b: int, t: int, attempt: int) -> np.ndarray:
    """A fresh block input row [d_model] for token (b, t), from stream (seed, 8, b, t, attempt)."""
    g = rng(cfg.seed, STREAM_BLOCK_REDRAW, b, t, attempt)
    return round_to(g.standard_normal(d_model), cfg.io_dtype)


@dataclass
class SsdInputs:
    X: np.ndarray       # [B, L, 1, H, P] bf16 bits
    B: np.ndarray       # [B, L, 1, N] bf16 bits
    C_mix: np.ndarray   # [B, L, N] bf16 bits
    gates: np.ndarray   # [B, L, 1] f32
    delta: np.ndarray   # [B, L, H] f32
    A: np.ndarray       # [H] f32
    D_skip: np.ndarray  # [H] f32
    S0: np.ndarray      # [B, H, P, N] f32


def draw_ssd_inputs(batch: int, seqlen: int, heads: int, head_dim: int, d_state: int, seed: int) -> SsdInputs:
    """The SSD-form workload's inputs (recipe in the module docstring), one stream per tensor."""
    g = lambda i: rng(seed, STREAM_SSD, i)
    B, L, H, P, N = batch, seqlen, heads, head_dim, d_state
    X = round_to(g(0).standard_normal((B, L, 1, H, P)), "bf16")
    Bm = round_to(g(1).standard_normal((B, L, 1, N)), "bf16")
    C = round_to(g(2).standard_normal((B, L, N)), "bf16")
    delta = np.exp(g(3).uniform(np.log(1e-3), np.log(1e-1), (B, L, H))).astype(np.float32)
    A = (-g(4).uniform(1.0, 16.0, H)).astype(np.float32)
    D_skip = g(5).standard_normal(H).astype(np.float32)
    S0 = (g(6).standard_normal((B, H, P, N)) * np.sqrt(0.1)).astype(np.float32)
    return SsdInputs(X, Bm, C, np.ones((B, L, 1), np.float32), delta, A, D_skip, S0)
