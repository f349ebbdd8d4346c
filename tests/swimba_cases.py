"""Shared helpers of the parity tests: seeded cases, the oracle side, the CUDA side, tolerances.

Inputs come from the seeded generator (``synth``), with tokens near a router tie redrawn by the
oracle-side conditioning; both sides then see the same stored arrays. Expected values come from
the fp64 oracle only.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from oracle import swimba_oracle as O
from oracle.conditioning import condition_router_margin
from parameter_space_moe_swimba_b200 import synth

# Layer-output tolerance, max|err| <= TOL * (1 + |y|): fp32 activations 1e-4, bf16 activations 2e-2.
TOL_Y = {"f32": 1e-4, "bf16": 2e-2}


@dataclass
class Case:
    cfg: object
    w: synth.LayerWeights
    x: np.ndarray  # stored form
    z: np.ndarray
    h0: np.ndarray | None

    def x64(self, rows=None):
        x = self.x if rows is None else self.x[rows]
        return synth.widen(x, self.cfg.io_dtype)

    def z64(self, rows=None):
        z = self.z if rows is None else self.z[rows]
        return synth.widen(z, self.cfg.io_dtype)

    def weights64(self):
        w, c = self.w, self.cfg
        return {
            "W_r": w.W_r.astype(np.float64),
            "W_x": synth.widen(w.W_x, c.w_dtype),
            "W_dt": synth.widen(w.W_dt, c.w_dtype),
            "b_dt": w.b_dt.astype(np.float64),
            "A": w.A.astype(np.float64),
            "D_skip": w.D_skip.astype(np.float64),
        }


def make_case(cfg, a_mode="structured", with_h0=False, condition=True, margin=1e-3) -> Case:
    w = synth.draw_weights(cfg, a_mode=a_mode)
    x, z = synth.draw_activations(cfg)
    if condition and cfg.n_experts > 1:
        condition_router_margin(
            x, lambda s: synth.widen(s, cfg.io_dtype), w.W_r, cfg.top_k,
            lambda b, t, a: synth.redraw_x_row(cfg, b, t, a), margin=margin,
        )
    h0 = synth.draw_h0(cfg) if with_h0 else None
    return Case(cfg, w, x, z, h0)


def oracle_layer(case: Case, rows=None, channels=None) -> dict:
    h0 = None if case.h0 is None else (case.h0 if rows is None else case.h0[rows]).astype(np.float64)
    return O.layer_forward(case.x64(rows), case.z64(rows), case.weights64(), case.cfg.top_k, h0=h0, channels=channels)


def oracle_route_proj(case: Case, rows, chunk=8192) -> dict:
    """The oracle's routing and mixed projections (idx, gates, dt_mix, B_mix, C_mix, delta) for
    every token of the given batch rows, all channels. Tokens are processed in chunks so that the
    fp64 temporaries stay bounded; each token's result depends only on that token."""
    cfg = case.cfg
    W = case.weights64()
    R, N = cfg.dt_rank, cfg.d_state
    parts = {k: [] for k in ("idx", "gates", "dt_mix", "B_mix", "C_mix")}
    for b in rows:
        xs = case.x[b]
        for t0 in range(0, xs.shape[0], chunk):
            x64 = synth.widen(xs[t0:t0 + chunk], cfg.io_dtype)
            idx, gates, _ = O.route(x64, W["W_r"], cfg.top_k)
            pr = O.expert_projections(x64, idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N)
            parts["idx"].append(idx)
            parts["gates"].append(gates)
            for k in ("dt_mix", "B_mix", "C_mix"):
                parts[k].append(pr[k])
    L = case.x.shape[1]
    out = {k: np.concatenate(v).reshape(len(rows), L, *v[0].shape[1:]) for k, v in parts.items()}
    out["delta"] = O.softplus(out["dt_mix"])
    return out


def scaled_err(got, ref):
    """max |got - ref| / (1 + |ref|)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref) / (1.0 + np.abs(ref)))) if ref.size else 0.0


def rel_rms_err(got, ref):
    """max |got - ref| / (rms(ref) + |ref|): the error relative to the field's own scale."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref))) + 1e-300
    return float(np.max(np.abs(got - ref) / (rms + np.abs(ref))))
