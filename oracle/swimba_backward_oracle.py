"""CPU fp64 oracle of the Swimba layer's BACKWARD pass -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module; the library's compute path never calls it and shares no code with it.

Source of the forward it differentiates: the layer definition of ``oracle.swimba_oracle`` ("Swimba:
Switch Mamba Model Scales State Space Models", §2 "Arquitectura de Swimba" / "Generación de
Parámetros" / "Mezcla en el Espacio de Parámetros"; "Mamba y las SSMs: el retorno del estado
persistente", "Mamba"). The pages train Swimba-14B ("Swimba", Dutch summary "Resultaten") but give
no training details, so the backward pass is the exact gradient of that forward, nothing more:
reverse-mode differentiation written out step by step (the chain rule through each forward
statement, in reverse order), in float64, with no blocking or fusion.

Forward, per sequence b, channel d, state n (Euler injection, the layer's definition):
    A_t[d, n] = Σ_j g_t,j A^{e_t,j}[d, n];   a_t = exp(Δ_t[d] A_t[d, n])
    h_t = a_t h_{t-1} + Δ_t[d] B_t[n] x_t[d]                   (h_{-1} = h0)
    y_t[d] = Σ_n C_t[n] h_t[d, n] + D[d] x_t[d];   out_t[d] = y_t[d] SiLU(z_t[d])
Backward, given G_t[d] = ∂L/∂out_t[d]:
    ∂L/∂y_t = G_t SiLU(z_t);   ∂L/∂z_t = G_t y_t SiLU'(z_t),  SiLU'(z) = σ(z)(1 + z(1 − σ(z)))
    λ_t = ∂L/∂h_t = C_t[n] ∂L/∂y_t[d] + a_{t+1} λ_{t+1}         (reverse in t; λ_L = 0)
    ∂L/∂C_t[n] = Σ_d ∂L/∂y_t[d] h_t[d, n];   ∂L/∂D[d] = Σ_t ∂L/∂y_t[d] x_t[d]
    ∂L/∂x_t[d] = D[d] ∂L/∂y_t[d] + Σ_n λ_t Δ_t B_t[n]
    ∂L/∂B_t[n] = Σ_d λ_t Δ_t x_t
    ∂L/∂Δ_t[d] = Σ_n λ_t (A_t a_t h_{t-1} + B_t x_t)
    ∂L/∂A_t[d, n] = λ_t Δ_t a_t h_{t-1}  ->  ∂L/∂A^e += g_t,j ∂L/∂A_t (e = e_t,j),
                                              ∂L/∂g_t,j += Σ_{d,n} ∂L/∂A_t A^{e_t,j}
    ∂L/∂h0 = a_0 λ_0
The projection and the router are differentiated the same way (their functions below); the
top-k choice itself is piecewise constant, so the indices carry no gradient.

Pins: ``tests/test_oracle_backward_pins.py`` checks every gradient against central finite
differences of the pinned forward oracle on small inputs, plus closed forms.
"""
from __future__ import annotations

import numpy as np

from oracle import swimba_oracle as O

__all__ = [
    "sigmoid",
    "silu_grad",
    "softplus_backward",
    "scan_backward",
    "projection_backward",
    "route_backward",
    "layer_backward",
]


def sigmoid(v):
    """σ(v) = 1 / (1 + e^{-v}), written as e^{v} / (1 + e^{v}) for v < 0 so that neither end
    loses its relative accuracy."""
    v = np.asarray(v, dtype=np.float64)
    e = np.exp(-np.abs(v))
    return np.where(v >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def silu_grad(z):
    """d SiLU(z) / dz = σ(z) (1 + z (1 − σ(z)))."""
    s = sigmoid(z)
    return s * (1.0 + np.asarray(z, dtype=np.float64) * (1.0 - s))


def softplus_backward(dt_mix, g_delta):
    """Δ = softplus(dt_mix) -> ∂L/∂dt_mix = ∂L/∂Δ · σ(dt_mix)."""
    return np.asarray(g_delta, dtype=np.float64) * sigmoid(dt_mix)


def scan_backward(x, z, delta, B_mix, C_mix, idx, gates, A, D_skip, g_out, h0=None):
    """Gradients of the selective scan (the library's scan: it takes Δ, not dt_mix).

    x, z, delta, g_out [B, L, D]; B_mix, C_mix [B, L, N]; idx, gates [B, L, k]; A [E, D, N];
    D_skip [D]; h0 [B, D, N] or None (zeros). Returns a dict with dx, dz, ddelta [B, L, D],
    dB, dC [B, L, N], dgates [B, L, k], dA [E, D, N], dD [D], dh0 [B, D, N], and the forward's
    out [B, L, D] and h_final [B, D, N].
    """
    f = lambda v: np.asarray(v, dtype=np.float64)
    x, z, delta, B_mix, C_mix, gates, A, D_skip, g_out = map(f, (x, z, delta, B_mix, C_mix, gates, A, D_skip, g_out))
    Bsz, L, D = x.shape
    N = A.shape[2]
    k = idx.shape[2]
    # forward, keeping every state h_t (h_prev[t] = h_{t-1}) and every transition
    h = np.zeros((Bsz, D, N)) if h0 is None else f(h0).copy()
    h_prev = np.empty((L, Bsz, D, N))
    hs = np.empty((L, Bsz, D, N))
    A_ts = np.empty((L, Bsz, D, N))
    a_ts = np.empty((L, Bsz, D, N))
    y = np.empty((Bsz, L, D))
    for t in range(L):
        A_t = np.zeros((Bsz, D, N))
        for j in range(k):
            A_t += gates[:, t, j, None, None] * A[idx[:, t, j]]
        a_t = np.exp(delta[:, t, :, None] * A_t)
        h_prev[t] = h
        h = a_t * h + delta[:, t, :, None] * B_mix[:, t, None, :] * x[:, t, :, None]
        hs[t], A_ts[t], a_ts[t] = h, A_t, a_t
        y[:, t, :] = np.einsum("bn,bdn->bd", C_mix[:, t, :], h) + D_skip[None, :] * x[:, t, :]
    out = y * O.silu(z)
    # backward through the gate
    dy = g_out * O.silu(z)
    dz = g_out * y * silu_grad(z)
    dx = np.zeros_like(x)
    ddelta = np.zeros_like(x)
    dB = np.zeros_like(B_mix)
    dC = np.zeros_like(C_mix)
    dg = np.zeros_like(gates)
    dA = np.zeros_like(A)
    dD = np.einsum("bld,bld->d", dy, x)
    carry = np.zeros((Bsz, D, N))  # a_{t+1} λ_{t+1}
    for t in range(L - 1, -1, -1):
        lam = carry + C_mix[:, t, None, :] * dy[:, t, :, None]  # λ_t
        dC[:, t, :] = np.einsum("bd,bdn->bn", dy[:, t, :], hs[t])
        d_t = delta[:, t, :]
        dx[:, t, :] = D_skip[None, :] * dy[:, t, :] + np.einsum("bdn,bn->bd", lam, B_mix[:, t, :]) * d_t
        dB[:, t, :] = np.einsum("bdn,bd->bn", lam, d_t * x[:, t, :])
        ddelta[:, t, :] = np.einsum("bdn,bdn->bd", lam, A_ts[t] * a_ts[t] * h_prev[t]) + \
            np.einsum("bdn,bn->bd", lam, B_mix[:, t, :]) * x[:, t, :]
        dA_t = lam * d_t[:, :, None] * a_ts[t] * h_prev[t]
        for j in range(k):
            e = idx[:, t, j]
            for b in range(Bsz):
                dA[e[b]] += gates[b, t, j] * dA_t[b]
                dg[b, t, j] += np.sum(dA_t[b] * A[e[b]])
        carry = a_ts[t] * lam
    return {"dx": dx, "dz": dz, "ddelta": ddelta, "dB": dB, "dC": dC, "dgates": dg, "dA": dA, "dD": dD,
            "dh0": carry, "out": out, "h_final": h}


def projection_backward(x, idx, gates, W_x, W_dt, b_dt, dt_rank, d_state, g_dtmix, g_B, g_C):
    """Gradients of ``expert_projections`` (the mixed streams dt_mix, B_mix, C_mix).

    x [T, D]; idx, gates [T, k]; W_x [E, D, R+2N]; W_dt [E, R, D]; b_dt [E, D];
    g_dtmix [T, D], g_B, g_C [T, N]. Returns dx [T, D], dgates [T, k], dW_x, dW_dt, db_dt.
    """
    f = lambda v: np.asarray(v, dtype=np.float64)
    x, gates, W_x, W_dt, b_dt, g_dtmix, g_B, g_C = map(f, (x, gates, W_x, W_dt, b_dt, g_dtmix, g_B, g_C))
    T, D = x.shape
    k = idx.shape[1]
    R, N = dt_rank, d_state
    fw = O.expert_projections(x, idx, gates, W_x, W_dt, b_dt, R, N)
    xdbl, dt_j = fw["xdbl"], fw["dt_j"]
    dx = np.zeros_like(x)
    dg = np.zeros_like(gates)
    dW_x = np.zeros_like(W_x)
    dW_dt = np.zeros_like(W_dt)
    db = np.zeros_like(b_dt)
    for j in range(k):
        # dt_mix = Σ_j g_j dt_j, B_mix = Σ_j g_j B_j, C_mix = Σ_j g_j C_j
        dg[:, j] = np.sum(g_dtmix * dt_j[:, j], axis=1) + np.sum(g_B * xdbl[:, j, R:R + N], axis=1) + \
            np.sum(g_C * xdbl[:, j, R + N:], axis=1)
        d_dtj = gates[:, j, None] * g_dtmix  # [T, D]
        dv = np.concatenate([np.zeros((T, R)), gates[:, j, None] * g_B, gates[:, j, None] * g_C], axis=1)
        for e in range(W_x.shape[0]):
            rows = np.nonzero(idx[:, j] == e)[0]
            if rows.size == 0:
                continue
            # dt_j = dt_low W_dt^e + b_dt^e
            db[e] += d_dtj[rows].sum(axis=0)
            dW_dt[e] += xdbl[rows, j, :R].T @ d_dtj[rows]
            dv_e = dv[rows].copy()
            dv_e[:, :R] = d_dtj[rows] @ W_dt[e].T
            # v = x W_x^e
            dW_x[e] += x[rows].T @ dv_e
            dx[rows] += dv_e @ W_x[e].T
    return {"dx": dx, "dgates": dg, "dW_x": dW_x, "dW_dt": dW_dt, "db_dt": db}


def route_backward(x, W_r, idx, g_gates):
    """Gradients of the router's gates (softmax over the k selected logits of logits = x W_r)
    with the selection held fixed. x [T, D]; W_r [D, E]; idx, g_gates [T, k].
    Returns dx [T, D], dW_r [D, E]."""
    x = np.asarray(x, dtype=np.float64)
    W_r = np.asarray(W_r, dtype=np.float64)
    g_gates = np.asarray(g_gates, dtype=np.float64)
    logits = x @ W_r
    sel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    w = np.exp(sel - sel.max(axis=1, keepdims=True))
    gates = w / w.sum(axis=1, keepdims=True)
    d_sel = gates * (g_gates - np.sum(gates * g_gates, axis=1, keepdims=True))
    d_logits = np.zeros_like(logits)
    np.put_along_axis(d_logits, idx.astype(np.int64), d_sel, axis=1)
    return {"dx": d_logits @ W_r.T, "dW_r": x.T @ d_logits}


def layer_backward(x, z, W, k, g_out, h0=None):
    """Gradients of the whole layer (route -> projections -> scan) for ∂L/∂out = g_out.

    x, z, g_out [B, L, D]; W as ``layer_forward`` (W_r, W_x, W_dt, b_dt, A, D_skip). Returns a dict
    with dx, dz [B, L, D], dW_r, dW_x, dW_dt, db_dt, dA, dD, dh0, and the intermediate gradients
    ddelta, dB, dC, dgates of the scan's inputs."""
    x = np.asarray(x, dtype=np.float64)
    Bsz, L, D = x.shape
    T = Bsz * L
    R = W["W_dt"].shape[1]
    N = W["A"].shape[2]
    xt = x.reshape(T, D)
    idx, gates, _ = O.route(xt, W["W_r"], k)
    pr = O.expert_projections(xt, idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N)
    delta = O.softplus(pr["dt_mix"])
    sh = lambda a: a.reshape(Bsz, L, *a.shape[1:])
    sb = scan_backward(x, z, sh(delta), sh(pr["B_mix"]), sh(pr["C_mix"]), sh(idx), sh(gates), W["A"],
                       W["D_skip"], g_out, h0)
    g_dtmix = softplus_backward(pr["dt_mix"], sb["ddelta"].reshape(T, D))
    pb = projection_backward(xt, idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N, g_dtmix,
                             sb["dB"].reshape(T, N), sb["dC"].reshape(T, N))
    g_gates = sb["dgates"].reshape(T, k) + pb["dgates"]
    rb = route_backward(xt, W["W_r"], idx, g_gates)
    dx = sb["dx"] + sh(pb["dx"]) + sh(rb["dx"])
    return {"dx": dx, "dz": sb["dz"], "dW_r": rb["dW_r"], "dW_x": pb["dW_x"], "dW_dt": pb["dW_dt"],
            "db_dt": pb["db_dt"], "dA": sb["dA"], "dD": sb["dD"], "dh0": sb["dh0"], "ddelta": sb["ddelta"],
            "dB": sb["dB"], "dC": sb["dC"], "dgates": sb["dgates"], "out": sb["out"]}
