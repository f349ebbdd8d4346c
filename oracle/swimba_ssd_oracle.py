"""CPU fp64 oracle of Swimba's scan in the Mamba-2 SSD form -- TEST INFRASTRUCTURE ONLY.

Only the tests may import this module; no part of the library calls it. Like the layer oracle, it
is written with numpy in float64, step by step, and shares no code with any CUDA path.

Sources (by title and section):

[SW]  "Swimba: Switch Mamba Model Scales State Space Models": Spanish summary §2 "Arquitectura de
      Swimba" (built on Mamba-2 and its state space duality; every expert makes its own token-
      dependent streams B^(e), C^(e), X^(e); the transition A is shared by all experts and all
      time steps; the state input mixes sum_e pi_e B^(e)_t X^(e)_t, the readout uses
      (sum_e pi_e C^(e)_t)^T h_t; one state update per token); Dutch summary §2 "Belangrijkste
      Bijdragen", Stelling 1 (parameter mixing keeps the structure of one selective SSM, so SSD
      implementations carry over) and "Architectuur Implementatie" (the SSD computation and the
      chunked processing stay as in Mamba-2).
[MB]  "Mamba y las SSMs: el retorno del estado persistente", section "Mamba" (A-bar = exp(Delta A)).

Readings where the pages are silent (the row "Swimba on Mamba-2 SSD" of the design notes):

* heads h = 0..H-1 of P channels each; the shared transition is one negative scalar A_h per head
  (Mamba-2's scalar-times-identity A), so the decay a_t[h] = exp(Delta_t[h] A_h) is a scalar;
* per token t and active slot j (expert e_j, gate g_j; the gates sum to 1): streams X^(j)_t [H, P],
  B^(j)_t [N], C^(j)_t [N]; one step size Delta_t [H] per token (already mixed and positive);
* state S_t[h] in R^{P x N}:
      S_t[h] = a_t[h] S_{t-1}[h] + Delta_t[h] sum_j g_j X^(j)_t[h] (outer) B^(j)_t
      y_t[h, p] = sum_n C_mix,t[n] S_t[h, p, n] + D_skip[h] X_mix,t[h, p]
  with C_mix = sum_j g_j C^(j) and X_mix = sum_j g_j X^(j) (the skip term of the "SSMs" output
  equation of [MB], taken on the mixed input);
* the chunked (SSD) evaluation with chunk length Q gives the same y and final state: inside a
  chunk, with cum[i] = sum_{r <= i} log a_r (per head, from the chunk start),
      y[i] = sum_{s <= i} exp(cum[i] - cum[s]) Delta_s sum_j g_j,s (C_mix,i . B^(j)_s) X^(j)_s
             + exp(cum[i]) S_in C_mix,i + D X_mix,i
      S_out = exp(cum[Q-1]) S_in + sum_s exp(cum[Q-1] - cum[s]) Delta_s sum_j g_j,s X^(j)_s (outer) B^(j)_s

Pinned by ``tests/test_oracle_ssd_pins.py`` (a brute-force unrolled sum, reduction to the pinned
selective scan of the layer oracle, identical experts, superposition, chunked = sequential); none is
"parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = ["ssd_scan_sequential", "ssd_scan_chunked"]


def _mixed(g, V):
    """sum_j g[..., j] V[..., j, ...] over the slot axis (axis 1 of V)."""
    return np.einsum("tj,tj...->t...", g, V)


def ssd_scan_sequential(X, B, C, gates, delta, A, D_skip, S0=None):
    """The recurrence token by token (one sequence).

    X [L, k, H, P]; B, C [L, k, N]; gates [L, k]; delta [L, H] (> 0); A [H] (< 0); D_skip [H];
    S0 [H, P, N] or None (zeros). Returns (y [L, H, P], S_final [H, P, N]).
    """
    X = np.asarray(X, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    g = np.asarray(gates, dtype=np.float64)
    delta = np.asarray(delta, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    L, k, H, P = X.shape
    N = B.shape[2]
    S = np.zeros((H, P, N)) if S0 is None else np.array(S0, dtype=np.float64)
    y = np.empty((L, H, P))
    for t in range(L):
        a = np.exp(delta[t] * A)  # [H]
        inj = np.zeros((H, P, N))
        for j in range(k):
            inj += g[t, j] * X[t, j][:, :, None] * B[t, j][None, None, :]
        S = a[:, None, None] * S + delta[t][:, None, None] * inj
        c_mix = g[t] @ C[t]  # [N]
        x_mix = np.einsum("j,jhp->hp", g[t], X[t])
        y[t] = S @ c_mix + np.asarray(D_skip, dtype=np.float64)[:, None] * x_mix
    return y, S


def ssd_scan_chunked(X, B, C, gates, delta, A, D_skip, S0=None, Q=64):
    """The same scan in the chunked state-space-dual form: per chunk of Q tokens, the in-chunk
    outputs through the masked decay matrix exp(cum[i] - cum[s]) (s <= i), the carried state's
    contribution through exp(cum[i]), and the state passed to the next chunk. Arguments and result
    as ``ssd_scan_sequential``."""
    X = np.asarray(X, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    g = np.asarray(gates, dtype=np.float64)
    delta = np.asarray(delta, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    D_skip = np.asarray(D_skip, dtype=np.float64)
    L, k, H, P = X.shape
    N = B.shape[2]
    S = np.zeros((H, P, N)) if S0 is None else np.array(S0, dtype=np.float64)
    y = np.empty((L, H, P))
    for c0 in range(0, L, Q):
        c1 = min(c0 + Q, L)
        n = c1 - c0
        cum = np.cumsum(delta[c0:c1] * A[None, :], axis=0)  # [n, H]: sum of log a from the chunk start
        decay = np.exp(cum[:, None, :] - cum[None, :, :])  # [i, s, H]
        mask = np.tril(np.ones((n, n)))[:, :, None]
        Lmat = decay * mask  # exp(cum[i] - cum[s]) for s <= i, else 0
        c_mix = _mixed(g[c0:c1], C[c0:c1])  # [n, N]
        x_mix = _mixed(g[c0:c1], X[c0:c1])  # [n, H, P]
        y_c = np.zeros((n, H, P))
        for j in range(k):
            cb = c_mix @ B[c0:c1, j].T  # [i, s]: C_mix,i . B^(j)_s
            w = Lmat * (cb * (g[c0:c1, j])[None, :])[:, :, None] * delta[c0:c1][None, :, :]  # [i, s, H]
            y_c += np.einsum("ish,shp->ihp", w, X[c0:c1, j])
        # the carried state's contribution and the skip term
        y_c += np.exp(cum)[:, :, None] * np.einsum("hpn,in->ihp", S, c_mix)
        y_c += D_skip[None, :, None] * x_mix
        y[c0:c1] = y_c
        # state passed on
        tail = np.exp(cum[-1][None, :] - cum)  # [s, H]
        S_new = np.exp(cum[-1])[:, None, None] * S
        for j in range(k):
            coef = tail * delta[c0:c1] * g[c0:c1, j][:, None]  # [s, H]
            S_new += np.einsum("sh,shp,sn->hpn", coef, X[c0:c1, j], B[c0:c1, j])
        S = S_new
    return y, S
