"""CPU fp64 oracle of the Swimba (Switch Mamba) layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module. The library's compute path never calls it, and it shares no code with that path: it
is written with numpy in float64, step by step in the order the sources give, with no blocking,
fusion or reordering.

Sources (cited by title and section; the pages give the method in prose only):

[SW]  "Swimba: Switch Mamba Model Scales State Space Models" (arXiv 2603.06938), summaries at
      gist.science in Spanish (technical summary §2 "Metodología", "Arquitectura de Swimba"),
      Dutch ("Methodologie", "Kernmechanisme van Swimba") and French ("2. Méthodologie",
      "Architecture de Swimba"; "Fondements Théoriques", Théorèmes 1-3).
[MB]  "Mamba y las SSMs: el retorno del estado persistente" (maquinaoraculo.com), sections
      "SSMs – Modelos de espacios de estados" (h_t = A h_{t-1} + B x_t, y_t = C h_t + D x_t),
      "Mamba" (selective SSM, Ā = exp(Δ_t A), Figura 2) and "Estado interno puramente lineal".

What [SW] fixes: a router gives per-token mixing weights π_t over the active experts (top-1 or
top-k); every expert has its own linear projections that produce token-dependent parameter
streams; the streams are mixed with π_t in parameter space -- injection Σ_e π_{t,e} B^(e)_t X_t,
readout (Σ_e π_{t,e} C^(e)_t)ᵀ h_t -- and ONE recurrence runs on a single state h_t.

What this library's layer definition adds where the pages are silent (each reading is listed with
its reason in the design notes of the repository):

* logits_t = x_t · W_r; idx_t = the k largest, in descending order, ties to the lower index;
  gates π_t = softmax over the k selected logits (so they sum to 1; top-1 gives exactly 1).
* expert e maps x_t to [dt_low (R) | B (N) | C (N)] = x_t · W_x^e, and dt^e = dt_low · W_dt^e
  + b_dt^e; the mixed streams are dt_mix = Σ_j π_j dt^{e_j}, B_mix = Σ_j π_j B^{e_j},
  C_mix = Σ_j π_j C^{e_j} (X_t is the shared input x_t).
* Δ_t = softplus(dt_mix); the transition A_t[d, n] = Σ_j π_j A^{e_j}[d, n] (a convex mix of
  per-expert diagonal A; all experts equal gives the shared A of [SW]); ā = exp(Δ_t A_t)
  as in [MB] "Mamba"; injection Δ_t · B_mix · x_t (the Euler form, not the ZOH B̄ of [MB]).
* h_t = ā ⊙ h_{t-1} + Δ_t B_mix x_t from h_{-1} = h0 (zeros when absent);
  y_t = Σ_n C_mix[n] h_t[·, n] + D_skip ⊙ x_t ([MB] "SSMs" output equation with its D term);
  out_t = y_t ⊙ SiLU(z_t).

The surrounding block (the steps on either side of the layer), from [MB] "Mamba" (Figura 3: a
linear projection that makes the two branches, a convolution and SiLU on the SSM branch, the
gated SSM, a linear output projection), [MB] "Estado interno puramente lineal" (output projection
followed by a residual connection) and [SW] Dutch summary §2 "Architectuur Implementatie" (the
in-projection of the base block becomes the module that makes the expert-specific parameters; the
rest of the block is unchanged). Readings where the pages are silent:

* [x_pre | z] = u · W_in with W_in [d_model, 2D]; x = SiLU(causal depthwise conv of x_pre, width W,
  per-channel taps and bias); the Swimba layer runs on (x, z); o = out · W_out + u, W_out [D, d_model].
* the convolution looks back W-1 tokens of the same sequence; before the first token it reads the
  carried conv state [B, W-1, D] (zeros when absent), and the last W-1 inputs are the new state.
* with bf16 activations, x_pre, z, x, the layer output and o are stored in bf16 (round to nearest
  even), each once, where the block stores them.

Every function below is pinned by the CPU tests (closed forms, brute force, invariants, special
cases that reduce to a dense selective scan or to a library convolution); none is "parity
unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "softplus",
    "silu",
    "router_logits",
    "route",
    "expert_projections",
    "selective_scan",
    "layer_forward",
    "decode_step",
    "scan_summary",
    "chain_summaries",
    "separate_ssm_moe",
    "round_bf16",
    "causal_conv1d",
    "block_branches",
    "block_forward",
    "block_decode_step",
]


def softplus(v):
    """softplus(v) = log(1 + e^v), written in the overflow-free form max(v,0) + log1p(e^{-|v|})."""
    v = np.asarray(v, dtype=np.float64)
    return np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))


def silu(z):
    """SiLU(z) = z · σ(z) = z / (1 + e^{-z}) (the gate nonlinearity of the Mamba block, [MB])."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def router_logits(x, W_r):
    """Router scores: logits[..., e] = Σ_d x[..., d] W_r[d, e]  ([SW]: the router computes π_t)."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(W_r, dtype=np.float64)


def route(x, W_r, k):
    """Top-k routing ([SW] "Routing": weights π_t for the active experts, top-1 or top-k).

    Returns (idx [..., k] int32, gates [..., k] float64, logits [..., E]). idx lists the k largest
    logits in descending order; equal logits keep the lower expert index first. gates are the
    softmax of the selected logits, so each row sums to 1.
    """
    logits = router_logits(x, W_r)
    E = logits.shape[-1]
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    order = np.argsort(-logits, axis=-1, kind="stable")[..., :k]
    sel = np.take_along_axis(logits, order, axis=-1)
    w = np.exp(sel - sel[..., :1])
    gates = w / w.sum(axis=-1, keepdims=True)
    return order.astype(np.int32), gates, logits


def expert_projections(x, idx, gates, W_x, W_dt, b_dt, dt_rank, d_state):
    """Per-expert parameter streams mixed with the gates ([SW] "Generación de Parámetros" and
    "Mezcla en el Espacio de Parámetros").

    x [T, D]; idx, gates [T, k]; W_x [E, D, R+2N]; W_dt [E, R, D]; b_dt [E, D] (all fp64 values).
    For slot j of token t with expert e = idx[t, j]:
        v = x_t · W_x^e = [dt_low | B^j | C^j];   dt^j = dt_low · W_dt^e + b_dt^e.
    Returns dict with xdbl [T, k, R+2N], dt_j [T, k, D], dt_mix [T, D], B_mix [T, N], C_mix [T, N].
    """
    x = np.asarray(x, dtype=np.float64)
    T, D = x.shape
    k = idx.shape[1]
    E = W_x.shape[0]
    R, N = dt_rank, d_state
    xdbl = np.zeros((T, k, R + 2 * N))
    dt_j = np.zeros((T, k, D))
    for j in range(k):
        for e in range(E):
            rows = np.nonzero(idx[:, j] == e)[0]
            if rows.size == 0:
                continue
            v = x[rows] @ W_x[e]
            xdbl[rows, j] = v
            dt_j[rows, j] = v[:, :R] @ W_dt[e] + b_dt[e]
    g = np.asarray(gates, dtype=np.float64)
    dt_mix = np.einsum("tj,tjd->td", g, dt_j)
    B_mix = np.einsum("tj,tjn->tn", g, xdbl[:, :, R:R + N])
    C_mix = np.einsum("tj,tjn->tn", g, xdbl[:, :, R + N:R + 2 * N])
    return {"xdbl": xdbl, "dt_j": dt_j, "dt_mix": dt_mix, "B_mix": B_mix, "C_mix": C_mix}


def selective_scan(x, z, dt_mix, B_mix, C_mix, idx, gates, A, D_skip, h0=None, channels=None, injection="euler"):
    """The single recurrence over the mixed parameters ([SW] one state trajectory; [MB] "Mamba").

    ``injection`` picks the input discretisation: "euler" (the layer's definition, Δ B x) or "zoh",
    the zero-order hold of [MB] "Mamba" (B̄ = A⁻¹(exp(ΔA) − I) B; with the diagonal mixed transition
    it is elementwise, (exp(Δ A_t) − 1) / A_t · B_mix · x, written with expm1).

    x, z, dt_mix [B, L, D]; B_mix, C_mix [B, L, N]; idx, gates [B, L, k]; A [E, D, N];
    D_skip [D]; h0 [B, D, N] or None (zeros). ``channels`` optionally restricts the work to a list
    of channel indices d; the recurrence of every (b, d, n) is independent, so the restricted
    result equals the corresponding columns of the full one.

    For t = 0 .. L-1 in order:
        Δ = softplus(dt_mix[:, t]);  A_t = Σ_j gates_j A^{idx_j};  ā = exp(Δ A_t)
        h = ā ⊙ h + Δ · B_mix[t] · x[t]
        y[t] = Σ_n C_mix[t, n] h[·, n] + D_skip ⊙ x[t];   out[t] = y[t] ⊙ SiLU(z[t]).
    Returns (y, out, h_final, delta) with y, out, delta [B, L, D'] and h_final [B, D', N].
    """
    x = np.asarray(x, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    dt_mix = np.asarray(dt_mix, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    D_skip = np.asarray(D_skip, dtype=np.float64)
    if channels is not None:
        ch = np.asarray(channels)
        x, z, dt_mix = x[:, :, ch], z[:, :, ch], dt_mix[:, :, ch]
        A, D_skip = A[:, ch, :], D_skip[ch]
        if h0 is not None:
            h0 = np.asarray(h0)[:, ch, :]
    Bsz, L, D = x.shape
    N = A.shape[2]
    h = np.zeros((Bsz, D, N)) if h0 is None else np.array(h0, dtype=np.float64)
    y = np.empty((Bsz, L, D))
    delta = softplus(dt_mix)
    g = np.asarray(gates, dtype=np.float64)
    for t in range(L):
        d_t = delta[:, t, :]  # [B, D]
        A_t = np.zeros((Bsz, D, N))
        for j in range(idx.shape[2]):
            A_t += g[:, t, j, None, None] * A[idx[:, t, j]]
        a_bar = np.exp(d_t[:, :, None] * A_t)
        if injection == "zoh":
            u = np.expm1(d_t[:, :, None] * A_t) / A_t * B_mix[:, t, None, :] * x[:, t, :, None]
        elif injection == "euler":
            u = d_t[:, :, None] * B_mix[:, t, None, :] * x[:, t, :, None]
        else:
            raise ValueError("injection must be 'euler' or 'zoh'")
        h = a_bar * h + u
        y[:, t, :] = np.einsum("bn,bdn->bd", C_mix[:, t, :], h) + D_skip[None, :] * x[:, t, :]
    out = y * silu(z)
    return y, out, h, delta


def layer_forward(x, z, W, k, h0=None, channels=None, injection="euler"):
    """The Swimba layer: route -> per-expert projections mixed by the gates -> one scan.

    x, z [B, L, D] fp64 values; W: a mapping with fp64 values W_r [D,E], W_x [E,D,R+2N],
    W_dt [E,R,D], b_dt [E,D], A [E,D,N], D_skip [D]; h0 [B,D,N] or None. Returns a dict with every
    intermediate: logits, idx, gates, xdbl, dt_mix, B_mix, C_mix, delta, y, out, h_final.
    ``channels`` restricts the scan (not the routing or the projections) to some channels.
    """
    x = np.asarray(x, dtype=np.float64)
    Bsz, L, D = x.shape
    E = W["W_r"].shape[1]
    N = W["A"].shape[2]
    R = W["W_dt"].shape[1]
    idx, gates, logits = route(x.reshape(-1, D), W["W_r"], k)
    proj = expert_projections(x.reshape(-1, D), idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N)
    shp = lambda a: a.reshape(Bsz, L, *a.shape[1:])
    idx_b, gates_b = shp(idx), shp(gates)
    dt_mix, B_mix, C_mix = shp(proj["dt_mix"]), shp(proj["B_mix"]), shp(proj["C_mix"])
    y, out, h_final, delta = selective_scan(
        x, z, dt_mix, B_mix, C_mix, idx_b, gates_b, W["A"], W["D_skip"], h0=h0, channels=channels,
        injection=injection,
    )
    assert E == W["W_x"].shape[0]
    return {
        "logits": shp(logits),
        "idx": idx_b,
        "gates": gates_b,
        "xdbl": shp(proj["xdbl"]),
        "dt_mix": dt_mix,
        "B_mix": B_mix,
        "C_mix": C_mix,
        "delta": delta,
        "y": y,
        "out": out,
        "h_final": h_final,
    }


def decode_step(h, x_t, z_t, W, k, channels=None):
    """One recurrent decode step: the layer with L = 1 continuing from the cached state h [B,D,N].

    x_t, z_t [B, 1, D]. Returns (out [B, 1, D'], h_new [B, D', N], full intermediates dict).
    """
    r = layer_forward(x_t, z_t, W, k, h0=h, channels=channels)
    return r["out"], r["h_final"], r


def scan_summary(x, dt_mix, B_mix, idx, gates, A):
    """What one piece of a sequence hands to the next ([MB] "Estado interno puramente lineal": the
    state is linear, so the recurrence can be split and recombined).

    Over the given tokens (x, dt_mix [B, L, D]; B_mix [B, L, N]; idx, gates [B, L, k]; A [E, D, N])
    the state after the last token is linear in the state before the first one:
        h_end(h_in) = exp(Σ_t Δ_t A_t) ⊙ h_in + h_end(0).
    Returns (h_zero [B, D, N], log_decay [B, D, N]): the end state of the recurrence started from
    zero, and Σ_t Δ_t A_t (the natural log of the product of the per-token decays ā_t).
    """
    x = np.asarray(x, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bsz, L, D = x.shape
    N = A.shape[2]
    delta = softplus(dt_mix)
    g = np.asarray(gates, dtype=np.float64)
    h = np.zeros((Bsz, D, N))
    log_decay = np.zeros((Bsz, D, N))
    for t in range(L):
        d_t = delta[:, t, :]
        A_t = np.zeros((Bsz, D, N))
        for j in range(idx.shape[2]):
            A_t += g[:, t, j, None, None] * A[idx[:, t, j]]
        log_decay += d_t[:, :, None] * A_t
        h = np.exp(d_t[:, :, None] * A_t) * h + d_t[:, :, None] * B_mix[:, t, None, :] * x[:, t, :, None]
    return h, log_decay


def chain_summaries(h_zero, log_decay, h0=None):
    """Start state of every piece of a sequence cut into P consecutive pieces, from the pieces'
    summaries (``scan_summary``) stacked on a leading axis [P, B, D, N]:
        H_0 = h0 (zeros when absent);   H_{p+1} = exp(log_decay_p) ⊙ H_p + h_zero_p.
    Returns H [P + 1, B, D, N]; H[P] is the state after the whole sequence."""
    h_zero = np.asarray(h_zero, dtype=np.float64)
    log_decay = np.asarray(log_decay, dtype=np.float64)
    P = h_zero.shape[0]
    H = np.zeros((P + 1,) + h_zero.shape[1:])
    if h0 is not None:
        H[0] = np.asarray(h0, dtype=np.float64)
    for p in range(P):
        H[p + 1] = np.exp(log_decay[p]) * H[p] + h_zero[p]
    return H


def separate_ssm_moe(x, z, dt_j, B_j, C_j, idx, gates, A, D_skip, h0=None):
    """The "MoE of separate SSMs" that [SW] sets against Swimba (Spanish summary §2 "Distinción de
    Diseños", Dutch "Methodologie", French "Distinction des deux designs MoE-SSM"): every expert
    keeps its own state trajectory and runs its own recurrent update, so the recurrence work grows
    with the experts; Teorema 2 is the claim that Swimba's single mixed recurrence avoids it.

    Reading (the pages give no equations for it): expert e has its own state h^(e) [B, D, N]; at
    token t the k active experts e_j = idx[t, j] advance their own states with their own, unmixed
    streams and their own transition,
        Δ^j = softplus(dt_j[t, j]);  h^(e_j) = exp(Δ^j A^{e_j}) ⊙ h^(e_j) + Δ^j B_j[t, j] x_t,
    the states of the experts not chosen at t are left as they are, and the outputs of the active
    experts are mixed with the gates:
        y_t = Σ_j g_j C_j[t, j] · h^(e_j) + D_skip ⊙ x_t;   out_t = y_t ⊙ SiLU(z_t).

    x, z [B, L, D]; dt_j [B, L, k, D]; B_j, C_j [B, L, k, N]; idx, gates [B, L, k]; A [E, D, N];
    D_skip [D]; h0 [E, B, D, N] or None (zeros). Returns (y, out, h [E, B, D, N])."""
    x = np.asarray(x, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    E = A.shape[0]
    Bsz, L, D = x.shape
    N = A.shape[2]
    k = idx.shape[2]
    h = np.zeros((E, Bsz, D, N)) if h0 is None else np.array(h0, dtype=np.float64)
    g = np.asarray(gates, dtype=np.float64)
    delta = softplus(dt_j)
    y = np.empty((Bsz, L, D))
    for t in range(L):
        y_t = D_skip[None, :] * x[:, t, :]
        for b in range(Bsz):
            for j in range(k):
                e = idx[b, t, j]
                d_bj = delta[b, t, j]  # [D]
                h[e, b] = np.exp(d_bj[:, None] * A[e]) * h[e, b] + d_bj[:, None] * B_j[b, t, j][None, :] * x[b, t, :, None]
                y_t[b] += g[b, t, j] * (h[e, b] @ C_j[b, t, j])
        y[:, t, :] = y_t
    out = y * silu(z)
    return y, out, h


# ------------------------------------------------------------------------------------------------
# The surrounding block
# ------------------------------------------------------------------------------------------------

def round_bf16(v):
    """Nearest bfloat16 value (8 significant bits, ties to even) of fp64 values in bf16's normal
    range or zero: with v = m 2^e, 0.5 <= |m| < 1, the result is rint(m 2^8) 2^(e-8)."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def causal_conv1d(x_pre, w, b, state=None):
    """Depthwise causal convolution over time, then SiLU ([MB] "Mamba", Figura 3: the convolution
    and the nonlinearity on the SSM branch of the block).

    x_pre [B, L, D]; w [D, W] taps; b [D] bias; state [B, W-1, D] = the W-1 inputs before the
    first token, oldest first (zeros when None). With p = [state; x_pre] along time:
        c[t, d] = b[d] + sum_{i=0}^{W-1} w[d, i] p[t + i, d]      (tap W-1 weighs the current token)
        x[t, d] = SiLU(c[t, d]);   state_out = the last W-1 rows of p.
    Returns (c, x, state_out).
    """
    x_pre = np.asarray(x_pre, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    Bsz, L, D = x_pre.shape
    W = w.shape[1]
    if state is None:
        state = np.zeros((Bsz, W - 1, D))
    p = np.concatenate([np.asarray(state, dtype=np.float64), x_pre], axis=1)
    c = np.empty((Bsz, L, D))
    for t in range(L):
        acc = np.array(b, dtype=np.float64)[None, :].repeat(Bsz, axis=0)
        for i in range(W):
            acc = acc + w[None, :, i] * p[:, t + i, :]
        c[:, t, :] = acc
    return c, silu(c), p[:, L:, :].copy()


def _store_fn(io):
    return round_bf16 if io == "bf16" else (lambda a: np.asarray(a, dtype=np.float64))


def block_branches(u, BW, conv_state=None, io="f32"):
    """The block's first two steps: the in-projection [x_pre | z] = u W_in and the convolution
    x = SiLU(conv(x_pre)), each stored in the io dtype. Returns (x_pre, z, x, conv_state_out)."""
    store = _store_fn(io)
    D = BW["conv_w"].shape[0]
    xz = np.asarray(u, dtype=np.float64) @ np.asarray(BW["W_in"], dtype=np.float64)
    x_pre, z = store(xz[..., :D]), store(xz[..., D:])
    _, x, conv_out = causal_conv1d(x_pre, BW["conv_w"], BW["conv_b"], conv_state)
    return x_pre, z, store(x), conv_out


def block_forward(u, BW, k, h0=None, conv_state=None, io="f32"):
    """The Swimba block: in-projection, convolution + SiLU, the Swimba layer, out-projection and
    residual (sources in the module header).

    u [B, L, d_model]; BW: W_in [d_model, 2D], conv_w [D, W], conv_b [D], W_out [D, d_model] and
    the layer's weights (W_r, W_x, W_dt, b_dt, A, D_skip); h0 [B, D, N] or None; conv_state
    [B, W-1, D] or None; io = "bf16" rounds x_pre, z, x, the layer output and o to bf16 where the
    block stores them. Returns a dict: x_pre, z, x, the layer's intermediates (layer), o,
    h_final, conv_state.
    """
    store = _store_fn(io)
    u = np.asarray(u, dtype=np.float64)
    x_pre, z, x, conv_out = block_branches(u, BW, conv_state, io)
    layer = layer_forward(x, z, BW, k, h0=h0)
    y_g = store(layer["out"])
    o = store(y_g @ np.asarray(BW["W_out"], dtype=np.float64) + u)
    return {"x_pre": x_pre, "z": z, "x": x, "layer": layer, "o": o, "h_final": layer["h_final"],
            "conv_state": conv_out}


def block_decode_step(u_t, BW, k, h, conv_state, io="f32"):
    """One decode step of the block (L = 1) from the cached (h, conv_state). Returns
    (o [B, 1, d_model], h_new, conv_state_new)."""
    r = block_forward(u_t, BW, k, h0=h, conv_state=conv_state, io=io)
    return r["o"], r["h_final"], r["conv_state"]
