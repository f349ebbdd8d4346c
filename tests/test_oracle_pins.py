"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

No source page prints a worked numeric example of the layer, so every pin is a closed form, a
brute-force evaluation on a tiny input, an invariant the sources state (gates sum to one, one
state trajectory, bounded output under a contractive transition), a special case that reduces to
a plain selective scan, or a library routine (math.log1p, torch's bf16 rounding).
"""
import itertools
import math

import numpy as np
import pytest

from oracle import swimba_oracle as O
from oracle.conditioning import condition_router_margin, near_tie_mask
from parameter_space_moe_swimba_b200 import synth
from parameter_space_moe_swimba_b200.configs import CONFIGS, LayerConfig

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def tiny_cfg(**kw):
    base = LayerConfig("t", 2, 9, 12, 4, 3, 5, 2, "f32", "f32", 7)
    return base.with_(**kw)


def weights64(cfg, a_mode="random"):
    w = synth.draw_weights(cfg, a_mode=a_mode)
    return {
        "W_r": w.W_r.astype(np.float64),
        "W_x": synth.widen(w.W_x, cfg.w_dtype),
        "W_dt": synth.widen(w.W_dt, cfg.w_dtype),
        "b_dt": w.b_dt.astype(np.float64),
        "A": w.A.astype(np.float64),
        "D_skip": w.D_skip.astype(np.float64),
    }


def acts64(cfg):
    x, z = synth.draw_activations(cfg)
    return synth.widen(x, cfg.io_dtype), synth.widen(z, cfg.io_dtype)


# ------------------------------------------------------------------------------------------
# elementwise functions
# ------------------------------------------------------------------------------------------

def test_softplus_special_values_and_library():
    assert O.softplus(0.0) == pytest.approx(math.log(2.0), rel=0, abs=1e-16)
    for v in [-30.0, -9.2, -4.6, -1.0, -1e-3, 0.5, 3.0, 19.0]:
        assert O.softplus(v) == pytest.approx(math.log1p(math.exp(v)), rel=1e-15)
    v = np.linspace(-40, 40, 1001)
    # softplus(v) - softplus(-v) = v
    np.testing.assert_allclose(O.softplus(v) - O.softplus(-v), v, rtol=0, atol=1e-13)
    assert O.softplus(800.0) == 800.0  # no overflow
    assert np.all(O.softplus(v) > 0)


def test_silu_identities():
    assert O.silu(0.0) == 0.0
    v = np.linspace(-30, 30, 601)
    # silu(v) - silu(-v) = v ; silu(v) -> v for large v
    np.testing.assert_allclose(O.silu(v) - O.silu(-v), v, rtol=0, atol=1e-13)
    assert O.silu(40.0) == pytest.approx(40.0, rel=1e-15)
    assert O.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-16)


# ------------------------------------------------------------------------------------------
# router
# ------------------------------------------------------------------------------------------

def test_router_logits_unit_vector_picks_a_row():
    rng = np.random.default_rng(1)
    W_r = rng.standard_normal((6, 4))
    for i in range(6):
        e = np.zeros(6)
        e[i] = 1.0
        np.testing.assert_array_equal(O.router_logits(e, W_r), W_r[i])


@pytest.mark.parametrize("E,k", [(4, 1), (4, 2), (5, 3), (3, 3), (6, 2)])
def test_route_brute_force(E, k):
    rng = np.random.default_rng(E * 10 + k)
    logits = rng.standard_normal((50, E))
    # introduce exact ties in some rows
    logits[::7, 1] = logits[::7, 0]
    logits[::5, E - 1] = logits[::5, 0]
    x = logits  # with W_r = I the logits are x itself
    idx, gates, lg = O.route(x, np.eye(E), k)
    np.testing.assert_array_equal(lg, logits)
    for r in range(logits.shape[0]):
        row = logits[r]
        # brute force: the lexicographically first (descending value, ascending index) ordering
        best = sorted(range(E), key=lambda e: (-row[e], e))[:k]
        assert list(idx[r]) == best
        # gates: renormalised full softmax over the selected experts
        p = np.exp(row - row.max())
        p /= p.sum()
        ref = p[best] / p[best].sum()
        np.testing.assert_allclose(gates[r], ref, rtol=1e-13, atol=0)
        assert abs(gates[r].sum() - 1.0) <= 1e-15
        assert np.all(gates[r] >= 0) and np.all(np.diff(gates[r]) <= 0)


def test_route_top1_gate_is_exactly_one():
    rng = np.random.default_rng(3)
    idx, gates, lg = O.route(rng.standard_normal((40, 8)), rng.standard_normal((8, 4)), 1)
    assert np.all(gates == 1.0)
    np.testing.assert_array_equal(idx[:, 0], np.argmax(lg, axis=1))


# ------------------------------------------------------------------------------------------
# expert projections and parameter-space mixing
# ------------------------------------------------------------------------------------------

def test_projection_unit_vector_selects_weight_row():
    cfg = tiny_cfg()
    W = weights64(cfg)
    D, R, N, E = cfg.d_inner, cfg.dt_rank, cfg.d_state, cfg.n_experts
    for i in [0, 5, D - 1]:
        x = np.zeros((E, D))
        x[:, i] = 1.0
        idx = np.stack([np.arange(E), (np.arange(E) + 1) % E], axis=1).astype(np.int32)
        gates = np.tile([0.75, 0.25], (E, 1))
        p = O.expert_projections(x, idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N)
        for t in range(E):
            for j in range(2):
                e = idx[t, j]
                np.testing.assert_array_equal(p["xdbl"][t, j], W["W_x"][e, i])
                np.testing.assert_allclose(
                    p["dt_j"][t, j], W["W_x"][e, i, :R] @ W["W_dt"][e] + W["b_dt"][e], rtol=1e-14, atol=1e-14
                )
            e0, e1 = idx[t]
            np.testing.assert_allclose(
                p["B_mix"][t], 0.75 * W["W_x"][e0, i, R:R + N] + 0.25 * W["W_x"][e1, i, R:R + N], rtol=1e-15
            )
            np.testing.assert_allclose(
                p["C_mix"][t], 0.75 * W["W_x"][e0, i, R + N:] + 0.25 * W["W_x"][e1, i, R + N:], rtol=1e-15
            )


def test_projection_brute_force_loops():
    cfg = tiny_cfg()
    W = weights64(cfg)
    x, _ = acts64(cfg)
    x = x.reshape(-1, cfg.d_inner)
    idx, gates, _ = O.route(x, W["W_r"], cfg.top_k)
    R, N, D = cfg.dt_rank, cfg.d_state, cfg.d_inner
    p = O.expert_projections(x, idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N)
    for t in range(x.shape[0]):
        dt_mix = [0.0] * D
        Bm = [0.0] * N
        Cm = [0.0] * N
        for j in range(cfg.top_k):
            e = idx[t, j]
            v = [sum(x[t, d] * W["W_x"][e, d, c] for d in range(D)) for c in range(R + 2 * N)]
            for d in range(D):
                dt_mix[d] += gates[t, j] * (sum(v[r] * W["W_dt"][e, r, d] for r in range(R)) + W["b_dt"][e, d])
            for n in range(N):
                Bm[n] += gates[t, j] * v[R + n]
                Cm[n] += gates[t, j] * v[R + N + n]
        np.testing.assert_allclose(p["dt_mix"][t], dt_mix, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(p["B_mix"][t], Bm, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(p["C_mix"][t], Cm, rtol=1e-12, atol=1e-13)


def test_mixing_streams_equals_mixing_weights():
    """Σ_j g_j (x W^{e_j}) = x (Σ_j g_j W^{e_j}): mixing in parameter space is linear."""
    cfg = tiny_cfg()
    W = weights64(cfg)
    x, _ = acts64(cfg)
    x = x.reshape(-1, cfg.d_inner)
    idx, gates, _ = O.route(x, W["W_r"], cfg.top_k)
    R, N = cfg.dt_rank, cfg.d_state
    p = O.expert_projections(x, idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N)
    for t in range(x.shape[0]):
        Wmix = sum(gates[t, j] * W["W_x"][idx[t, j]] for j in range(cfg.top_k))
        v = x[t] @ Wmix
        np.testing.assert_allclose(p["B_mix"][t], v[R:R + N], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(p["C_mix"][t], v[R + N:], rtol=1e-12, atol=1e-14)


def test_zero_dt_projection_leaves_mixed_bias():
    cfg = tiny_cfg()
    W = weights64(cfg)
    W["W_dt"][:] = 0.0
    x, _ = acts64(cfg)
    x = x.reshape(-1, cfg.d_inner)
    idx, gates, _ = O.route(x, W["W_r"], cfg.top_k)
    p = O.expert_projections(x, idx, gates, W["W_x"], W["W_dt"], W["b_dt"], cfg.dt_rank, cfg.d_state)
    ref = sum(gates[:, j, None] * W["b_dt"][idx[:, j]] for j in range(cfg.top_k))
    np.testing.assert_allclose(p["dt_mix"], ref, rtol=1e-15, atol=0)


# ------------------------------------------------------------------------------------------
# scan
# ------------------------------------------------------------------------------------------

def test_scan_closed_form_constant_inputs_scalar_state():
    """N = D = 1, constant Δ, A, B, x, C: h_t = a^{t+1} h0 + u (1 - a^{t+1}) / (1 - a)."""
    L = 10_000
    dt, A, Bv, Cv, xv, Dv, h0 = -2.0, -0.7, 0.9, -1.3, 0.8, 0.45, 0.6
    delta = math.log1p(math.exp(dt))
    a = math.exp(delta * A)
    u = delta * Bv * xv
    x = np.full((1, L, 1), xv)
    z = np.full((1, L, 1), 2.0)
    y, out, hT, _ = O.selective_scan(
        x, z, np.full((1, L, 1), dt), np.full((1, L, 1), Bv), np.full((1, L, 1), Cv),
        np.zeros((1, L, 1), np.int32), np.ones((1, L, 1)), np.full((1, 1, 1), A), np.array([Dv]),
        h0=np.full((1, 1, 1), h0),
    )
    t = np.arange(L)
    h = a ** (t + 1) * h0 + u * (1 - a ** (t + 1)) / (1 - a)
    np.testing.assert_allclose(y[0, :, 0], Cv * h + Dv * xv, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(hT[0, 0, 0], h[-1], rtol=1e-12)
    np.testing.assert_allclose(out[0, :, 0], y[0, :, 0] * 2.0 / (1 + math.exp(-2.0)), rtol=1e-14)


@pytest.mark.parametrize("L", [1, 2, 5, 8])
def test_scan_brute_force_unrolled_sum(L):
    """h_t = Σ_{s≤t} (Π_{r=s+1..t} a_r) u_s + (Π_{r≤t} a_r) h0 with random mixed parameters."""
    rng = np.random.default_rng(100 + L)
    Bsz, D, N, E, k = 2, 3, 4, 5, 2
    x = rng.standard_normal((Bsz, L, D))
    z = rng.standard_normal((Bsz, L, D))
    dt = rng.normal(-2, 1, (Bsz, L, D))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(Bsz * L)]).reshape(Bsz, L, k).astype(np.int32)
    g = rng.random((Bsz, L, k))
    g /= g.sum(-1, keepdims=True)
    A = -np.exp(rng.uniform(-1, 3, (E, D, N)))
    Dsk = rng.standard_normal(D)
    h0 = rng.standard_normal((Bsz, D, N))
    y, out, hT, delta = O.selective_scan(x, z, dt, Bm, Cm, idx, g, A, Dsk, h0=h0)
    for b in range(Bsz):
        for d in range(D):
            for n in range(N):
                a = []
                u = []
                for t in range(L):
                    dl = math.log1p(math.exp(dt[b, t, d]))
                    At = sum(g[b, t, j] * A[idx[b, t, j], d, n] for j in range(k))
                    a.append(math.exp(dl * At))
                    u.append(dl * Bm[b, t, n] * x[b, t, d])
                for t in range(L):
                    h = math.prod(a[: t + 1]) * h0[b, d, n]
                    for s in range(t + 1):
                        h += math.prod(a[s + 1: t + 1]) * u[s]
                    if t == L - 1:
                        assert hT[b, d, n] == pytest.approx(h, rel=1e-13, abs=1e-14)
    # readout: y_t = C_t · h_t + D x_t, checked through a second brute-force pass over n
    for b in range(Bsz):
        for d in range(D):
            hs = np.zeros((L, N))
            for n in range(N):
                hcur = h0[b, d, n]
                for t in range(L):
                    dl = math.log1p(math.exp(dt[b, t, d]))
                    At = sum(g[b, t, j] * A[idx[b, t, j], d, n] for j in range(k))
                    hcur = math.exp(dl * At) * hcur + dl * Bm[b, t, n] * x[b, t, d]
                    hs[t, n] = hcur
            ref = (Cm[b] * hs).sum(-1) + Dsk[d] * x[b, :, d]
            np.testing.assert_allclose(y[b, :, d], ref, rtol=1e-13, atol=1e-14)


def test_identical_experts_reduce_to_dense_scan():
    """Theorem 1: mixing identical experts is one selective SSM; routing becomes irrelevant."""
    cfg = tiny_cfg(batch=2, seqlen=17)
    W = weights64(cfg)
    for key in ["W_x", "W_dt", "b_dt", "A"]:
        W[key][:] = W[key][2]
    x, z = acts64(cfg)
    r1 = O.layer_forward(x, z, W, cfg.top_k)
    W2 = dict(W)
    W2["W_r"] = np.random.default_rng(9).standard_normal(W["W_r"].shape)  # a different router
    r2 = O.layer_forward(x, z, W2, cfg.top_k)
    assert not np.array_equal(r1["idx"], r2["idx"])
    np.testing.assert_allclose(r1["y"], r2["y"], rtol=1e-12, atol=1e-13)
    # ... and equals the single-expert (E=1, k=1) layer
    W1 = {k_: (v[2:3] if k_ in ("W_x", "W_dt", "b_dt", "A") else v) for k_, v in W.items()}
    W1["W_r"] = W["W_r"][:, :1]
    r3 = O.layer_forward(x, z, W1, 1)
    np.testing.assert_allclose(r1["y"], r3["y"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r1["h_final"], r3["h_final"], rtol=1e-12, atol=1e-13)


def test_invariants_and_bibo_bound_under_fast_switching():
    """Theorem 3: a contractive mixed transition and bounded streams give a bounded state."""
    cfg = tiny_cfg(batch=3, seqlen=200, n_experts=6, top_k=2)
    W = weights64(cfg)
    x, z = acts64(cfg)
    r = O.layer_forward(x, z, W, cfg.top_k)
    g = r["gates"]
    assert np.all(g >= 0)
    np.testing.assert_allclose(g.sum(-1), 1.0, rtol=0, atol=1e-15)
    # the router switches experts from token to token
    assert np.mean(r["idx"][:, 1:, 0] != r["idx"][:, :-1, 0]) > 0.3
    A_t = sum(g[..., j, None, None] * W["A"][r["idx"][..., j]] for j in range(cfg.top_k))
    assert np.all(A_t < 0)
    a_bar = np.exp(r["delta"][..., None] * A_t)
    assert np.all((a_bar > 0) & (a_bar < 1))
    u = r["delta"][..., None] * r["B_mix"][:, :, None, :] * x[..., None]
    bound = np.max(np.abs(u), axis=1) / (1 - np.max(a_bar, axis=1))  # per (b, d, n)
    h = np.zeros((cfg.batch, cfg.d_inner, cfg.d_state))
    for t in range(cfg.seqlen):
        h = a_bar[:, t] * h + u[:, t]
        assert np.all(np.abs(h) <= bound + 1e-15)
    np.testing.assert_allclose(h, r["h_final"], rtol=1e-12, atol=1e-15)


def test_skip_path_alone_when_injection_or_readout_is_zero():
    cfg = tiny_cfg()
    W = weights64(cfg)
    R, N = cfg.dt_rank, cfg.d_state
    x, z = acts64(cfg)
    Wb = {k: v.copy() for k, v in W.items()}
    Wb["W_x"][:, :, R:R + N] = 0.0  # B = 0: the state never leaves zero
    r = O.layer_forward(x, z, Wb, cfg.top_k)
    np.testing.assert_array_equal(r["h_final"], 0.0)
    np.testing.assert_allclose(r["y"], W["D_skip"] * x, rtol=0, atol=0)
    Wc = {k: v.copy() for k, v in W.items()}
    Wc["W_x"][:, :, R + N:] = 0.0  # C = 0: nothing is read out
    h0 = np.random.default_rng(2).standard_normal((cfg.batch, cfg.d_inner, N))
    r = O.layer_forward(x, z, Wc, cfg.top_k, h0=h0)
    np.testing.assert_allclose(r["y"], W["D_skip"] * x, rtol=0, atol=0)
    assert np.any(r["h_final"] != 0)


def test_free_decay_of_the_initial_state():
    """x = 0: h_t = (Π_{r≤t} ā_r) h0, y_t = C_t · h_t (a closed-form product)."""
    cfg = tiny_cfg(seqlen=6)
    W = weights64(cfg)
    x = np.zeros((cfg.batch, cfg.seqlen, cfg.d_inner))
    x[..., 0] = 1.0  # a token that routes and projects, but channel d > 0 sees x = 0
    z = np.ones_like(x)
    h0 = np.random.default_rng(4).standard_normal((cfg.batch, cfg.d_inner, cfg.d_state))
    r = O.layer_forward(x, z, W, cfg.top_k, h0=h0)
    g = r["gates"]
    A_t = sum(g[..., j, None, None] * W["A"][r["idx"][..., j]] for j in range(cfg.top_k))
    logdecay = np.cumsum(r["delta"][..., None] * A_t, axis=1)  # Σ_r Δ_r A_r
    h = np.exp(logdecay) * h0[:, None]
    y = np.einsum("btn,btdn->btd", r["C_mix"], h)
    np.testing.assert_allclose(r["y"][..., 1:], y[..., 1:], rtol=1e-12, atol=1e-14)


def test_channel_subset_equals_full_columns():
    cfg = tiny_cfg(seqlen=11)
    W = weights64(cfg)
    x, z = acts64(cfg)
    h0 = np.random.default_rng(5).standard_normal((cfg.batch, cfg.d_inner, cfg.d_state))
    full = O.layer_forward(x, z, W, cfg.top_k, h0=h0)
    ch = [0, 7, 3]
    sub = O.layer_forward(x, z, W, cfg.top_k, h0=h0, channels=ch)
    np.testing.assert_array_equal(sub["y"], full["y"][:, :, ch])
    np.testing.assert_array_equal(sub["h_final"], full["h_final"][:, ch])


def test_chunk_split_and_step_by_step_equal_prefill():
    cfg = tiny_cfg(seqlen=13)
    W = weights64(cfg)
    x, z = acts64(cfg)
    h0 = np.random.default_rng(6).standard_normal((cfg.batch, cfg.d_inner, cfg.d_state))
    full = O.layer_forward(x, z, W, cfg.top_k, h0=h0)
    a = O.layer_forward(x[:, :5], z[:, :5], W, cfg.top_k, h0=h0)
    b = O.layer_forward(x[:, 5:], z[:, 5:], W, cfg.top_k, h0=a["h_final"])
    np.testing.assert_allclose(np.concatenate([a["out"], b["out"]], 1), full["out"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b["h_final"], full["h_final"], rtol=1e-13, atol=1e-15)
    h = h0
    outs = []
    for t in range(cfg.seqlen):
        o, h, _ = O.decode_step(h, x[:, t:t + 1], z[:, t:t + 1], W, cfg.top_k)
        outs.append(o)
    np.testing.assert_allclose(np.concatenate(outs, 1), full["out"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(h, full["h_final"], rtol=1e-13, atol=1e-15)


def test_gate_placement_out_is_y_times_silu_z():
    cfg = tiny_cfg()
    W = weights64(cfg)
    x, _ = acts64(cfg)
    z0 = np.zeros_like(x)
    assert np.all(O.layer_forward(x, z0, W, cfg.top_k)["out"] == 0)
    zbig = np.full_like(x, 50.0)
    r = O.layer_forward(x, zbig, W, cfg.top_k)
    np.testing.assert_allclose(r["out"], 50.0 * r["y"], rtol=1e-15)


# ------------------------------------------------------------------------------------------
# storage rounding and conditioning (used by both sides' inputs)
# ------------------------------------------------------------------------------------------

def test_bf16_rounding_matches_torch_and_is_direct_from_fp64():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(8)
    v32 = (rng.standard_normal(100_000) * np.exp(rng.uniform(-20, 20, 100_000))).astype(np.float32)
    bits = synth.round_f64_to_bf16_bits(v32.astype(np.float64))
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)
    one = 1.0
    cases = {
        one + 2.0 ** -8: one,  # tie -> even (down)
        one + 3 * 2.0 ** -8: one + 2.0 ** -6,  # tie -> even (up)
        one + 2.0 ** -8 + 2.0 ** -40: one + 2.0 ** -7,  # above the tie: direct rounding goes up
        -(one + 2.0 ** -8 + 2.0 ** -40): -(one + 2.0 ** -7),
    }
    for v, want in cases.items():
        got = synth.bf16_bits_to_f32(synth.round_f64_to_bf16_bits(np.array([v])))[0]
        assert got == want


def test_router_conditioning_removes_near_ties_and_fp32_agrees():
    cfg = CONFIGS["tiny_fp32"].with_(batch=2, seqlen=300, n_experts=8, top_k=2, io_dtype="bf16")
    w = synth.draw_weights(cfg)
    x, _ = synth.draw_activations(cfg)
    n = condition_router_margin(
        x, lambda s: synth.widen(s, cfg.io_dtype), w.W_r, cfg.top_k,
        lambda b, t, a: synth.redraw_x_row(cfg, b, t, a), margin=0.05,
    )
    assert n > 0
    x64 = synth.widen(x, cfg.io_dtype)
    lg = O.router_logits(x64, w.W_r)
    assert not near_tie_mask(lg, cfg.top_k, 0.05).any()
    idx64, _, _ = O.route(x64, w.W_r, cfg.top_k)
    lg32 = x64.astype(np.float32) @ w.W_r.astype(np.float32)
    idx32 = np.argsort(-lg32, axis=-1, kind="stable")[..., : cfg.top_k]
    np.testing.assert_array_equal(idx64, idx32)


def test_synthetic_draws_are_reproducible_and_piecewise():
    cfg = CONFIGS["mamba130m_like"].with_(seqlen=16)
    a, _ = synth.draw_activations(cfg)
    b, _ = synth.draw_activations(cfg, batch_rows=[2])
    np.testing.assert_array_equal(a[2], b[0])
    w1 = synth.draw_weights(cfg)
    w2 = synth.draw_weights(cfg)
    np.testing.assert_array_equal(w1.W_x, w2.W_x)
    assert w1.W_x.dtype == np.uint16 and w1.A.dtype == np.float32
    # A = -(n+1) u per (expert, channel), u in [0.5, 2]
    u = -w1.A[..., 0]
    assert np.all((u >= 0.5) & (u <= 2.0))
    np.testing.assert_allclose(w1.A, -u[..., None] * np.arange(1, cfg.d_state + 1), rtol=1e-6)
    # dt = softplus(b_dt) in [1e-3, 1e-1]
    dt = O.softplus(w1.b_dt.astype(np.float64))
    assert dt.min() >= 1e-3 * (1 - 1e-6) and dt.max() <= 1e-1 * (1 + 1e-6)


# ------------------------------------------------------------------------------------------
# splitting a sequence into pieces: summaries and their chain
# ------------------------------------------------------------------------------------------

def _random_scan_inputs(rng, Bsz, L, D, N, E, k):
    x = rng.standard_normal((Bsz, L, D))
    dt = rng.normal(-2, 1, (Bsz, L, D))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(Bsz * L)]).reshape(Bsz, L, k).astype(np.int32)
    g = rng.random((Bsz, L, k))
    g /= g.sum(-1, keepdims=True)
    A = -np.exp(rng.uniform(-1, 3, (E, D, N)))
    return x, dt, Bm, Cm, idx, g, A


def test_summary_closed_form_constant_inputs_scalar_state():
    """N = D = 1, constant Δ, A, B, x over L tokens: h_zero = u (1 - a^L) / (1 - a) and
    log_decay = L Δ A (a = e^{ΔA}, u = Δ B x)."""
    L = 5000
    dt, A, Bv, xv = -1.5, -0.3, 0.7, -1.1
    delta = math.log1p(math.exp(dt))
    a, u = math.exp(delta * A), delta * Bv * xv
    hz, ld = O.scan_summary(np.full((1, L, 1), xv), np.full((1, L, 1), dt), np.full((1, L, 1), Bv),
                            np.zeros((1, L, 1), np.int32), np.ones((1, L, 1)), np.full((1, 1, 1), A))
    np.testing.assert_allclose(hz[0, 0, 0], u * (1 - a ** L) / (1 - a), rtol=1e-12)
    np.testing.assert_allclose(ld[0, 0, 0], L * delta * A, rtol=1e-12)


@pytest.mark.parametrize("L", [1, 3, 7])
def test_summary_brute_force(L):
    """h_zero = Σ_s (Π_{r=s+1..L-1} a_r) u_s and log_decay = log Π_t a_t, by explicit loops."""
    rng = np.random.default_rng(200 + L)
    Bsz, D, N, E, k = 2, 3, 4, 5, 2
    x, dt, Bm, _, idx, g, A = _random_scan_inputs(rng, Bsz, L, D, N, E, k)
    hz, ld = O.scan_summary(x, dt, Bm, idx, g, A)
    for b in range(Bsz):
        for d in range(D):
            for n in range(N):
                a, u = [], []
                for t in range(L):
                    dl = math.log1p(math.exp(dt[b, t, d]))
                    At = sum(g[b, t, j] * A[idx[b, t, j], d, n] for j in range(k))
                    a.append(math.exp(dl * At))
                    u.append(dl * Bm[b, t, n] * x[b, t, d])
                want = sum(math.prod(a[s + 1:]) * u[s] for s in range(L))
                assert hz[b, d, n] == pytest.approx(want, rel=1e-12, abs=1e-14)
                assert ld[b, d, n] == pytest.approx(math.log(math.prod(a)), rel=1e-12, abs=1e-14)


def test_chain_of_piece_summaries_gives_the_prefix_states():
    """Cut a random sequence into uneven pieces: the chained start state of piece p equals the
    state after the first p pieces by the (separately pinned) sequential scan, from h0; and the
    state after any piece is exp(log_decay) h_in + h_zero (superposition of the linear state)."""
    rng = np.random.default_rng(7)
    Bsz, L, D, N, E, k = 2, 29, 3, 4, 5, 2
    x, dt, Bm, Cm, idx, g, A = _random_scan_inputs(rng, Bsz, L, D, N, E, k)
    z = rng.standard_normal((Bsz, L, D))
    Dsk = rng.standard_normal(D)
    h0 = rng.standard_normal((Bsz, D, N))
    cuts = [0, 4, 5, 17, 29]
    pieces = [(cuts[i], cuts[i + 1]) for i in range(len(cuts) - 1)]
    summ = [O.scan_summary(x[:, a:b], dt[:, a:b], Bm[:, a:b], idx[:, a:b], g[:, a:b], A) for a, b in pieces]
    H = O.chain_summaries(np.stack([s[0] for s in summ]), np.stack([s[1] for s in summ]), h0=h0)
    for p, (_, b) in enumerate(pieces):
        _, _, hT, _ = O.selective_scan(x[:, :b], z[:, :b], dt[:, :b], Bm[:, :b], Cm[:, :b], idx[:, :b], g[:, :b],
                                       A, Dsk, h0=h0)
        np.testing.assert_allclose(H[p + 1], hT, rtol=1e-12, atol=1e-13)
    # each piece run from its chained start state continues the whole sequence
    h_in = rng.standard_normal((Bsz, D, N))
    a, b = pieces[2]
    _, _, hT, _ = O.selective_scan(x[:, a:b], z[:, a:b], dt[:, a:b], Bm[:, a:b], Cm[:, a:b], idx[:, a:b], g[:, a:b],
                                   A, Dsk, h0=h_in)
    np.testing.assert_allclose(hT, np.exp(summ[2][1]) * h_in + summ[2][0], rtol=1e-12, atol=1e-13)
    # no h0: the chain starts from zero
    H0 = O.chain_summaries(np.stack([s[0] for s in summ]), np.stack([s[1] for s in summ]))
    assert np.all(H0[0] == 0)
    np.testing.assert_allclose(H0[1], summ[0][0], rtol=0, atol=0)


# ------------------------------------------------------------------------------------------
# the "MoE of separate SSMs" (one state trajectory per expert)
# ------------------------------------------------------------------------------------------

def _separate_inputs(rng, Bsz, L, D, N, E, k):
    x = rng.standard_normal((Bsz, L, D))
    z = rng.standard_normal((Bsz, L, D))
    dt = rng.normal(-2, 1, (Bsz, L, k, D))
    Bj = rng.standard_normal((Bsz, L, k, N))
    Cj = rng.standard_normal((Bsz, L, k, N))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(Bsz * L)]).reshape(Bsz, L, k).astype(np.int32)
    g = rng.random((Bsz, L, k))
    g /= g.sum(-1, keepdims=True)
    A = -np.exp(rng.uniform(-1, 3, (E, D, N)))
    Dsk = rng.standard_normal(D)
    h0 = rng.standard_normal((E, Bsz, D, N))
    return x, z, dt, Bj, Cj, idx, g, A, Dsk, h0


def test_separate_moe_one_expert_is_the_selective_scan():
    """E = 1, k = 1: one trajectory, the unmixed streams are the mixed ones -- the (pinned) scan."""
    rng = np.random.default_rng(11)
    x, z, dt, Bj, Cj, idx, g, A, Dsk, h0 = _separate_inputs(rng, 2, 17, 3, 4, 1, 1)
    y, out, h = O.separate_ssm_moe(x, z, dt, Bj, Cj, idx, g, A, Dsk, h0=h0)
    y2, out2, hT, _ = O.selective_scan(x, z, dt[:, :, 0], Bj[:, :, 0], Cj[:, :, 0], idx, g, A, Dsk, h0=h0[0])
    np.testing.assert_allclose(y, y2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(out, out2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(h[0], hT, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("L", [1, 4, 6])
def test_separate_moe_brute_force(L):
    """Explicit loops: each expert's state follows only the tokens routed to it; the output mixes
    the active experts' readouts with the gates and adds the skip term."""
    rng = np.random.default_rng(300 + L)
    Bsz, D, N, E, k = 2, 2, 3, 3, 2
    x, z, dt, Bj, Cj, idx, g, A, Dsk, h0 = _separate_inputs(rng, Bsz, L, D, N, E, k)
    y, out, h = O.separate_ssm_moe(x, z, dt, Bj, Cj, idx, g, A, Dsk, h0=h0)
    for b in range(Bsz):
        for d in range(D):
            state = {(e, n): h0[e, b, d, n] for e in range(E) for n in range(N)}
            for t in range(L):
                want = Dsk[d] * x[b, t, d]
                for j in range(k):
                    e = int(idx[b, t, j])
                    dl = math.log1p(math.exp(dt[b, t, j, d]))
                    for n in range(N):
                        state[e, n] = math.exp(dl * A[e, d, n]) * state[e, n] + dl * Bj[b, t, j, n] * x[b, t, d]
                    want += g[b, t, j] * sum(Cj[b, t, j, n] * state[e, n] for n in range(N))
                assert y[b, t, d] == pytest.approx(want, rel=1e-12, abs=1e-13)
                assert out[b, t, d] == pytest.approx(want * z[b, t, d] / (1 + math.exp(-z[b, t, d])), rel=1e-12,
                                                     abs=1e-13)
            for e in range(E):
                for n in range(N):
                    assert h[e, b, d, n] == pytest.approx(state[e, n], rel=1e-12, abs=1e-13)


def test_separate_moe_unchosen_expert_keeps_its_state_and_switching_differs_from_one_trajectory():
    """An expert never routed to keeps its initial state exactly. With identical experts, constant
    routing gives the single-trajectory scan; routing that switches between experts does not
    (the pages' Théorème 4: the compressed and the separate models differ when routing varies)."""
    rng = np.random.default_rng(12)
    Bsz, L, D, N, E = 1, 12, 3, 4, 3
    x, z, dt, Bj, Cj, _, _, A, Dsk, h0 = _separate_inputs(rng, Bsz, L, D, N, E, 1)
    A[:] = A[0]
    g = np.ones((Bsz, L, 1))
    const = np.zeros((Bsz, L, 1), np.int32)
    y, _, h = O.separate_ssm_moe(x, z, dt, Bj, Cj, const, g, A, Dsk, h0=h0)
    np.testing.assert_array_equal(h[1], h0[1])
    np.testing.assert_array_equal(h[2], h0[2])
    y1, _, _, _ = O.selective_scan(x, z, dt[:, :, 0], Bj[:, :, 0], Cj[:, :, 0], const, g, A, Dsk, h0=h0[0])
    np.testing.assert_allclose(y, y1, rtol=1e-13, atol=1e-14)
    switching = (np.arange(L) % 2).reshape(Bsz, L, 1).astype(np.int32)
    y2, _, _ = O.separate_ssm_moe(x, z, dt, Bj, Cj, switching, g, A, Dsk, h0=np.zeros_like(h0))
    y3, _, _, _ = O.selective_scan(x, z, dt[:, :, 0], Bj[:, :, 0], Cj[:, :, 0], switching, g, A, Dsk)
    assert np.max(np.abs(y2 - y3)) > 1e-3


# ------------------------------------------------------------------------------------------
# the zero-order-hold injection
# ------------------------------------------------------------------------------------------

def test_zoh_is_the_exact_solution_for_held_inputs():
    """With A, B and x held constant and only the step Δ_t varying, the zero-order hold integrates
    dh/dt = A h + B x exactly: after L steps h = e^{A T} h0 + (e^{A T} - 1) / A · B x, T = Σ Δ_t,
    however T is split into steps."""
    rng = np.random.default_rng(21)
    L = 1000
    A, Bv, xv, h0 = -0.37, 1.3, -0.8, 0.45
    dt = rng.normal(-3, 1.5, (1, L, 1))
    delta = np.log1p(np.exp(dt))
    T = float(delta.sum())
    _, _, hT, _ = O.selective_scan(np.full((1, L, 1), xv), np.ones((1, L, 1)), dt, np.full((1, L, 1), Bv),
                                   np.ones((1, L, 1)), np.zeros((1, L, 1), np.int32), np.ones((1, L, 1)),
                                   np.full((1, 1, 1), A), np.zeros(1), h0=np.full((1, 1, 1), h0), injection="zoh")
    want = math.exp(A * T) * h0 + math.expm1(A * T) / A * Bv * xv
    assert hT[0, 0, 0] == pytest.approx(want, rel=1e-11)


@pytest.mark.parametrize("L", [1, 3, 5])
def test_zoh_brute_force_and_small_step_limit(L):
    """Unrolled sum with u_t = (e^{Δ A_t} - 1) / A_t B x; and for tiny steps the ZOH injection tends
    to the Euler one, u_zoh / u_euler = 1 + Δ A_t / 2 + O(Δ²)."""
    rng = np.random.default_rng(400 + L)
    Bsz, D, N, E, k = 2, 2, 3, 4, 2
    x, dt, Bm, Cm, idx, g, A = _random_scan_inputs(rng, Bsz, L, D, N, E, k)
    z = rng.standard_normal((Bsz, L, D))
    Dsk = rng.standard_normal(D)
    h0 = rng.standard_normal((Bsz, D, N))
    y, _, hT, _ = O.selective_scan(x, z, dt, Bm, Cm, idx, g, A, Dsk, h0=h0, injection="zoh")
    for b in range(Bsz):
        for d in range(D):
            for t in range(L):
                want = Dsk[d] * x[b, t, d]
                for n in range(N):
                    a, u = [], []
                    for s in range(t + 1):
                        dl = math.log1p(math.exp(dt[b, s, d]))
                        At = sum(g[b, s, j] * A[idx[b, s, j], d, n] for j in range(k))
                        a.append(math.exp(dl * At))
                        u.append(math.expm1(dl * At) / At * Bm[b, s, n] * x[b, s, d])
                    h = math.prod(a) * h0[b, d, n] + sum(math.prod(a[s + 1:]) * u[s] for s in range(t + 1))
                    want += Cm[b, t, n] * h
                assert y[b, t, d] == pytest.approx(want, rel=1e-11, abs=1e-12)
    tiny = np.full_like(dt, -16.0)  # Δ = softplus(-16) ~ 1.1e-7
    _, _, hz, _ = O.selective_scan(x, z, tiny, Bm, Cm, idx, g, A, Dsk, injection="zoh")
    _, _, he, _ = O.selective_scan(x, z, tiny, Bm, Cm, idx, g, A, Dsk, injection="euler")
    np.testing.assert_allclose(hz, he, rtol=2e-5, atol=0)
