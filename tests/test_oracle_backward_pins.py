"""Pins of the backward oracle (oracle/swimba_backward_oracle.py) to something other than itself:
every gradient against central finite differences of the pinned FORWARD oracle
(oracle/swimba_oracle.py) on small fp64 inputs, a closed form for one token, and linearity in the
incoming gradient. A finite difference of step ε has error O(ε²); the bound 1e-6 relative to the
gradient's scale is far below any dropped term, wrong sign, wrong index or transposed operand."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import swimba_backward_oracle as BO
from oracle import swimba_oracle as O

EPS = 1e-5
TOL = 1e-6


def fd_grad(loss, arr, eps=EPS, max_entries=None, rng=None):
    """Central differences of loss() w.r.t. every entry of ``arr`` (modified in place and restored);
    ``max_entries`` samples that many flat positions."""
    flat = arr.reshape(-1)
    pos = np.arange(flat.size)
    if max_entries is not None and flat.size > max_entries:
        pos = np.sort(rng.choice(flat.size, max_entries, replace=False))
    out = np.zeros(pos.size)
    for i, p in enumerate(pos):
        keep = flat[p]
        flat[p] = keep + eps
        lp = loss()
        flat[p] = keep - eps
        lm = loss()
        flat[p] = keep
        out[i] = (lp - lm) / (2 * eps)
    return pos, out


def assert_close(analytic, pos, numeric, name):
    a = analytic.reshape(-1)[pos]
    scale = max(1.0, float(np.max(np.abs(analytic))))
    err = float(np.max(np.abs(a - numeric))) / scale if pos.size else 0.0
    assert err <= TOL, f"{name}: {err:.2e}"


def small_scan(seed=0, Bsz=2, L=5, D=3, N=2, E=3, k=2):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((Bsz, L, D))
    z = rng.standard_normal((Bsz, L, D))
    delta = np.exp(rng.uniform(np.log(0.05), np.log(0.8), (Bsz, L, D)))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(Bsz * L)]).reshape(Bsz, L, k).astype(np.int32)
    g = rng.uniform(0.2, 1.0, (Bsz, L, k))
    g /= g.sum(axis=-1, keepdims=True)
    A = -rng.uniform(0.3, 2.0, (E, D, N))
    Dsk = rng.standard_normal(D)
    h0 = rng.standard_normal((Bsz, D, N)) * 0.5
    G = rng.standard_normal((Bsz, L, D))
    return dict(x=x, z=z, delta=delta, Bm=Bm, Cm=Cm, idx=idx, g=g, A=A, Dsk=Dsk, h0=h0, G=G)


def scan_loss(c):
    # the forward oracle takes dt_mix and applies softplus: pass softplus^-1(Δ)
    dt_mix = np.log(np.expm1(c["delta"]))
    _, out, _, _ = O.selective_scan(c["x"], c["z"], dt_mix, c["Bm"], c["Cm"], c["idx"], c["g"], c["A"], c["Dsk"],
                                    h0=c["h0"])
    return float(np.sum(out * c["G"]))


@pytest.mark.parametrize("seed", [0, 1])
def test_scan_backward_matches_finite_differences(seed):
    c = small_scan(seed)
    gr = BO.scan_backward(c["x"], c["z"], c["delta"], c["Bm"], c["Cm"], c["idx"], c["g"], c["A"], c["Dsk"], c["G"],
                          h0=c["h0"])
    for key, name in [("x", "dx"), ("z", "dz"), ("delta", "ddelta"), ("Bm", "dB"), ("Cm", "dC"), ("g", "dgates"),
                      ("A", "dA"), ("Dsk", "dD"), ("h0", "dh0")]:
        pos, num = fd_grad(lambda: scan_loss(c), c[key])
        assert_close(gr[name], pos, num, name)


def test_scan_backward_forward_outputs_equal_the_forward_oracle():
    c = small_scan(3)
    gr = BO.scan_backward(c["x"], c["z"], c["delta"], c["Bm"], c["Cm"], c["idx"], c["g"], c["A"], c["Dsk"], c["G"],
                          h0=c["h0"])
    _, out, hf, _ = O.selective_scan(c["x"], c["z"], np.log(np.expm1(c["delta"])), c["Bm"], c["Cm"], c["idx"], c["g"],
                                     c["A"], c["Dsk"], h0=c["h0"])
    np.testing.assert_allclose(gr["out"], out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gr["h_final"], hf, rtol=1e-12, atol=1e-12)


def test_scan_backward_one_token_closed_form():
    """L = 1, h0 = 0: out = (Δ x Σ_n C_n B_n + D x) SiLU(z), so
    ∂out/∂x = (Δ Σ_n C_n B_n + D) SiLU(z), ∂out/∂Δ = x Σ_n C_n B_n SiLU(z),
    ∂out/∂B_n = Σ_d Δ x C_n SiLU(z) G, and A gets no gradient (h_{-1} = 0)."""
    c = small_scan(4, Bsz=1, L=1, D=4, N=3)
    gr = BO.scan_backward(c["x"], c["z"], c["delta"], c["Bm"], c["Cm"], c["idx"], c["g"], c["A"], c["Dsk"], c["G"])
    cb = float(np.sum(c["Cm"][0, 0] * c["Bm"][0, 0]))
    s = O.silu(c["z"][0, 0])
    G, d, x = c["G"][0, 0], c["delta"][0, 0], c["x"][0, 0]
    np.testing.assert_allclose(gr["dx"][0, 0], (d * cb + c["Dsk"]) * s * G, rtol=1e-12)
    np.testing.assert_allclose(gr["ddelta"][0, 0], x * cb * s * G, rtol=1e-12)
    np.testing.assert_allclose(gr["dB"][0, 0], c["Cm"][0, 0] * np.sum(d * x * s * G), rtol=1e-12)
    np.testing.assert_allclose(gr["dC"][0, 0], c["Bm"][0, 0] * np.sum(d * x * s * G), rtol=1e-12)
    assert np.all(gr["dA"] == 0) and np.all(gr["dgates"] == 0)


def test_scan_backward_is_linear_in_the_incoming_gradient():
    c = small_scan(5)
    args = (c["x"], c["z"], c["delta"], c["Bm"], c["Cm"], c["idx"], c["g"], c["A"], c["Dsk"])
    G2 = np.random.default_rng(9).standard_normal(c["G"].shape)
    g1 = BO.scan_backward(*args, c["G"], h0=c["h0"])
    g2 = BO.scan_backward(*args, G2, h0=c["h0"])
    g12 = BO.scan_backward(*args, 2.0 * c["G"] - 3.0 * G2, h0=c["h0"])
    for name in ("dx", "dz", "ddelta", "dB", "dC", "dgates", "dA", "dD", "dh0"):
        np.testing.assert_allclose(g12[name], 2.0 * g1[name] - 3.0 * g2[name], rtol=1e-10, atol=1e-12)


def small_proj(seed=0, T=6, D=5, R=3, N=2, E=3, k=2):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, D))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    g = rng.uniform(0.2, 1.0, (T, k))
    g /= g.sum(axis=-1, keepdims=True)
    W_x = rng.standard_normal((E, D, R + 2 * N)) / np.sqrt(D)
    W_dt = rng.standard_normal((E, R, D)) / np.sqrt(R)
    b_dt = rng.standard_normal((E, D))
    G1, G2, G3 = rng.standard_normal((T, D)), rng.standard_normal((T, N)), rng.standard_normal((T, N))
    return dict(x=x, idx=idx, g=g, W_x=W_x, W_dt=W_dt, b_dt=b_dt, G1=G1, G2=G2, G3=G3, R=R, N=N)


@pytest.mark.parametrize("seed", [0, 1])
def test_projection_backward_matches_finite_differences(seed):
    c = small_proj(seed)

    def loss():
        pr = O.expert_projections(c["x"], c["idx"], c["g"], c["W_x"], c["W_dt"], c["b_dt"], c["R"], c["N"])
        return float(np.sum(pr["dt_mix"] * c["G1"]) + np.sum(pr["B_mix"] * c["G2"]) + np.sum(pr["C_mix"] * c["G3"]))

    gr = BO.projection_backward(c["x"], c["idx"], c["g"], c["W_x"], c["W_dt"], c["b_dt"], c["R"], c["N"], c["G1"],
                                c["G2"], c["G3"])
    for key, name in [("x", "dx"), ("g", "dgates"), ("W_x", "dW_x"), ("W_dt", "dW_dt"), ("b_dt", "db_dt")]:
        pos, num = fd_grad(loss, c[key])
        assert_close(gr[name], pos, num, name)


def test_softplus_backward_matches_finite_differences():
    v = np.linspace(-30, 30, 61)
    G = np.cos(v)
    num = (np.sum(O.softplus(v + EPS) * G) - np.sum(O.softplus(v - EPS) * G)) / (2 * EPS)
    ana = np.sum(BO.softplus_backward(v, G))
    assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana))
    # σ(v) elementwise: 1/2 at 0, → 1 and → 0 at the ends
    s = BO.softplus_backward(np.array([0.0, 40.0, -40.0]), np.ones(3))
    np.testing.assert_allclose(s, [0.5, 1.0, np.exp(-40.0)], rtol=1e-12)


def test_route_backward_matches_finite_differences():
    rng = np.random.default_rng(2)
    T, D, E, k = 5, 4, 4, 2
    x = rng.standard_normal((T, D))
    W_r = rng.standard_normal((D, E))
    idx, _, logits = O.route(x, W_r, k)
    srt = np.sort(logits, axis=1)
    assert np.min(srt[:, -k] - srt[:, -k - 1]) > 1e-3  # no selection flips under ±ε
    G = rng.standard_normal((T, k))

    def loss():
        i2, g2, _ = O.route(x, W_r, k)
        assert np.array_equal(i2, idx)
        return float(np.sum(g2 * G))

    gr = BO.route_backward(x, W_r, idx, G)
    for arr, name in [(x, "dx"), (W_r, "dW_r")]:
        pos, num = fd_grad(loss, arr)
        assert_close(gr[name], pos, num, name)


def test_top1_gate_has_no_gradient():
    rng = np.random.default_rng(4)
    x, W_r = rng.standard_normal((3, 4)), rng.standard_normal((4, 5))
    idx, _, _ = O.route(x, W_r, 1)
    gr = BO.route_backward(x, W_r, idx, rng.standard_normal((3, 1)))
    assert np.all(gr["dx"] == 0) and np.all(gr["dW_r"] == 0)


def test_layer_backward_matches_finite_differences():
    rng = np.random.default_rng(7)
    Bsz, L, D, N, R, E, k = 1, 4, 4, 2, 2, 3, 2
    x = rng.standard_normal((Bsz, L, D))
    z = rng.standard_normal((Bsz, L, D))
    W = {
        "W_r": rng.standard_normal((D, E)), "W_x": rng.standard_normal((E, D, R + 2 * N)) / 2,
        "W_dt": rng.standard_normal((E, R, D)) / 2, "b_dt": rng.standard_normal((E, D)) - 1.0,
        "A": -rng.uniform(0.3, 2.0, (E, D, N)), "D_skip": rng.standard_normal(D),
    }
    h0 = rng.standard_normal((Bsz, D, N)) * 0.5
    G = rng.standard_normal((Bsz, L, D))
    _, _, logits = O.route(x.reshape(-1, D), W["W_r"], k)
    srt = np.sort(logits, axis=1)
    assert np.min(srt[:, -k] - srt[:, -k - 1]) > 1e-3

    def loss():
        return float(np.sum(O.layer_forward(x, z, W, k, h0=h0)["out"] * G))

    gr = BO.layer_backward(x, z, W, k, G, h0=h0)
    np.testing.assert_allclose(gr["out"], O.layer_forward(x, z, W, k, h0=h0)["out"], rtol=1e-12, atol=1e-12)
    for arr, name in [(x, "dx"), (z, "dz"), (W["W_r"], "dW_r"), (W["W_x"], "dW_x"), (W["W_dt"], "dW_dt"),
                      (W["b_dt"], "db_dt"), (W["A"], "dA"), (W["D_skip"], "dD"), (h0, "dh0")]:
        pos, num = fd_grad(loss, arr)
        assert_close(gr[name], pos, num, name)
