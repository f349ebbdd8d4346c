"""Pins of the oracle's surrounding-block functions (causal convolution, bf16 storage rounding, the
block) against facts that do not come from the oracle itself: a library convolution, torch's
bf16 rounding, impulse responses, causality, the residual, state hand-off and linearity."""
import numpy as np
import pytest
import torch

from oracle import swimba_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def conv_inputs(Bsz=2, L=11, D=5, W=4, seed=3):
    g = np.random.default_rng(seed)
    return (g.standard_normal((Bsz, L, D)), g.standard_normal((D, W)), g.standard_normal(D),
            g.standard_normal((Bsz, W - 1, D)))


def block_weights(dm=6, D=8, N=4, R=3, E=4, W=4, seed=5):
    g = np.random.default_rng(seed)
    return {
        "W_in": g.standard_normal((dm, 2 * D)) / np.sqrt(dm),
        "conv_w": g.standard_normal((D, W)) / np.sqrt(W),
        "conv_b": 0.3 * g.standard_normal(D),
        "W_out": g.standard_normal((D, dm)) / np.sqrt(D),
        "W_r": g.standard_normal((D, E)) / np.sqrt(D),
        "W_x": g.standard_normal((E, D, R + 2 * N)) / np.sqrt(D),
        "W_dt": g.standard_normal((E, R, D)) / np.sqrt(R),
        "b_dt": np.log(np.expm1(np.exp(g.uniform(np.log(1e-3), np.log(1e-1), (E, D))))),
        "A": -np.exp(g.uniform(np.log(0.5), np.log(8.0), (E, D, N))),
        "D_skip": g.standard_normal(D),
    }


def block_input(Bsz=2, L=10, dm=6, seed=9):
    return np.random.default_rng(seed).standard_normal((Bsz, L, dm))


# ------------------------------------------------------------------------------------------
# causal convolution
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("W", [1, 2, 4, 5])
def test_conv1d_matches_library_convolution(W):
    x, w, b, st = conv_inputs(W=W)
    c, xo, st_out = O.causal_conv1d(x, w, b, st)
    p = np.concatenate([st, x], axis=1)
    for bb in range(x.shape[0]):
        for d in range(x.shape[2]):
            # np.convolve flips its second argument: reversed taps give sum_i w[i] p[t+i]
            ref = np.convolve(p[bb, :, d], w[d, ::-1], mode="valid") + b[d]
            np.testing.assert_allclose(c[bb, :, d], ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(xo, c / (1.0 + np.exp(-c)), rtol=1e-14)
    np.testing.assert_array_equal(st_out, p[:, -(W - 1):, :] if W > 1 else p[:, :0, :])


def test_conv1d_impulse_taps_are_identity_and_shift():
    x, w, b, st = conv_inputs(W=4)
    D, W = w.shape
    last = np.zeros((D, W))
    last[:, W - 1] = 1.0
    c, _, _ = O.causal_conv1d(x, last, np.zeros(D), st)
    np.testing.assert_array_equal(c, x)  # the current token only
    first = np.zeros((D, W))
    first[:, 0] = 1.0
    c, _, _ = O.causal_conv1d(x, first, np.zeros(D), st)
    np.testing.assert_array_equal(c[:, W - 1:], x[:, :-(W - 1)])  # W-1 tokens back
    np.testing.assert_array_equal(c[:, :W - 1], st)  # ... reaching into the carried state


def test_conv1d_zero_state_when_absent():
    x, w, b, _ = conv_inputs(W=3)
    c0, _, _ = O.causal_conv1d(x, w, b, None)
    c1, _, _ = O.causal_conv1d(x, w, b, np.zeros((x.shape[0], 2, x.shape[2])))
    np.testing.assert_array_equal(c0, c1)
    # the first output sees only the current token and the bias
    np.testing.assert_allclose(c0[:, 0], w[None, :, 2] * x[:, 0] + b[None, :], rtol=1e-15)


@pytest.mark.parametrize("L1", [1, 2, 7])
def test_conv1d_state_handoff_equals_whole(L1):
    x, w, b, st = conv_inputs(L=9, W=4)
    c, _, s_all = O.causal_conv1d(x, w, b, st)
    c1, _, s1 = O.causal_conv1d(x[:, :L1], w, b, st)
    c2, _, s2 = O.causal_conv1d(x[:, L1:], w, b, s1)
    np.testing.assert_allclose(np.concatenate([c1, c2], axis=1), c, rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(s2, s_all)


def test_round_bf16_matches_torch():
    g = np.random.default_rng(4)
    v = np.concatenate([
        g.standard_normal(20000) * np.exp(g.uniform(-20, 20, 20000)),
        # exact ties between two bf16 neighbours: 1 + (2j+1) 2^-8, and their negatives
        1.0 + (2 * np.arange(64) + 1) * 2.0 ** -8,
        -(3.0 + (2 * np.arange(64) + 1) * 2.0 ** -7),
        [0.0, 1.0, -2.5],
    ])
    # torch rounds fp32 -> bf16; go through fp32 only for values fp32 holds exactly
    v = v.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(v), ref)


# ------------------------------------------------------------------------------------------
# the block
# ------------------------------------------------------------------------------------------

def test_block_is_residual_when_W_out_is_zero():
    BW = block_weights()
    BW["W_out"] = np.zeros_like(BW["W_out"])
    u = block_input()
    np.testing.assert_array_equal(O.block_forward(u, BW, 2)["o"], u)


def test_block_zero_gate_branch_gives_residual():
    BW = block_weights()
    D = BW["conv_w"].shape[0]
    BW["W_in"][:, D:] = 0.0  # z = 0, SiLU(0) = 0: the gated layer output vanishes
    u = block_input()
    r = O.block_forward(u, BW, 2)
    np.testing.assert_array_equal(r["o"], u)
    assert np.abs(r["x"]).max() > 0.05  # the SSM branch itself is not zero


def test_block_zero_convolution_gives_residual():
    BW = block_weights()
    BW["conv_w"] = np.zeros_like(BW["conv_w"])
    BW["conv_b"] = np.zeros_like(BW["conv_b"])  # x = SiLU(0) = 0: no input reaches the state
    u = block_input()
    r = O.block_forward(u, BW, 2)
    np.testing.assert_array_equal(r["o"], u)
    assert np.abs(r["x_pre"]).max() > 0.1


def test_block_ssm_branch_takes_the_first_half_of_W_in():
    BW = block_weights()
    D = BW["conv_w"].shape[0]
    u = block_input()
    r = O.block_forward(u, BW, 2)
    # the convolution input is u times the first D columns, the gate the last D columns
    BW2 = dict(BW, W_in=np.concatenate([BW["W_in"][:, :D], np.zeros_like(BW["W_in"][:, D:])], axis=1))
    np.testing.assert_allclose(O.block_forward(u, BW2, 2)["x"], r["x"], rtol=1e-14, atol=1e-15)


def test_block_is_causal():
    BW = block_weights()
    u = block_input(L=12)
    o = O.block_forward(u, BW, 2)["o"]
    u2 = u.copy()
    u2[:, 7:] += np.random.default_rng(1).standard_normal(u2[:, 7:].shape)
    o2 = O.block_forward(u2, BW, 2)["o"]
    np.testing.assert_array_equal(o2[:, :7], o[:, :7])
    assert np.all(np.abs(o2[:, 7] - o[:, 7]).max(axis=-1) > 1e-6)


@pytest.mark.parametrize("L1", [1, 2, 6])
def test_block_split_and_decode_equal_whole(L1):
    BW = block_weights()
    Bsz, L = 2, 9
    u = block_input(Bsz=Bsz, L=L)
    g = np.random.default_rng(2)
    h0 = 0.3 * g.standard_normal((Bsz, 8, 4))
    cs0 = g.standard_normal((Bsz, 3, 8))
    whole = O.block_forward(u, BW, 2, h0=h0, conv_state=cs0)
    a = O.block_forward(u[:, :L1], BW, 2, h0=h0, conv_state=cs0)
    b = O.block_forward(u[:, L1:], BW, 2, h0=a["h_final"], conv_state=a["conv_state"])
    np.testing.assert_allclose(np.concatenate([a["o"], b["o"]], axis=1), whole["o"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b["h_final"], whole["h_final"], rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(b["conv_state"], whole["conv_state"])
    h, cs = h0, cs0
    for t in range(L):
        o_t, h, cs = O.block_decode_step(u[:, t:t + 1], BW, 2, h, cs)
        np.testing.assert_allclose(o_t[:, 0], whole["o"][:, t], rtol=1e-12, atol=1e-12)


def test_block_output_minus_residual_is_linear_in_W_out():
    BW = block_weights()
    u = block_input()
    g = np.random.default_rng(6)
    W1 = g.standard_normal(BW["W_out"].shape)
    W2 = g.standard_normal(BW["W_out"].shape)
    f = lambda W: O.block_forward(u, dict(BW, W_out=W), 2)["o"] - u
    np.testing.assert_allclose(f(W1 + 2.0 * W2), f(W1) + 2.0 * f(W2), rtol=1e-11, atol=1e-11)


def test_block_bf16_stores_bf16_values():
    BW = block_weights()
    u = O.round_bf16(block_input())
    r = O.block_forward(u, BW, 2, io="bf16")
    for key in ("x_pre", "z", "x", "o"):
        np.testing.assert_array_equal(O.round_bf16(r[key]), r[key])
    rf = O.block_forward(u, BW, 2, io="f32")
    assert np.abs(r["o"] - rf["o"]).max() < 0.05 * (1 + np.abs(rf["o"]).max())


# ------------------------------------------------------------------------------------------
# the block's seeded inputs
# ------------------------------------------------------------------------------------------

def test_block_draws_are_reproducible_piecewise_and_follow_the_recipe():
    from parameter_space_moe_swimba_b200 import synth
    from parameter_space_moe_swimba_b200.configs import CONFIGS

    cfg = CONFIGS["mamba130m_like"].with_(seqlen=24)
    dm, W = 256, 4
    w1, w2 = synth.draw_block_weights(cfg, dm, W), synth.draw_block_weights(cfg, dm, W)
    np.testing.assert_array_equal(w1.W_in, w2.W_in)
    np.testing.assert_array_equal(w1.conv_w, w2.conv_w)
    assert w1.W_in.shape == (dm, 2 * cfg.d_inner) and w1.W_in.dtype == np.uint16
    assert w1.W_out.shape == (cfg.d_inner, dm) and w1.conv_w.shape == (cfg.d_inner, W)
    bound = 1.0 / np.sqrt(W)
    assert np.all(np.abs(w1.conv_w) <= bound) and np.all(np.abs(w1.conv_b) <= bound)
    # the layer's weights inside the block are the layer's own draw
    np.testing.assert_array_equal(w1.layer.W_x, synth.draw_weights(cfg).W_x)
    # scale: W_in ~ N(0, 1/d_model)
    w_in = synth.widen(w1.W_in, "bf16")
    assert abs(w_in.std() * np.sqrt(dm) - 1.0) < 0.02
    u = synth.draw_block_input(cfg, dm)
    u2 = synth.draw_block_input(cfg, dm, batch_rows=[3])
    np.testing.assert_array_equal(u[3], u2[0])
    cs = synth.draw_conv_state(cfg, W)
    assert cs.shape == (cfg.batch, W - 1, cfg.d_inner) and cs.dtype == np.uint16
    r1 = synth.redraw_u_row(cfg, dm, 1, 5, 0)
    np.testing.assert_array_equal(r1, synth.redraw_u_row(cfg, dm, 1, 5, 0))
    assert not np.array_equal(r1, synth.redraw_u_row(cfg, dm, 1, 5, 1))
