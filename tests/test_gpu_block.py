"""Parity of the surrounding block's CUDA path (through the C ABI) with the fp64 oracle.

* swimba_conv1d_fwd / swimba_conv1d_step: x = SiLU(causal depthwise conv) against the oracle's
  ``causal_conv1d`` on the same stored inputs. bf16 outputs: every element within one bf16 spacing
  of the oracle's (rounded) value and at least 99 % of them equal; fp32: within 1e-5 (1 + |x|).
  The carried conv state is a copy of stored inputs: bit-exact.
* swimba_block_fwd / swimba_block_step: o within 2e-2 (1 + |o|) (bf16 activations) or
  1e-4 (1 + |o|) (fp32) of the oracle's ``block_forward`` (which stores x_pre, z, x, the layer
  output and o in the io dtype where the block does); h_final within the layer's state tolerance;
  the carried conv state (in-projection outputs) as the convolution's outputs above;
  block inputs are conditioned so that no token of x sits within 2e-3 of a router tie.
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import swimba_oracle as O
from oracle.conditioning import condition_block_router_margin
from parameter_space_moe_swimba_b200 import synth
from parameter_space_moe_swimba_b200.configs import LayerConfig
from tests.swimba_cases import TOL_Y, rel_rms_err, scaled_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


def tdt(io):
    return torch.bfloat16 if io == "bf16" else torch.float32


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def bf16_spacing(v):
    """Distance to the next bf16 value above |v| (2^-7 of the leading power of two)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return np.ldexp(1.0, np.floor(np.log2(a)).astype(int) - 7)


def check_conv_values(got, ref, io):
    if io == "bf16":
        diff = np.abs(got - ref)
        assert np.all(diff <= bf16_spacing(ref) + 1e-30), f"max diff {diff.max()}"
        assert np.mean(diff == 0) >= 0.99, f"only {np.mean(diff == 0):.4f} equal"
    else:
        assert scaled_err(got, ref) <= 1e-5


# ------------------------------------------------------------------------------------------
# causal convolution
# ------------------------------------------------------------------------------------------

def conv_draw(Bsz, L, D, W, io, seed):
    g = synth.rng(seed, 100, Bsz, L, D, W)
    x_pre = synth.round_to(g.standard_normal((Bsz, L, D)), io)
    bound = 1.0 / np.sqrt(W)
    w = g.uniform(-bound, bound, (D, W)).astype(np.float32)
    b = g.uniform(-bound, bound, D).astype(np.float32)
    st = synth.round_to(g.standard_normal((Bsz, max(W - 1, 0), D)), io)
    return x_pre, w, b, st


CONV_CASES = [
    # B, L, D, W, io, with_state
    (2, 100, 256, 4, "bf16", True),
    (3, 37, 64, 4, "bf16", False),
    (1, 2, 128, 4, "bf16", True),  # fewer tokens than the state holds
    (2, 50, 136, 8, "bf16", True),  # 17 groups of 8 channels: a partial CTA
    (1, 300, 4096, 4, "bf16", True),
    (2, 65, 96, 3, "f32", True),
    (1, 33, 40, 1, "f32", False),  # no state at all
    (2, 64, 64, 2, "f32", True),  # runs end exactly at the sequence end
]


@pytest.mark.parametrize("Bsz,L,D,W,io,with_state", CONV_CASES)
def test_conv1d_fwd_matches_oracle(S, Bsz, L, D, W, io, with_state):
    x_pre, w, b, st = conv_draw(Bsz, L, D, W, io, 1)
    dims = S.swimba_dims(Bsz, L, D, 16, 8, 4, 1, S._dtype_code(io), S._dtype_code(io))
    xp_d = S.to_device(x_pre, io)
    st_d = S.to_device(st, io) if (with_state and W > 1) else None
    x_d = torch.empty((Bsz, L, D), dtype=tdt(io), device="cuda")
    so_d = torch.full((Bsz, max(W - 1, 1), D), 7.0, dtype=tdt(io), device="cuda")
    w_d, b_d = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    S.check(S.swimba_conv1d_fwd(dims, W, xp_d, w_d, b_d, st_d, x_d, so_d), "swimba_conv1d_fwd")
    torch.cuda.synchronize()
    st64 = synth.widen(st, io) if (with_state and W > 1) else None
    _, x_ref, so_ref = O.causal_conv1d(synth.widen(x_pre, io), w.astype(np.float64), b.astype(np.float64), st64)
    ref = O.round_bf16(x_ref) if io == "bf16" else x_ref
    check_conv_values(host(x_d), ref, io)
    if W > 1:
        np.testing.assert_array_equal(host(so_d)[:, : W - 1], so_ref)


def test_conv1d_split_prefill_equals_whole(S):
    Bsz, L, D, W, io = 2, 97, 256, 4, "bf16"
    x_pre, w, b, st = conv_draw(Bsz, L, D, W, io, 2)
    dims = lambda n: S.swimba_dims(Bsz, n, D, 16, 8, 4, 1, 1, 1)
    w_d, b_d = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    xp = S.to_device(x_pre, io)
    st0 = S.to_device(st, io)
    whole = torch.empty((Bsz, L, D), dtype=torch.bfloat16, device="cuda")
    s_whole = torch.empty((Bsz, W - 1, D), dtype=torch.bfloat16, device="cuda")
    S.check(S.swimba_conv1d_fwd(dims(L), W, xp, w_d, b_d, st0, whole, s_whole))
    L1 = 45
    a, b2 = xp[:, :L1].contiguous(), xp[:, L1:].contiguous()
    xa = torch.empty_like(a)
    xb = torch.empty_like(b2)
    s1 = torch.empty_like(s_whole)
    s2 = torch.empty_like(s_whole)
    S.check(S.swimba_conv1d_fwd(dims(L1), W, a, w_d, b_d, st0, xa, s1))
    S.check(S.swimba_conv1d_fwd(dims(L - L1), W, b2, w_d, b_d, s1, xb, s2))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([xa, xb], dim=1), whole)
    assert torch.equal(s2, s_whole)


@pytest.mark.parametrize("io,W,D", [("bf16", 4, 512), ("f32", 3, 96), ("bf16", 1, 64)])
def test_conv1d_step_matches_oracle(S, io, W, D):
    Bsz, steps = 3, 6
    x_pre, w, b, st = conv_draw(Bsz, steps, D, W, io, 3)
    dims = S.swimba_dims(Bsz, 1, D, 16, 8, 4, 1, S._dtype_code(io), S._dtype_code(io))
    w_d, b_d = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    state = S.to_device(st, io) if W > 1 else None
    st64 = synth.widen(st, io) if W > 1 else None
    _, x_ref, so_ref = O.causal_conv1d(synth.widen(x_pre, io), w.astype(np.float64), b.astype(np.float64), st64)
    ref = O.round_bf16(x_ref) if io == "bf16" else x_ref
    xp = S.to_device(x_pre, io)
    for t in range(steps):
        x_t = torch.empty((Bsz, 1, D), dtype=tdt(io), device="cuda")
        S.check(S.swimba_conv1d_step(dims, W, xp[:, t:t + 1].contiguous(), w_d, b_d, state, x_t), "swimba_conv1d_step")
        torch.cuda.synchronize()
        check_conv_values(host(x_t)[:, 0], ref[:, t], io)
    if W > 1:
        np.testing.assert_array_equal(host(state), so_ref)


# ------------------------------------------------------------------------------------------
# the block
# ------------------------------------------------------------------------------------------

BLOCK_CASES = [
    # layer config, d_model, d_conv
    (LayerConfig("block_bf16", 2, 300, 512, 16, 32, 8, 2, "bf16", "bf16", 11), 256, 4),
    (LayerConfig("block_bf16_tc", 1, 2200, 256, 16, 16, 8, 2, "bf16", "bf16", 12), 128, 4),
    (LayerConfig("block_f32", 1, 70, 128, 8, 8, 4, 1, "f32", "f32", 13), 64, 3),
]


def block_case(cfg, d_model, d_conv):
    bw = synth.draw_block_weights(cfg, d_model, d_conv)
    u = synth.draw_block_input(cfg, d_model)
    cs = synth.draw_conv_state(cfg, d_conv)
    h0 = synth.draw_h0(cfg)
    BW = block_weights64(cfg, bw)
    condition_block_router_margin(
        u, lambda s: synth.widen(s, cfg.io_dtype), BW, cfg.top_k, cfg.io_dtype,
        lambda b, t, a: synth.redraw_u_row(cfg, d_model, b, t, a), conv_state=synth.widen(cs, cfg.io_dtype),
    )
    return bw, BW, u, cs, h0


def block_weights64(cfg, bw):
    lw = bw.layer
    return {
        "W_in": synth.widen(bw.W_in, cfg.w_dtype),
        "conv_w": bw.conv_w.astype(np.float64),
        "conv_b": bw.conv_b.astype(np.float64),
        "W_out": synth.widen(bw.W_out, cfg.w_dtype),
        "W_r": lw.W_r.astype(np.float64),
        "W_x": synth.widen(lw.W_x, cfg.w_dtype),
        "W_dt": synth.widen(lw.W_dt, cfg.w_dtype),
        "b_dt": lw.b_dt.astype(np.float64),
        "A": lw.A.astype(np.float64),
        "D_skip": lw.D_skip.astype(np.float64),
    }


class DeviceBlock:
    def __init__(self, S, cfg, bw, d_model, d_conv, seqlen=None):
        self.dims = S.swimba_block_dims(S.make_dims(cfg, seqlen=seqlen), d_model, d_conv)
        self.lw = S.upload_weights(bw.layer)
        self.W_in = S.to_device(bw.W_in, cfg.w_dtype)
        self.W_out = S.to_device(bw.W_out, cfg.w_dtype)
        self.conv_w = torch.from_numpy(bw.conv_w).cuda()
        self.conv_b = torch.from_numpy(bw.conv_b).cuda()
        self.w = S.swimba_block_weights(self.W_in.data_ptr(), self.conv_w.data_ptr(), self.conv_b.data_ptr(),
                                        self.W_out.data_ptr(), self.lw.struct())
        n = S.swimba_block_workspace_size(self.dims)
        assert n > 0
        self.ws = torch.zeros(n, dtype=torch.uint8, device="cuda")


def check_block(cfg, o, ref_o, h, ref_h, cs, ref_cs):
    tol = TOL_Y[cfg.io_dtype]
    assert scaled_err(o, ref_o) <= tol, scaled_err(o, ref_o)
    assert rel_rms_err(h, ref_h) <= (1e-5 if cfg.io_dtype == "f32" else 1e-2)
    # the carried conv state holds in-projection outputs: the GEMM's fp32 accumulation against the
    # oracle's fp64, then (bf16) one rounding, so within one bf16 spacing / 1e-5 (fp32)
    check_conv_values(cs, ref_cs, cfg.io_dtype)


@pytest.mark.parametrize("cfg,d_model,d_conv", BLOCK_CASES, ids=[c[0].name for c in BLOCK_CASES])
def test_block_fwd_matches_oracle(S, cfg, d_model, d_conv):
    bw, BW, u, cs, h0 = block_case(cfg, d_model, d_conv)
    dev = DeviceBlock(S, cfg, bw, d_model, d_conv)
    u_d = S.to_device(u, cfg.io_dtype)
    cs_d = S.to_device(cs, cfg.io_dtype)
    h_d = torch.from_numpy(h0).cuda()
    out = torch.empty_like(u_d)
    h_fin = torch.empty_like(h_d)
    cs_out = torch.empty_like(cs_d)
    S.check(S.swimba_block_fwd(dev.dims, u_d, dev.w, h_d, cs_d, out, h_fin, cs_out, dev.ws, dev.ws.numel()),
            "swimba_block_fwd")
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(dev.ws) == 0
    ref = O.block_forward(synth.widen(u, cfg.io_dtype), BW, cfg.top_k, h0=h0.astype(np.float64),
                          conv_state=synth.widen(cs, cfg.io_dtype), io=cfg.io_dtype)
    check_block(cfg, host(out), ref["o"], host(h_fin), ref["h_final"], host(cs_out), ref["conv_state"])


@pytest.mark.parametrize("cfg,d_model,d_conv", BLOCK_CASES[::2], ids=[c[0].name for c in BLOCK_CASES[::2]])
def test_block_prefill_then_decode_matches_oracle(S, cfg, d_model, d_conv):
    """Prefill L - 3 tokens with swimba_block_fwd, then 3 swimba_block_step calls; every output
    against the oracle's whole-sequence block."""
    bw, BW, u, cs, h0 = block_case(cfg, d_model, d_conv)
    L, Lp = cfg.seqlen, cfg.seqlen - 3
    pre = DeviceBlock(S, cfg, bw, d_model, d_conv, seqlen=Lp)
    step = DeviceBlock(S, cfg, bw, d_model, d_conv, seqlen=1)
    u_d = S.to_device(u, cfg.io_dtype)
    cs_d = S.to_device(cs, cfg.io_dtype)
    h = torch.from_numpy(h0).cuda()
    out_pre = torch.empty((cfg.batch, Lp, d_model), dtype=tdt(cfg.io_dtype), device="cuda")
    cs_state = torch.empty_like(cs_d)
    S.check(S.swimba_block_fwd(pre.dims, u_d[:, :Lp].contiguous(), pre.w, h, cs_d, out_pre, h, cs_state, pre.ws,
                               pre.ws.numel()), "swimba_block_fwd")
    outs = [host(out_pre)]
    for t in range(Lp, L):
        o_t = torch.empty((cfg.batch, 1, d_model), dtype=tdt(cfg.io_dtype), device="cuda")
        S.check(S.swimba_block_step(step.dims, u_d[:, t:t + 1].contiguous(), step.w, h, cs_state, o_t, step.ws,
                                    step.ws.numel()), "swimba_block_step")
        outs.append(host(o_t))
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(step.ws) == 0
    ref = O.block_forward(synth.widen(u, cfg.io_dtype), BW, cfg.top_k, h0=h0.astype(np.float64),
                          conv_state=synth.widen(cs, cfg.io_dtype), io=cfg.io_dtype)
    check_block(cfg, np.concatenate(outs, axis=1), ref["o"], host(h), ref["h_final"], host(cs_state),
                ref["conv_state"])
