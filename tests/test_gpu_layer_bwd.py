"""Backward pass of the mixed projection (swimba_proj_bwd), of the router (swimba_route_bwd) and
of the whole layer (scan -> projection -> router, chained through the C ABI with the input
gradient accumulated in place) against the fp64 backward oracle (oracle/swimba_backward_oracle.py,
pinned by finite differences of the forward oracle).

Tolerance, from the arithmetic: the projection's products run on the tensor cores with bf16
operands (x exactly; dL/d(dt_mix), g_j q_j, g_j dL/dB, g_j dL/dC and g_j dt_low rounded once, each
by at most 2^-9 relative) and fp32 accumulation: mixed-precision gradients as training uses them.
A product of two rounded operands carries up to 2^-8 relative error per term; in a sum whose terms
cancel, the worst element of a field lands at several times that against the field's scale
(measured up to 2.2e-2 for ∂L/∂W_dt, whose both operands are rounded). The fields are held to
5e-2 of their scale (max |err| / (rms + |ref|)) against the exact oracle, AND the weight
gradients are checked at 2e-3 against the same products formed in the test from the oracle's
intermediates with the operands rounded to bf16 where the kernel rounds them -- which pins that
the gap to the exact oracle is that rounding and nothing else. The router's backward is fp32 SIMT
on stored inputs: 1e-4."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import swimba_backward_oracle as BO
from oracle import swimba_oracle as O
from parameter_space_moe_swimba_b200 import synth
from parameter_space_moe_swimba_b200.configs import LayerConfig
from tests.swimba_cases import make_case, oracle_route_proj, rel_rms_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

TOL_BF16_GRAD = 5e-2
TOL_ROUNDED = 2e-3


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


SHAPES = [
    # B, L, D, N, R, E, k
    (2, 64, 128, 16, 16, 4, 2),
    (1, 100, 256, 16, 32, 8, 2),   # ragged token counts per expert
    (1, 50, 64, 16, 8, 3, 1),      # top-1
    (1, 4, 64, 16, 8, 8, 2),       # experts that no token chose
]


def dev(a, dtype=np.float32):
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=dtype))).cuda()


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}L{}D{}N{}R{}E{}k{}".format(*s))
def test_proj_and_route_backward_match_the_oracle(S, shape):
    B, L, D, N, R, E, k = shape
    cfg = LayerConfig("proj_bwd", B, L, D, N, R, E, k, "bf16", "bf16", seed=13 + L)
    case = make_case(cfg, a_mode="random")
    W = case.weights64()
    T = B * L
    fw = oracle_route_proj(case, list(range(B)))
    idx = fw["idx"].reshape(T, k).astype(np.int32)
    gates = np.asarray(fw["gates"].reshape(T, k), dtype=np.float32)
    delta = np.asarray(fw["delta"].reshape(T, D), dtype=np.float32)
    rng = np.random.default_rng(L)
    g_delta = rng.standard_normal((T, D)).astype(np.float32)
    g_B = rng.standard_normal((T, N)).astype(np.float32)
    g_C = rng.standard_normal((T, N)).astype(np.float32)
    x64 = case.x64().reshape(T, D)
    # the oracle's dt_mix is softplus^-1 of the Δ the kernel reads: σ(dt_mix) = 1 - e^{-Δ}
    g_dtmix = g_delta.astype(np.float64) * -np.expm1(-delta.astype(np.float64))
    ref = BO.projection_backward(x64, idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N, g_dtmix, g_B, g_C)

    dims = S.make_dims(cfg)
    w = S.upload_weights(case.w)
    ws_w = w.struct()
    x = S.to_device(case.x, "bf16")
    f = dict(dtype=torch.float32, device="cuda")
    dx = torch.full((T, D), float("nan"), **f)
    dg = torch.full((T, k), float("nan"), **f)
    dWx = torch.full((E, D, R + 2 * N), float("nan"), **f)
    dWdt = torch.full((E, R, D), float("nan"), **f)
    db = torch.full((E, D), float("nan"), **f)
    ws = S.new_workspace(dims, S.SWIMBA_OP_PROJ_BWD)
    st = S.swimba_proj_bwd(dims, x, dev(idx, np.int32), dev(gates), ws_w, dev(delta), dev(g_delta), dev(g_B), dev(g_C),
                           dx, 0, dg, dWx, dWdt, db, ws, ws.numel())
    assert st == 0, S.swimba_status_string(st)
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(ws) == 0
    errs = {"dx": rel_rms_err(dx.cpu().numpy(), ref["dx"]), "dgates": rel_rms_err(dg.cpu().numpy(), ref["dgates"]),
            "dW_x": rel_rms_err(dWx.cpu().numpy(), ref["dW_x"]), "dW_dt": rel_rms_err(dWdt.cpu().numpy(), ref["dW_dt"]),
            "db_dt": rel_rms_err(db.cpu().numpy(), ref["db_dt"])}

    # the router's backward on its own, with the gate gradient in two parts
    g1 = rng.standard_normal((T, k)).astype(np.float32)
    g2 = rng.standard_normal((T, k)).astype(np.float32)
    rref = BO.route_backward(x64, W["W_r"], idx, g1.astype(np.float64) + g2)
    rdx = torch.full((T, D), float("nan"), **f)
    dWr = torch.full((D, E), float("nan"), **f)
    wsr = S.new_workspace(dims, S.SWIMBA_OP_ROUTE_BWD)
    assert S.swimba_route_bwd(dims, x, dev(case.w.W_r), dev(idx, np.int32), dev(gates), dev(g1), dev(g2), rdx, 0, dWr,
                              wsr, wsr.numel()) == 0
    torch.cuda.synchronize()
    errs["route_dx"] = rel_rms_err(rdx.cpu().numpy(), rref["dx"])
    errs["dW_r"] = rel_rms_err(dWr.cpu().numpy(), rref["dW_r"])
    # the weight gradients from operands rounded where the kernel rounds them (bf16, nearest even)
    bf = lambda a: synth.widen(synth.round_to(a, "bf16"), "bf16")
    pr = O.expert_projections(x64, idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N)
    G = bf(g_dtmix)
    emu_dWdt = np.zeros((E, R, D))
    emu_db = np.zeros((E, D))
    for j in range(k):
        g = gates[:, j].astype(np.float64)
        dts = bf(g[:, None] * pr["xdbl"][:, j, :R])
        gb = bf(g)
        for e in range(E):
            rows = np.nonzero(idx[:, j] == e)[0]
            emu_dWdt[e] += dts[rows].T @ G[rows]
            emu_db[e] += gb[rows] @ G[rows]
    errs["dW_dt_rounded"] = rel_rms_err(dWdt.cpu().numpy(), emu_dWdt)
    errs["db_dt_rounded"] = rel_rms_err(db.cpu().numpy(), emu_db)
    print(shape, {kk: f"{v:.2e}" for kk, v in errs.items()})
    for name in ("dx", "dgates", "dW_x", "dW_dt", "db_dt"):
        assert errs[name] <= TOL_BF16_GRAD, (name, errs[name])
    assert errs["dW_dt_rounded"] <= TOL_ROUNDED and errs["db_dt_rounded"] <= TOL_ROUNDED
    assert errs["route_dx"] <= 1e-4 and errs["dW_r"] <= 1e-4


@pytest.mark.parametrize("shape", [(2, 80, 128, 16, 16, 4, 2), (1, 64, 256, 16, 32, 8, 1)],
                         ids=lambda s: "B{}L{}D{}N{}R{}E{}k{}".format(*s))
def test_layer_backward_chain_matches_the_oracle(S, shape):
    """forward (route, mixed projection, scan) then scan_bwd -> proj_bwd (dx accumulated) ->
    route_bwd (both gate-gradient parts, dx accumulated), against the oracle's layer_backward."""
    B, L, D, N, R, E, k = shape
    cfg = LayerConfig("layer_bwd", B, L, D, N, R, E, k, "bf16", "bf16", seed=29 + L)
    case = make_case(cfg, a_mode="random", with_h0=True)
    W = case.weights64()
    g_out = synth.draw_out_grad(cfg)
    ref = BO.layer_backward(case.x64(), case.z64(), W, k, synth.widen(g_out, "bf16"),
                            h0=case.h0.astype(np.float64))

    dims = S.make_dims(cfg)
    w = S.upload_weights(case.w)
    ws_w = w.struct()
    x, z, go = S.to_device(case.x, "bf16"), S.to_device(case.z, "bf16"), S.to_device(g_out, "bf16")
    h0 = dev(case.h0)
    buf = S.LayerBuffers(dims, torch.bfloat16)
    S.layer_forward(dims, x, z, ws_w, buf, h0=h0)
    f = dict(dtype=torch.float32, device="cuda")
    dx, dz, ddelta = (torch.empty((B, L, D), **f) for _ in range(3))
    dB, dC = torch.empty((B, L, N), **f), torch.empty((B, L, N), **f)
    dg_scan, dg_proj = torch.empty((B, L, k), **f), torch.empty((B, L, k), **f)
    dA, dD, dh0 = torch.empty((E, D, N), **f), torch.empty((D,), **f), torch.empty((B, D, N), **f)
    dWx, dWdt, db = torch.empty((E, D, R + 2 * N), **f), torch.empty((E, R, D), **f), torch.empty((E, D), **f)
    dWr = torch.empty((D, E), **f)
    ws1 = S.new_workspace(dims, S.SWIMBA_OP_SCAN_BWD)
    assert S.swimba_scan_bwd(dims, x, z, buf.delta, buf.B_mix, buf.C_mix, buf.idx, buf.gates, ws_w, h0, go, dx, dz,
                             ddelta, dB, dC, dg_scan, dA, dD, dh0, ws1, ws1.numel()) == 0
    ws2 = S.new_workspace(dims, S.SWIMBA_OP_PROJ_BWD)
    assert S.swimba_proj_bwd(dims, x, buf.idx, buf.gates, ws_w, buf.delta, ddelta, dB, dC, dx, 1, dg_proj, dWx, dWdt,
                             db, ws2, ws2.numel()) == 0
    ws3 = S.new_workspace(dims, S.SWIMBA_OP_ROUTE_BWD)
    assert S.swimba_route_bwd(dims, x, ws_w.W_r, buf.idx, buf.gates, dg_scan, dg_proj, dx, 1, dWr, ws3,
                              ws3.numel()) == 0
    torch.cuda.synchronize()
    for wsb in (ws1, ws2):
        assert S.swimba_get_device_status(wsb) == 0
    got = {"dx": dx, "dz": dz, "dW_r": dWr, "dW_x": dWx, "dW_dt": dWdt, "db_dt": db, "dA": dA, "dD": dD, "dh0": dh0}
    errs = {name: rel_rms_err(t.cpu().numpy(), ref[name]) for name, t in got.items()}
    print(shape, {kk: f"{v:.2e}" for kk, v in errs.items()})
    for name, e in errs.items():
        assert e <= TOL_BF16_GRAD, (name, e)


def test_proj_bwd_rejects_bad_arguments(S):
    cfg = LayerConfig("proj_bwd_args", 1, 16, 64, 16, 8, 4, 2, "bf16", "bf16", seed=1)
    dims = S.make_dims(cfg)
    t = torch.empty(1 << 16, device="cuda")
    W = S.upload_weights(make_case(cfg).w).struct()
    ws = S.new_workspace(dims, S.SWIMBA_OP_PROJ_BWD)
    assert S.swimba_proj_bwd(dims, t, t, t, W, t, t, t, t, None, 0, t, t, t, t, ws, ws.numel()) == 1
    assert S.swimba_proj_bwd(dims, t, t, t, W, t, t, t, t, t, 0, t, t, t, t, ws, 16) == 4
    cfg32 = LayerConfig("proj_bwd_f32", 1, 16, 64, 16, 8, 4, 2, "f32", "f32", seed=1)
    d32 = S.make_dims(cfg32)
    W32 = S.upload_weights(make_case(cfg32).w).struct()
    assert S.swimba_proj_bwd(d32, t, t, t, W32, t, t, t, t, t, 0, t, t, t, t, ws, ws.numel()) == 2
