"""The scan's backward pass through the C ABI (swimba_scan_bwd) against the fp64 backward oracle
(oracle/swimba_backward_oracle.py, pinned by finite differences of the forward oracle) on the same
stored inputs: the scan inputs are the oracle's routing and mixed projections of the synthetic
layer (stored as the library stores them: Δ, B_mix, C_mix, gates fp32), g_out ~ N(0, 1) in the io
dtype.

Tolerance, from the arithmetic: the kernel runs in fp32 with the special-function unit's exp2
(relative error about 2^-22) on inputs both sides read exactly, so each per-element gradient
(dx, dz, dΔ, dh0) carries fp32 rounding of a short chain plus the adjoint recurrence's sum over the
tokens after it (decaying): 1e-4 of the field's scale leaves a margin of 10-100 over what that
gives. The reduced gradients sum many terms in fp32 -- dB, dC and dgates over D channels (and N
states), dA and dD over B L tokens -- and are held to 1e-3 of their scale."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import swimba_backward_oracle as BO
from parameter_space_moe_swimba_b200 import synth
from parameter_space_moe_swimba_b200.configs import LayerConfig
from tests.swimba_cases import make_case, oracle_route_proj, rel_rms_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


SHAPES = [
    # B, L, D, N, R, E, k, io, h0
    (2, 50, 64, 16, 8, 8, 2, "bf16", True),    # ragged last chunk (3 x 16 + 2), one channel tile
    (1, 33, 136, 16, 8, 4, 1, "f32", False),   # ragged channel tile (136 = 2 x 64 + 8), top-1
    (2, 40, 72, 5, 3, 6, 3, "f32", True),      # N = 5 < 16, k = 3
    (3, 1, 16, 16, 4, 4, 2, "bf16", True),     # one token
    (2, 300, 256, 16, 16, 8, 2, "bf16", True),  # several chunks and tiles
    (1, 45, 208, 16, 8, 4, 1, "f32", True),    # packed layout, last tile one warp wide (208 = 3 x 64 + 16)
    (2, 50, 72, 16, 8, 8, 2, "bf16", False),   # N = 16, k = 2 but D % 16 != 0: the one-channel layout
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}L{}D{}N{}R{}E{}k{}{}h{}".format(*s))
def test_scan_backward_matches_the_oracle(S, shape):
    B, L, D, N, R, E, k, io, with_h0 = shape
    cfg = LayerConfig("scan_bwd", B, L, D, N, R, E, k, io, io, seed=71 + L)
    case = make_case(cfg, a_mode="random", with_h0=with_h0)
    ref_in = oracle_route_proj(case, list(range(B)))
    W = case.weights64()
    f32 = lambda a: np.asarray(a, dtype=np.float32)
    delta, Bm, Cm, gates = f32(ref_in["delta"]), f32(ref_in["B_mix"]), f32(ref_in["C_mix"]), f32(ref_in["gates"])
    idx = ref_in["idx"].astype(np.int32)
    g_out = synth.draw_out_grad(cfg)
    h0 = case.h0
    ref = BO.scan_backward(case.x64(), case.z64(), delta, Bm, Cm, idx, gates, W["A"], W["D_skip"],
                           synth.widen(g_out, io), h0=None if h0 is None else h0.astype(np.float64))

    dims = S.make_dims(cfg)
    Wd = S.upload_weights(case.w)
    ws_w = Wd.struct()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    x, z, go = S.to_device(case.x, io), S.to_device(case.z, io), S.to_device(g_out, io)
    f = dict(dtype=torch.float32, device="cuda")
    out = {name: torch.full(shp, float("nan"), **f) for name, shp in [
        ("dx", (B, L, D)), ("dz", (B, L, D)), ("ddelta", (B, L, D)), ("dB", (B, L, N)), ("dC", (B, L, N)),
        ("dgates", (B, L, k)), ("dA", (E, D, N)), ("dD", (D,)), ("dh0", (B, D, N))]}
    ws = S.new_workspace(dims, S.SWIMBA_OP_SCAN_BWD)
    st = S.swimba_scan_bwd(dims, x, z, dev(delta), dev(Bm), dev(Cm), dev(idx), dev(gates), ws_w,
                           None if h0 is None else dev(h0), go, out["dx"], out["dz"], out["ddelta"], out["dB"],
                           out["dC"], out["dgates"], out["dA"], out["dD"], out["dh0"], ws, ws.numel())
    assert st == 0, S.swimba_status_string(st)
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(ws) == 0
    errs = {name: rel_rms_err(t.cpu().numpy(), ref[name]) for name, t in out.items()}
    print(shape, {kk: f"{v:.2e}" for kk, v in errs.items()})
    for name in ("dx", "dz", "ddelta", "dh0"):
        assert errs[name] <= 1e-4, (name, errs[name])
    for name in ("dB", "dC", "dgates", "dA", "dD"):
        assert errs[name] <= 1e-3, (name, errs[name])


def test_scan_backward_is_deterministic(S):
    cfg = LayerConfig("scan_bwd_det", 2, 100, 128, 16, 8, 4, 2, "bf16", "bf16", seed=5)
    case = make_case(cfg, a_mode="random")
    ref_in = oracle_route_proj(case, [0, 1])
    dims = S.make_dims(cfg)
    ws_w = S.upload_weights(case.w).struct()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float32))).cuda()
    args = (S.to_device(case.x, "bf16"), S.to_device(case.z, "bf16"), dev(ref_in["delta"]), dev(ref_in["B_mix"]),
            dev(ref_in["C_mix"]), torch.from_numpy(ref_in["idx"].astype(np.int32)).cuda(), dev(ref_in["gates"]), ws_w,
            None, S.to_device(synth.draw_out_grad(cfg), "bf16"))
    runs = []
    for _ in range(2):
        o = [torch.empty(s, dtype=torch.float32, device="cuda") for s in
             [(2, 100, 128)] * 3 + [(2, 100, 16)] * 2 + [(2, 100, 2), (4, 128, 16), (128,)]]
        ws = S.new_workspace(dims, S.SWIMBA_OP_SCAN_BWD)
        assert S.swimba_scan_bwd(dims, *args, *o, None, ws, ws.numel()) == 0
        torch.cuda.synchronize()
        runs.append(o)
    for a, b in zip(*runs):
        assert torch.equal(a, b)


def test_scan_backward_rejects_bad_arguments(S):
    cfg = LayerConfig("scan_bwd_args", 1, 16, 32, 16, 8, 4, 2, "bf16", "bf16", seed=1)
    dims = S.make_dims(cfg)
    t = torch.empty(4096, device="cuda")
    W = S.upload_weights(make_case(cfg).w).struct()
    ws = S.new_workspace(dims, S.SWIMBA_OP_SCAN_BWD)
    full = [t] * 7
    outs = [t] * 8
    assert S.swimba_scan_bwd(dims, *full, W, None, None, *outs, None, ws, ws.numel()) == 1  # g_out missing
    assert S.swimba_scan_bwd(dims, *full, W, None, t, *outs, None, ws, 16) == 4
    assert S.swimba_scan_bwd(dims, *full, W, None, t, *outs, t.data_ptr() + 4, ws, ws.numel()) == 3
    assert S.swimba_scan_bwd(dims, *full, W, None, t, t.data_ptr() + 8, *outs[1:], None, ws, ws.numel()) == 3
    bad_b = [t, t, t, t.data_ptr() + 4, t, t, t]  # B_mix off its 16-byte boundary
    assert S.swimba_scan_bwd(dims, *bad_b, W, None, t, *outs, None, ws, ws.numel()) == 3
