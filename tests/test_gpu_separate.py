"""The MoE of separate SSMs (one state trajectory per expert, the design the pages set against
Swimba) through the C ABI, against the fp64 oracle's ``separate_ssm_moe``: router indices bit-exact,
the per-slot streams of swimba_separate_proj, and y, out and every expert's final state of
swimba_separate_scan, on the tensor-memory path (bf16, N = 16, k <= 2, E <= 8) and the SIMT path."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import swimba_oracle as O
from parameter_space_moe_swimba_b200.configs import LayerConfig
from tests.swimba_cases import TOL_Y, make_case, rel_rms_err, scaled_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


SHAPES = [
    # B, L, D, N, R, E, k, io, w
    (2, 100, 64, 16, 16, 8, 2, "bf16", "bf16"),   # tensor-memory path, a ragged last chunk
    (3, 33, 48, 16, 8, 4, 1, "bf16", "bf16"),     # top-1
    (1, 40, 32, 16, 16, 3, 2, "bf16", "bf16"),    # E = 3
    (2, 29, 40, 5, 3, 5, 3, "f32", "f32"),        # SIMT path: fp32, N = 5, k = 3
    (1, 21, 24, 16, 4, 12, 2, "bf16", "f32"),     # SIMT path: E = 12 > 8
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}L{}D{}N{}R{}E{}k{}{}{}".format(*s))
def test_separate_ssm_moe_matches_the_oracle(S, shape):
    B, L, D, N, R, E, k, io, wd = shape
    cfg = LayerConfig("separate", B, L, D, N, R, E, k, io, wd, seed=41)
    case = make_case(cfg, a_mode="random")
    W = case.weights64()
    x64, z64 = case.x64(), case.z64()
    idx, gates, _ = O.route(x64.reshape(-1, D), W["W_r"], k)
    pr = O.expert_projections(x64.reshape(-1, D), idx, gates, W["W_x"], W["W_dt"], W["b_dt"], R, N)
    dt_j = pr["dt_j"].reshape(B, L, k, D)
    xdbl = pr["xdbl"].reshape(B, L, k, R + 2 * N)
    B_j, C_j = xdbl[..., R:R + N], xdbl[..., R + N:]
    h0 = np.random.default_rng(5).standard_normal((E, B, D, N)) * 0.3
    y_ref, out_ref, h_ref = O.separate_ssm_moe(x64, z64, dt_j, B_j, C_j, idx.reshape(B, L, k),
                                               gates.reshape(B, L, k), W["A"], W["D_skip"], h0=h0)

    dims = S.make_dims(cfg)
    Wd = S.upload_weights(case.w)
    ws = Wd.struct()
    io_t = torch.bfloat16 if io == "bf16" else torch.float32
    x = S.to_device(case.x, io)
    z = S.to_device(case.z, io)
    f32 = dict(dtype=torch.float32, device="cuda")
    idx_d = torch.empty((B, L, k), dtype=torch.int32, device="cuda")
    g_d = torch.empty((B, L, k), **f32)
    dj = torch.empty((B, L, k, D), **f32)
    bj = torch.empty((B, L, k, N), **f32)
    cj = torch.empty((B, L, k, N), **f32)
    out = torch.empty((B, L, D), dtype=io_t, device="cuda")
    y = torch.empty((B, L, D), **f32)
    hf = torch.empty((E, B, D, N), **f32)
    wsb = S.new_workspace(dims, S.SWIMBA_OP_SEPARATE)
    S.check(S.swimba_route(dims, x, ws.W_r, idx_d, g_d), "route")
    S.check(S.swimba_separate_proj(dims, x, idx_d, g_d, ws, dj, bj, cj), "separate_proj")
    S.check(S.swimba_separate_scan(dims, x, z, dj, bj, cj, idx_d, g_d, ws, torch.from_numpy(h0).float().cuda(), out,
                                   hf, y, wsb, wsb.numel()), "separate_scan")
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(wsb) == 0
    np.testing.assert_array_equal(idx_d.cpu().numpy(), idx.reshape(B, L, k))
    sp = O.softplus(dt_j)
    errs = {
        "delta_j": rel_rms_err(dj.cpu().numpy(), sp),
        "B_j": rel_rms_err(bj.cpu().numpy(), B_j),
        "C_j": rel_rms_err(cj.cpu().numpy(), C_j),
        "y": scaled_err(y.cpu().numpy(), y_ref),
        "out": scaled_err(out.float().cpu().numpy(), out_ref),
        "y_ssm": rel_rms_err(y.cpu().numpy() - case.w.D_skip * x64, y_ref - W["D_skip"] * x64),
        "h_final": rel_rms_err(hf.cpu().numpy(), h_ref),
    }
    print(shape, {kk: f"{v:.2e}" for kk, v in errs.items()})
    tol = TOL_Y[io]
    assert errs["delta_j"] <= 1e-5 and errs["B_j"] <= 1e-5 and errs["C_j"] <= 1e-5
    assert errs["y"] <= tol and errs["out"] <= tol and errs["y_ssm"] <= tol
    assert errs["h_final"] <= (1e-5 if io == "f32" else 1e-2)


def test_separate_scan_rejects_bad_arguments(S):
    cfg = LayerConfig("separate", 1, 16, 32, 16, 16, 4, 2, "bf16", "bf16", seed=1)
    dims = S.make_dims(cfg)
    t = torch.empty(1024, device="cuda")
    W = S.upload_weights(make_case(cfg).w).struct()
    wsb = S.new_workspace(dims, S.SWIMBA_OP_SEPARATE)
    assert S.swimba_separate_scan(dims, t, t, t, t, t, t, t, W, None, None, None, None, wsb, wsb.numel()) == 1
    assert S.swimba_separate_scan(dims, t, t, t, t, t, t, t, W, None, t, None, None, wsb, 8) == 4
    assert S.swimba_separate_scan(dims, t.data_ptr() + 4, t, t, t, t, t, t, W, None, t, None, None, wsb,
                                  wsb.numel()) == 3
    assert S.swimba_separate_proj(dims, None, t, t, W, t, t, t) == 1
