"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on the five workloads and on
edge shapes. Tolerances: router indices bit-exact; y and out within TOL*(1+|y|) with TOL = 1e-4
for fp32 activations and 2e-2 for bf16 activations with fp32 state; the state-space part of y
(y - D_skip x), which the skip term would otherwise dominate, within TOL relative to its own
scale; h_final within 1e-5 (fp32) / 1e-2 (bf16) of its scale."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import swimba_oracle as O
from oracle.conditioning import condition_router_margin
from parameter_space_moe_swimba_b200 import synth
from parameter_space_moe_swimba_b200.configs import CONFIGS, LayerConfig, dense_variant
from tests.swimba_cases import TOL_Y, make_case, oracle_layer, oracle_route_proj, rel_rms_err, scaled_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


def io_torch(cfg):
    return torch.bfloat16 if cfg.io_dtype == "bf16" else torch.float32


def run_gpu_layer(S, case, dims=None):
    cfg = case.cfg
    dims = dims or S.make_dims(cfg)
    W = S.upload_weights(case.w)
    x = S.to_device(case.x, cfg.io_dtype)
    z = S.to_device(case.z, cfg.io_dtype)
    buf = S.LayerBuffers(dims, io_torch(cfg), with_y=True)
    h0 = None if case.h0 is None else torch.from_numpy(case.h0).cuda()
    S.layer_forward(dims, x, z, W.struct(), buf, h0=h0)
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(buf.ws) == 0
    return {
        "idx": buf.idx.cpu().numpy(),
        "gates": buf.gates.cpu().numpy(),
        "delta": buf.delta.cpu().numpy(),
        "B_mix": buf.B_mix.cpu().numpy(),
        "C_mix": buf.C_mix.cpu().numpy(),
        "y": buf.y.cpu().numpy(),
        "out": buf.out.float().cpu().numpy(),
        "h_final": buf.h_final.cpu().numpy(),
    }


def check_layer(case, got, ref, rows=None, channels=None, report=None):
    cfg = case.cfg
    tol = TOL_Y[cfg.io_dtype]
    sel = (lambda a: a) if rows is None else (lambda a: a[rows])
    ch = (lambda a: a) if channels is None else (lambda a: a[..., channels])
    np.testing.assert_array_equal(sel(got["idx"]), ref["idx"])
    errs = {
        "gates": float(np.max(np.abs(sel(got["gates"]) - ref["gates"]))),
        "B_mix": rel_rms_err(sel(got["B_mix"]), ref["B_mix"]),
        "C_mix": rel_rms_err(sel(got["C_mix"]), ref["C_mix"]),
        "delta": rel_rms_err(ch(sel(got["delta"])), ref["delta"]),
        "y": scaled_err(ch(sel(got["y"])), ref["y"]),
        "out": scaled_err(ch(sel(got["out"])), ref["out"]),
    }
    x64 = case.x64(rows)
    dsk = case.w.D_skip.astype(np.float64)
    if channels is not None:
        x64, dsk = x64[..., channels], dsk[channels]
    y_ssm_ref = ref["y"] - dsk * x64
    y_ssm_got = ch(sel(got["y"])) - dsk * x64
    errs["y_ssm"] = rel_rms_err(y_ssm_got, y_ssm_ref)
    hf = sel(got["h_final"])
    if channels is not None:
        hf = hf[:, channels]
    errs["h_final"] = rel_rms_err(hf, ref["h_final"])
    if report is not None:
        report.update(errs)
    print(cfg.name, {k: f"{v:.2e}" for k, v in errs.items()})
    assert errs["gates"] <= 1e-5
    assert errs["B_mix"] <= 1e-4 and errs["C_mix"] <= 1e-4
    assert errs["delta"] <= (1e-5 if cfg.io_dtype == "f32" else 1e-2)
    assert errs["y"] <= tol and errs["out"] <= tol
    assert errs["y_ssm"] <= tol
    assert errs["h_final"] <= (1e-5 if cfg.io_dtype == "f32" else 1e-2)


# ------------------------------------------------------------------------------------------------
# the five workloads
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("with_h0", [False, True])
def test_tiny_fp32_full(S, with_h0):
    case = make_case(CONFIGS["tiny_fp32"], with_h0=with_h0)
    check_layer(case, run_gpu_layer(S, case), oracle_layer(case))


def test_mamba130m_like_full(S):
    case = make_case(CONFIGS["mamba130m_like"])
    check_layer(case, run_gpu_layer(S, case), oracle_layer(case))


def _sampled_channels(D, n, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, 1, 31, 32, D - 1], rng.choice(D, n, replace=False)]))


def check_route_proj_all_tokens(case, got):
    """Every token of every batch row: router indices bit-exact, gates, B_mix and C_mix, and Δ on
    every channel, against the oracle's routing and mixed projections."""
    cfg = case.cfg
    worst = {"gates": 0.0, "B_mix": 0.0, "C_mix": 0.0, "delta": 0.0}
    for b in range(cfg.batch):
        ref = oracle_route_proj(case, [b])
        np.testing.assert_array_equal(got["idx"][b:b + 1], ref["idx"], err_msg=f"batch row {b}")
        worst["gates"] = max(worst["gates"], float(np.max(np.abs(got["gates"][b:b + 1] - ref["gates"]))))
        for k in ("B_mix", "C_mix", "delta"):
            worst[k] = max(worst[k], rel_rms_err(got[k][b:b + 1], ref[k]))
    print(cfg.name, "all tokens", {k: f"{v:.2e}" for k, v in worst.items()})
    assert worst["gates"] <= 1e-5
    assert worst["B_mix"] <= 1e-4 and worst["C_mix"] <= 1e-4
    assert worst["delta"] <= (1e-5 if cfg.io_dtype == "f32" else 1e-2)


def test_mamba1p4b_like_full_size(S):
    """Routing and projections on all 32768 tokens; the scan on every channel of batch row 0 and
    on sampled channels of the last row."""
    cfg = CONFIGS["mamba1p4b_like"]
    case = make_case(cfg)
    got = run_gpu_layer(S, case)
    check_route_proj_all_tokens(case, got)
    check_layer(case, got, oracle_layer(case, rows=[0]), rows=[0])
    last = [cfg.batch - 1]
    ch = _sampled_channels(cfg.d_inner, 27, 11)
    check_layer(case, got, oracle_layer(case, rows=last, channels=ch), rows=last, channels=ch)


def test_mamba1p4b_like_dense_e1(S):
    cfg = dense_variant(CONFIGS["mamba1p4b_like"])
    case = make_case(cfg)
    got = run_gpu_layer(S, case)
    assert np.all(got["idx"] == 0) and np.all(got["gates"] == 1.0)
    check_route_proj_all_tokens(case, got)
    check_layer(case, got, oracle_layer(case, rows=[3]), rows=[3])


def test_long_seq_65536_full(S):
    """All 65536 tokens and all 2048 channels (the sequence is split into segments whose start
    states are carried from one to the next)."""
    cfg = CONFIGS["long_seq_65536"]
    case = make_case(cfg)
    got = run_gpu_layer(S, case)
    check_route_proj_all_tokens(case, got)
    check_layer(case, got, oracle_layer(case))


def test_decode_b256_1000_steps(S):
    """1000 consecutive decode steps on the cached state; every step's router indices and output of
    32 sequences spread over the batch, and their final state, are compared with the oracle's
    sequential run."""
    cfg = CONFIGS["decode_b256"]
    steps = cfg.decode_steps
    w = synth.draw_weights(cfg)
    Wd = S.upload_weights(w)
    ws = Wd.struct()
    dims = S.make_dims(cfg, seqlen=1)
    buf = S.LayerBuffers(dims, torch.bfloat16)
    h0 = synth.draw_h0(cfg)
    h = torch.from_numpy(h0).cuda()
    rows = np.unique(np.linspace(0, cfg.batch - 1, 32).astype(int)).tolist()
    assert len(rows) == 32
    W64 = {
        "W_r": w.W_r.astype(np.float64), "W_x": synth.widen(w.W_x, "bf16"), "W_dt": synth.widen(w.W_dt, "bf16"),
        "b_dt": w.b_dt.astype(np.float64), "A": w.A.astype(np.float64), "D_skip": w.D_skip.astype(np.float64),
    }
    h_ref = h0[rows].astype(np.float64)
    worst = {"out": 0.0}
    for s in range(steps):
        x, z = synth.draw_step_activations(cfg, s)
        condition_router_margin(x, lambda a: synth.widen(a, "bf16"), w.W_r, cfg.top_k,
                                lambda b, t, a: synth.redraw_x_row(cfg, b, t, a, step=s))
        xd = S.to_device(x, "bf16")
        zd = S.to_device(z, "bf16")
        S.decode_step(dims, xd, zd, ws, buf, h)
        out_ref, h_ref, r = O.decode_step(h_ref, synth.widen(x[rows], "bf16"), synth.widen(z[rows], "bf16"), W64,
                                          cfg.top_k)
        np.testing.assert_array_equal(buf.idx.cpu().numpy()[rows], r["idx"])
        e = scaled_err(buf.out.float().cpu().numpy()[rows], out_ref)
        worst["out"] = max(worst["out"], e)
        assert e <= TOL_Y["bf16"], (s, e)
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(buf.ws) == 0
    eh = rel_rms_err(h.cpu().numpy()[rows], h_ref)
    print("decode_b256", worst, "h_final", eh)
    assert eh <= 1e-2


# ------------------------------------------------------------------------------------------------
# edge shapes
# ------------------------------------------------------------------------------------------------

EDGE = [
    # B, L, D, N, R, E, k, io, w
    (3, 37, 40, 5, 3, 3, 3, "f32", "f32"),     # ragged channel tile, N < 16, k = E (dynamic k)
    (1, 1, 8, 16, 1, 1, 1, "f32", "f32"),      # a single token, one expert
    (2, 19, 264, 16, 16, 16, 16, "bf16", "bf16"),  # every expert active, ragged D tile
    (2, 33, 96, 16, 8, 6, 3, "bf16", "f32"),   # bf16 activations with fp32 tables, k = 3
    (5, 3, 48, 1, 2, 2, 1, "f32", "bf16"),     # scalar state
    (1, 300, 64, 16, 4, 4, 2, "bf16", "bf16"),
    # shapes on the tensor-core projection path (bf16, k <= 2, N = 16, R % 16 == 0, D % 64 == 0)
    (3, 77, 128, 16, 16, 4, 2, "bf16", "bf16"),    # R + 2N = 48
    (2, 50, 192, 16, 48, 8, 2, "bf16", "bf16"),    # R = 48, a partial 256-column chunk
    (1, 200, 320, 16, 64, 5, 1, "bf16", "bf16"),   # top-1, D = 256 + 64
    (4, 129, 256, 16, 128, 6, 2, "bf16", "bf16"),  # R = 128, many ragged tiles
    (2, 1000, 128, 16, 32, 3, 2, "bf16", "bf16"),  # several full tiles per expert pair
    # tensor-core router shapes (bf16 x, D % 64 == 0, E % 4 == 0, more than 2048 tokens): E = 12
    # and E = 16, a ragged last token tile
    (3, 700, 128, 16, 16, 12, 2, "bf16", "bf16"),
    (1, 2100, 64, 16, 16, 16, 1, "bf16", "bf16"),
    # the SIMT tile router for more than 2048 tokens (E % 4 != 0; fp32 x)
    (1, 2100, 96, 16, 8, 6, 3, "bf16", "f32"),
    (1, 2100, 40, 5, 3, 3, 3, "f32", "f32"),
    # k = 2 with at most 1024 tokens runs the projection on (token, slot) pairs bucketed by single
    # expert: both sides of that limit
    (1, 1024, 64, 16, 16, 4, 2, "bf16", "bf16"),
    (1, 1025, 64, 16, 16, 4, 2, "bf16", "bf16"),
    # the one-CTA bucketing of the tensor-core projection covers up to 4096 tokens: both sides of it
    (2, 2048, 64, 16, 16, 4, 2, "bf16", "bf16"),
    (1, 4097, 64, 16, 16, 8, 1, "bf16", "bf16"),
    # the fast scan (bf16, N = 16, k <= 2, D % 16 == 0): one token and one 16-channel warp tile;
    # E = 16 (the widest TMEM window) with a 1-token last segment; hundreds of 16-token segments
    # chained by the carry pass (ragged last segment); E = 1; many sequences, no segments, a
    # ragged last chunk
    (1, 1, 16, 16, 16, 2, 1, "bf16", "bf16"),
    (2, 17, 48, 16, 16, 16, 2, "bf16", "bf16"),
    (3, 4111, 32, 16, 16, 5, 2, "bf16", "bf16"),
    (1, 5000, 16, 16, 16, 1, 1, "bf16", "bf16"),
    (64, 40, 512, 16, 32, 8, 1, "bf16", "bf16"),
]


@pytest.mark.parametrize("shape", EDGE, ids=lambda s: "B{}L{}D{}N{}R{}E{}k{}{}{}".format(*s))
@pytest.mark.parametrize("with_h0", [False, True])
def test_edge_shapes(S, shape, with_h0):
    B, L, D, N, R, E, k, io, wd = shape
    cfg = LayerConfig("edge", B, L, D, N, R, E, k, io, wd, seed=21, cached_state=with_h0)
    case = make_case(cfg, a_mode="random", with_h0=with_h0, margin=1e-3)
    check_layer(case, run_gpu_layer(S, case), oracle_layer(case))


@pytest.mark.parametrize("name", ["mamba130m_like", "tiny_fp32"])
def test_layer_is_deterministic(S, name):
    """Two runs give bitwise equal results: the token bucketing is a stable counting sort (the slot
    order does not depend on scheduling) and every output row depends only on its own token."""
    cfg = CONFIGS[name]
    if cfg.batch * cfg.seqlen > 4096:
        cfg = cfg.with_(batch=2, seqlen=1024)
    case = make_case(cfg)
    a, b = run_gpu_layer(S, case), run_gpu_layer(S, case)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_exact_router_ties_go_to_the_lower_index(S, io):
    """f32, 100 tokens: the one-CTA-per-token router; bf16, 2200 tokens (D = 128, E = 8): the
    tensor-core router, whose tied B columns get bitwise equal partial logits."""
    if io == "f32":
        cfg = LayerConfig("ties", 2, 50, 64, 16, 4, 6, 2, "f32", "f32", seed=5)
    else:
        cfg = LayerConfig("ties", 2, 1100, 128, 16, 16, 8, 2, "bf16", "bf16", seed=5)
    case = make_case(cfg, condition=False)
    case.w.W_r[:, 3] = case.w.W_r[:, 1]  # experts 1 and 3 always tie (same fp32 sums on both sides)
    case.w.W_r[:, 5] = case.w.W_r[:, 0]
    got = run_gpu_layer(S, case)
    ref = oracle_layer(case)
    np.testing.assert_array_equal(got["idx"], ref["idx"])
    # a tied pair is never ordered (higher, lower)
    for a, b in [(1, 3), (0, 5)]:
        assert not np.any((got["idx"][..., 0] == b) & (got["idx"][..., 1] == a))


def test_prefill_split_and_steps_continue_the_state(S):
    cfg = LayerConfig("split", 2, 24, 96, 16, 8, 4, 2, "f32", "f32", seed=9)
    case = make_case(cfg, with_h0=True)
    dims = S.make_dims(cfg)
    W = S.upload_weights(case.w)
    ws = W.struct()
    x = S.to_device(case.x, "f32")
    z = S.to_device(case.z, "f32")
    h0 = torch.from_numpy(case.h0).cuda()
    full = S.LayerBuffers(dims, torch.float32)
    S.layer_forward(dims, x, z, ws, full, h0=h0)
    L1 = 10
    d1, d2 = S.make_dims(cfg, seqlen=L1), S.make_dims(cfg, seqlen=cfg.seqlen - L1)
    a, b = S.LayerBuffers(d1, torch.float32), S.LayerBuffers(d2, torch.float32)
    S.layer_forward(d1, x[:, :L1].contiguous(), z[:, :L1].contiguous(), ws, a, h0=h0)
    S.layer_forward(d2, x[:, L1:].contiguous(), z[:, L1:].contiguous(), ws, b, h0=a.h_final)
    torch.testing.assert_close(torch.cat([a.out, b.out], 1), full.out, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(b.h_final, full.h_final, rtol=1e-5, atol=1e-6)
    # token by token through swimba_step
    d_step = S.make_dims(cfg, seqlen=1)
    st = S.LayerBuffers(d_step, torch.float32)
    h = h0.clone()
    outs = []
    for t in range(cfg.seqlen):
        S.decode_step(d_step, x[:, t:t + 1].contiguous(), z[:, t:t + 1].contiguous(), ws, st, h)
        outs.append(st.out.clone())
    torch.testing.assert_close(torch.cat(outs, 1), full.out, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(h, full.h_final, rtol=1e-5, atol=1e-6)


def test_scan_alone_on_oracle_streams(S):
    """swimba_scan_fwd fed with the oracle's routing and mixed streams (rounded to fp32)."""
    cfg = CONFIGS["mamba130m_like"].with_(batch=2, seqlen=333)
    case = make_case(cfg, a_mode="random", with_h0=True)
    ref = oracle_layer(case)
    dims = S.make_dims(cfg)
    W = S.upload_weights(case.w)
    f = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()
    out = torch.empty((cfg.batch, cfg.seqlen, cfg.d_inner), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((cfg.batch, cfg.seqlen, cfg.d_inner), dtype=torch.float32, device="cuda")
    hf = torch.empty((cfg.batch, cfg.d_inner, cfg.d_state), dtype=torch.float32, device="cuda")
    ws = S.new_workspace(dims)
    S.check(S.swimba_scan_fwd(dims, S.to_device(case.x, "bf16"), S.to_device(case.z, "bf16"), f(ref["delta"]),
                              f(ref["B_mix"]), f(ref["C_mix"]), f(ref["idx"], torch.int32), f(ref["gates"]),
                              W.struct(), f(case.h0), out, hf, y, ws, ws.numel()))
    torch.cuda.synchronize()
    assert scaled_err(y.cpu().numpy(), ref["y"]) <= 1e-4
    assert rel_rms_err(hf.cpu().numpy(), ref["h_final"]) <= 1e-4


def test_bad_arguments_are_rejected_before_launch(S):
    cfg = CONFIGS["tiny_fp32"]
    dims = S.make_dims(cfg)
    W = S.upload_weights(synth.draw_weights(cfg))
    x = torch.zeros((1, 128, 128), device="cuda")
    idx = torch.empty((1, 128, 1), dtype=torch.int32, device="cuda")
    g = torch.empty((1, 128, 1), device="cuda")
    assert S.swimba_route(dims, None, W.W_r, idx, g) == 1
    assert S.swimba_route(dims, x.data_ptr() + 4, W.W_r, idx, g) == 3
    bad = S.make_dims(cfg, top_k=5)
    assert S.swimba_route(bad, x, W.W_r, idx, g) == 1
    ws = S.new_workspace(dims)
    d = torch.empty((1, 128, 128), device="cuda")
    bc = torch.empty((1, 128, 16), device="cuda")
    assert S.swimba_mixed_proj(dims, x, idx, g, W.struct(), d, bc, bc, ws, 16) == 4
    assert S.swimba_get_device_status(ws) == 0


@pytest.mark.parametrize("shape", [
    (2, 333, 1536, 16, 48, 8, 2, "bf16", "bf16"),  # fast path, several segments per sequence
    (8, 300, 4096, 16, 128, 8, 2, "bf16", "bf16"),  # fast path, no segments
    (2, 45, 40, 5, 3, 3, 3, "f32", "f32"),          # generic path
], ids=lambda s: "B{}L{}D{}N{}R{}E{}k{}{}{}".format(*s))
def test_zoh_scan_on_oracle_streams(S, shape):
    """swimba_scan_fwd_zoh fed with the oracle's routing and mixed streams, against the oracle's
    scan with the zero-order-hold injection; the Euler scan on the same streams differs from it."""
    B, L, D, N, R, E, k, io, wd = shape
    cfg = LayerConfig("zoh", B, L, D, N, R, E, k, io, wd, seed=17, cached_state=True)
    case = make_case(cfg, a_mode="random", with_h0=True)
    W = case.weights64()
    ref = oracle_layer(case, channels=None)
    y_z, out_z, h_z, _ = O.selective_scan(case.x64(), case.z64(), ref["dt_mix"], ref["B_mix"], ref["C_mix"],
                                          ref["idx"], ref["gates"], W["A"], W["D_skip"], h0=case.h0,
                                          injection="zoh")
    dims = S.make_dims(cfg)
    Wd = S.upload_weights(case.w)
    f = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()
    io_t = torch.bfloat16 if io == "bf16" else torch.float32
    out = torch.empty((B, L, D), dtype=io_t, device="cuda")
    y = torch.empty((B, L, D), dtype=torch.float32, device="cuda")
    hf = torch.empty((B, D, N), dtype=torch.float32, device="cuda")
    ws = S.new_workspace(dims)
    S.check(S.swimba_scan_fwd_zoh(dims, S.to_device(case.x, io), S.to_device(case.z, io), f(ref["delta"]),
                                  f(ref["B_mix"]), f(ref["C_mix"]), f(ref["idx"], torch.int32), f(ref["gates"]),
                                  Wd.struct(), f(case.h0), out, hf, y, ws, ws.numel()), "scan_fwd_zoh")
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(ws) == 0
    tol = 1e-4
    ey = scaled_err(y.cpu().numpy(), y_z)
    ess = rel_rms_err(y.cpu().numpy() - W["D_skip"] * case.x64(), y_z - W["D_skip"] * case.x64())
    eh = rel_rms_err(hf.cpu().numpy(), h_z)
    eo = scaled_err(out.float().cpu().numpy(), out_z)
    print(shape, {"y": ey, "y_ssm": ess, "h_final": eh, "out": eo})
    assert ey <= tol and ess <= tol and eh <= tol
    assert eo <= (1e-4 if io == "f32" else TOL_Y["bf16"])
    # the two injections are different discretisations
    assert rel_rms_err(ref["h_final"], h_z) > 10 * tol
