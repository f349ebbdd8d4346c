"""swimba_scan_fwd_noalloc: the scan for callers that cannot allocate device memory (a plugin inside a
framework that owns all device memory and offers it no allocator, or a latency-critical loop that
must not call cudaMalloc). It must give the same results as swimba_scan_fwd with a caller
workspace, call after call, on a shape whose scan splits sequences into segments (so the fixed
scratch really holds the segment carries), and refuse shapes whose scratch would not fit."""
import numpy as np
import pytest

from parameter_space_moe_swimba_b200 import synth
from parameter_space_moe_swimba_b200.configs import CONFIGS, LayerConfig

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


def test_noalloc_scan_equals_workspace_scan_on_two_calls(S):
    cfg = CONFIGS["mamba130m_like"]
    dims = S.make_dims(cfg)
    assert S.swimba_workspace_size(dims, S.SWIMBA_OP_SCAN) > 256  # this shape uses scratch
    w = synth.draw_weights(cfg)
    x, z = synth.draw_activations(cfg)
    W = S.upload_weights(w)
    ws = W.struct()
    xd, zd = S.to_device(x, "bf16"), S.to_device(z, "bf16")
    buf = S.LayerBuffers(dims, torch.bfloat16, with_y=True)
    h0 = torch.from_numpy(synth.draw_h0(cfg.with_(cached_state=True))).cuda()
    S.check(S.swimba_route(dims, xd, W.W_r, buf.idx, buf.gates), "route")
    S.check(S.swimba_mixed_proj(dims, xd, buf.idx, buf.gates, ws, buf.delta, buf.B_mix, buf.C_mix, buf.ws,
                                buf.ws.numel()), "proj")
    S.check(S.swimba_scan_fwd(dims, xd, zd, buf.delta, buf.B_mix, buf.C_mix, buf.idx, buf.gates, ws, h0, buf.out,
                              buf.h_final, buf.y, buf.ws, buf.ws.numel()), "scan")
    torch.cuda.synchronize()
    ref = (buf.out.float().cpu().numpy(), buf.y.cpu().numpy(), buf.h_final.cpu().numpy())
    for _ in range(2):
        out = torch.empty_like(buf.out)
        y = torch.empty_like(buf.y)
        hf = torch.empty_like(buf.h_final)
        S.check(S.swimba_scan_fwd_noalloc(dims, xd, zd, buf.delta, buf.B_mix, buf.C_mix, buf.idx, buf.gates, ws, h0,
                                          out, hf, y), "scan_noalloc")
        torch.cuda.synchronize()
        got = (out.float().cpu().numpy(), y.cpu().numpy(), hf.cpu().numpy())
        for a, b in zip(got, ref):
            np.testing.assert_allclose(a, b, rtol=1e-5, atol=1e-6)


def test_noalloc_scan_refuses_a_shape_whose_scratch_does_not_fit(S):
    # one wide sequence: when its channels alone cannot fill the GPU the scan splits it into
    # segments, whose carries need 3 x S x D x 16 floats; the width that exceeds the 8 MiB array
    # depends on the SM count, so it is searched for
    L = 256
    found = None
    for D in (4096, 8192, 12288, 16384, 18432, 24576, 32768, 49152):
        cfg = LayerConfig("wide", 1, L, D, 16, 16, 8, 2, "bf16", "bf16", seed=3)
        if S.swimba_workspace_size(S.make_dims(cfg), S.SWIMBA_OP_SCAN) > (8 << 20):
            found = cfg
            break
    if found is None:
        pytest.skip("no single-sequence shape on this GPU needs more than the fixed scratch")
    cfg, D = found, found.d_inner
    dims = S.make_dims(cfg)
    dev = dict(device="cuda")
    x = torch.zeros((1, L, D), dtype=torch.bfloat16, **dev)
    f = lambda *shape: torch.zeros(shape, dtype=torch.float32, **dev)
    idx = torch.zeros((1, L, 2), dtype=torch.int32, **dev)
    w = synth.draw_weights(cfg.with_(d_inner=64))  # tables are never read: the call stops first
    W = S.upload_weights(w)
    st = S.swimba_scan_fwd_noalloc(dims, x, x, f(1, L, D), f(1, L, 16), f(1, L, 16), idx, f(1, L, 2),
                                   W.struct(), None, torch.empty_like(x), None, None)
    assert st == 4  # SWIMBA_ERR_WORKSPACE
    assert "fixed array holds" in S.swimba_last_error_string()


def test_noalloc_status_reports_a_wait_that_gave_up(S):
    """A bounded wait that runs out on the fixed array's status block is reported by
    swimba_scan_fwd_noalloc_status (then cleared), and the next call works."""
    block = S.swimba_scan_fwd_noalloc_status_block()
    assert block
    assert S.swimba_check_wait_timeout(block, 256, 20_000_000) == 0
    assert S.swimba_scan_fwd_noalloc_status() == 6  # SWIMBA_ERR_TIMEOUT
    assert S.swimba_scan_fwd_noalloc_status() == 0  # cleared
    test_noalloc_scan_equals_workspace_scan_on_two_calls(S)
    assert S.swimba_scan_fwd_noalloc_status() == 0
