"""The entry points allocate nothing and never synchronise, so a serving loop can capture them in a
CUDA graph: the decode step (route -> mixed projection -> state step) and the whole-sequence layer
(route -> mixed projection -> scan) are captured once and replayed, and every output equals the
eager calls' bit for bit (the kernels are deterministic)."""
from __future__ import annotations

import pytest

from parameter_space_moe_swimba_b200 import synth
from parameter_space_moe_swimba_b200.configs import CONFIGS

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


def capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
        fn(torch.cuda.current_stream())
    torch.cuda.synchronize()
    return g


def test_decode_step_replays_as_a_graph(S):
    cfg = CONFIGS["decode_b256"]
    w = S.upload_weights(synth.draw_weights(cfg))
    ws = w.struct()
    dims = S.make_dims(cfg, seqlen=1)
    h0 = torch.from_numpy(synth.draw_h0(cfg)).cuda()
    eager = S.LayerBuffers(dims, torch.bfloat16)
    graphed = S.LayerBuffers(dims, torch.bfloat16)
    x, z = synth.draw_step_activations(cfg, 0)
    xd, zd = S.to_device(x, "bf16"), S.to_device(z, "bf16")
    h_e, h_g = h0.clone(), h0.clone()
    g = capture(lambda s: S.decode_step(dims, xd, zd, ws, graphed, h_g, s))
    h_g.copy_(h0)
    for step in range(3):  # the state evolves through the replays
        S.decode_step(dims, xd, zd, ws, eager, h_e)
        g.replay()
        torch.cuda.synchronize()
        for name in ("idx", "gates", "delta", "B_mix", "C_mix", "out"):
            assert torch.equal(getattr(eager, name), getattr(graphed, name)), (step, name)
        assert torch.equal(h_e, h_g), step
    assert S.swimba_get_device_status(graphed.ws) == 0
    del g


def test_layer_forward_replays_as_a_graph(S):
    cfg = CONFIGS["mamba130m_like"].with_(batch=2, seqlen=512)
    w = S.upload_weights(synth.draw_weights(cfg))
    ws = w.struct()
    dims = S.make_dims(cfg)
    x, z = synth.draw_activations(cfg)
    xd, zd = S.to_device(x, cfg.io_dtype), S.to_device(z, cfg.io_dtype)
    eager = S.LayerBuffers(dims, torch.bfloat16)
    graphed = S.LayerBuffers(dims, torch.bfloat16)
    S.layer_forward(dims, xd, zd, ws, eager)
    g = capture(lambda s: S.layer_forward(dims, xd, zd, ws, graphed, stream=s))
    g.replay()
    torch.cuda.synchronize()
    for name in ("idx", "gates", "delta", "B_mix", "C_mix", "out", "h_final"):
        assert torch.equal(getattr(eager, name), getattr(graphed, name)), name
    assert S.swimba_get_device_status(graphed.ws) == 0
    del g
