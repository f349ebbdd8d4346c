"""Swimba on the Mamba-2 SSD form through the C ABI (swimba_ssd_scan: chunks of 128 tokens on the
tcgen05 tensor cores) against the fp64 oracle's sequential recurrence and its chunked (SSD) form
on the same bf16 inputs: y within the layer's bf16 bound 2e-2 (1 + |y|). The operands the kernel
makes itself (the carried state's copy, W, X_w) enter the MMAs as bf16 hi + lo pairs (about 16
significant bits) with fp32 accumulation, so the result is held to fp32-like bounds as well: y and
its state-space part within 1e-3 of their scale and the final state within 1e-3 of its scale (a
single bf16 copy of those operands gives about 2e-2 and 1e-2 here); ragged last chunks, one token,
and a start state."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import swimba_ssd_oracle as SSD
from parameter_space_moe_swimba_b200 import synth
from tests.swimba_cases import rel_rms_err, scaled_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


def run_gpu(S, inp, with_s0):
    B, L, _, H, P = inp.X.shape
    N = inp.B.shape[-1]
    dims = S.swimba_ssd_dims(batch=B, seqlen=L, n_heads=H, head_dim=P, d_state=N, top_k=1)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    X = S.to_device(inp.X, "bf16")
    Bm = S.to_device(inp.B, "bf16")
    C = S.to_device(inp.C_mix, "bf16")
    y = torch.empty((B, L, H, P), dtype=torch.float32, device="cuda")
    sf = torch.empty((B, H, P, N), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    S.check(S.swimba_ssd_scan(dims, X, Bm, C, t(inp.gates), t(inp.delta), t(inp.A), t(inp.D_skip),
                              t(inp.S0) if with_s0 else None, y, sf, ws, ws.numel()), "swimba_ssd_scan")
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(ws) == 0
    return y.cpu().numpy(), sf.cpu().numpy()


def oracle(inp, with_s0, chunked):
    B = inp.X.shape[0]
    ys, ss = [], []
    for b in range(B):
        args = (synth.widen(inp.X[b], "bf16"), synth.widen(inp.B[b], "bf16"),
                synth.widen(inp.C_mix[b], "bf16")[:, None, :], inp.gates[b].astype(np.float64),
                inp.delta[b].astype(np.float64), inp.A.astype(np.float64), inp.D_skip.astype(np.float64))
        s0 = inp.S0[b].astype(np.float64) if with_s0 else None
        if chunked:
            y, s = SSD.ssd_scan_chunked(*args, S0=s0, Q=128)
        else:
            y, s = SSD.ssd_scan_sequential(*args, S0=s0)
        ys.append(y)
        ss.append(s)
    return np.stack(ys), np.stack(ss)


@pytest.mark.parametrize("shape", [
    (2, 300, 3, True),    # three chunks, the last one ragged, with a start state
    (1, 128, 2, False),   # exactly one chunk, no start state
    (1, 1, 1, True),      # one token
    (3, 700, 2, True),    # six chunks
], ids=lambda s: "B{}L{}H{}s0{}".format(*s))
def test_ssd_scan_matches_sequential_and_chunked_oracle(S, shape):
    B, L, H, with_s0 = shape
    inp = synth.draw_ssd_inputs(B, L, H, 64, 128, seed=L + H)
    y, sf = run_gpu(S, inp, with_s0)
    skip = inp.D_skip.astype(np.float64)[None, None, :, None] * synth.widen(inp.X[:, :, 0], "bf16")
    for chunked in (False, True):
        y_ref, s_ref = oracle(inp, with_s0, chunked)
        e = {"y": scaled_err(y, y_ref), "y_ssm": rel_rms_err(y - skip, y_ref - skip), "S_final": rel_rms_err(sf, s_ref)}
        print(shape, "chunked" if chunked else "sequential", {k: f"{v:.2e}" for k, v in e.items()})
        assert e["y"] <= 2e-2 and e["y_ssm"] <= 2e-2
        assert e["y"] <= 1e-3 and e["y_ssm"] <= 1e-3 and e["S_final"] <= 1e-3


def test_ssd_scan_rejects_unsupported_and_bad_arguments(S):
    inp = synth.draw_ssd_inputs(1, 16, 1, 64, 128, seed=1)
    t = torch.zeros(1 << 16, dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    mk = lambda **kw: S.swimba_ssd_dims(**{**dict(batch=1, seqlen=16, n_heads=1, head_dim=64, d_state=128, top_k=1),
                                           **kw})
    args = lambda: (t, t, t, t, t, t, t, None, t, None, ws, ws.numel())
    assert S.swimba_ssd_scan(mk(head_dim=32), *args()) == 2
    assert S.swimba_ssd_scan(mk(d_state=64), *args()) == 2
    assert S.swimba_ssd_scan(mk(top_k=2), *args()) == 2
    assert S.swimba_ssd_scan(mk(), None, *args()[1:]) == 1
    assert S.swimba_ssd_scan(mk(), t.data_ptr() + 4, *args()[1:]) == 3
    assert S.swimba_ssd_scan(mk(), *args()[:10], ws, 8) == 4
    del inp
