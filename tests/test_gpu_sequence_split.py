"""The sequence split's kernels through the C ABI on one GPU: a sequence cut into pieces (as the
ranks of a sequence-parallel run would own them), every piece routed, projected and summarised
(swimba_scan_summary), the summaries chained (swimba_scan_chain), every piece scanned from its
chained start state -- against the fp64 oracle on the whole sequence, and the summaries against
the oracle's piece summaries. The pieces run one after another on one stream; no kernel waits on
another piece's kernel."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import swimba_oracle as O
from parameter_space_moe_swimba_b200.configs import LayerConfig
from tests.swimba_cases import TOL_Y, make_case, oracle_layer, rel_rms_err, scaled_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


def io_torch(cfg):
    return torch.bfloat16 if cfg.io_dtype == "bf16" else torch.float32


SHAPES = [
    # B, L, D, N, R, E, k, io, w, pieces
    (2, 3000, 256, 16, 32, 8, 2, "bf16", "bf16", 3),   # fast path (TMA scan, segmented summaries)
    (1, 4100, 64, 16, 16, 16, 1, "bf16", "bf16", 4),   # E = 16, top-1, a ragged last piece
    (2, 333, 40, 5, 3, 3, 3, "f32", "f32", 2),         # generic path (fp32, N = 5, k = 3)
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}L{}D{}N{}R{}E{}k{}{}{}P{}".format(*s))
def test_pieces_chained_equal_the_whole_sequence(S, shape):
    from parameter_space_moe_swimba_b200.parallel import CudaPieceOps, sequence_piece

    B, L, D, N, R, E, k, io, wd, P = shape
    cfg = LayerConfig("pieces", B, L, D, N, R, E, k, io, wd, seed=31, cached_state=True)
    case = make_case(cfg, a_mode="random", with_h0=True)
    ref = oracle_layer(case)
    W = S.upload_weights(case.w)
    ws = W.struct()
    ops = CudaPieceOps(S, ws)
    x_all = S.to_device(case.x, io)
    z_all = S.to_device(case.z, io)
    h0 = torch.from_numpy(case.h0).cuda()

    pieces, summaries = [], []
    for r in range(P):
        a, b = sequence_piece(L, P, r)
        dims = S.make_dims(cfg, seqlen=b - a)
        buf = S.LayerBuffers(dims, io_torch(cfg), with_y=True)
        piece = (dims, x_all[:, a:b].contiguous(), z_all[:, a:b].contiguous(), buf)
        ops.route_and_project(piece)
        pieces.append((a, b, piece))
        summaries.append(ops.summary(piece))
    hz_all = torch.stack([s[0] for s in summaries])
    ld_all = torch.stack([s[1] for s in summaries])
    h_start = ops.chain(hz_all, ld_all, h0)
    for r, (_, _, piece) in enumerate(pieces):
        ops.scan(piece, h_start[r])
    torch.cuda.synchronize()
    for _, _, piece in pieces:
        assert S.swimba_get_device_status(piece[3].ws) == 0

    # the summaries against the oracle's, on the oracle's own streams of each piece
    W64 = case.weights64()
    tol = 1e-5 if io == "f32" else 1e-2
    for r, (a, b, _) in enumerate(pieces):
        sl = slice(a, b)
        hz, ld = O.scan_summary(case.x64()[:, sl], ref["dt_mix"][:, sl], ref["B_mix"][:, sl], ref["idx"][:, sl],
                                ref["gates"][:, sl], W64["A"])
        assert rel_rms_err(hz_all[r].cpu().numpy(), hz) <= tol, r
        assert rel_rms_err(ld_all[r].cpu().numpy(), ld) <= tol, r
    # the pieces together against the whole sequence
    y = np.concatenate([p[3].y.cpu().numpy() for _, _, p in pieces], 1)
    out = np.concatenate([p[3].out.float().cpu().numpy() for _, _, p in pieces], 1)
    h_last = pieces[-1][2][3].h_final.cpu().numpy()
    t = TOL_Y[io]
    ey, eo = scaled_err(y, ref["y"]), scaled_err(out, ref["out"])
    ys = y - case.w.D_skip.astype(np.float64) * case.x64()
    ys_ref = ref["y"] - case.w.D_skip.astype(np.float64) * case.x64()
    ess = rel_rms_err(ys, ys_ref)
    eh = rel_rms_err(h_last, ref["h_final"])
    eH = rel_rms_err(h_start[P].cpu().numpy(), ref["h_final"])
    print(shape, {"y": ey, "out": eo, "y_ssm": ess, "h_final": eh, "chained end": eH})
    assert ey <= t and eo <= t and ess <= t
    assert eh <= (1e-5 if io == "f32" else 1e-2)
    assert eH <= (1e-5 if io == "f32" else 1e-2)


def test_summary_and_chain_reject_bad_arguments(S):
    cfg = LayerConfig("pieces", 1, 32, 64, 16, 16, 4, 2, "bf16", "bf16", seed=1)
    dims = S.make_dims(cfg)
    t = torch.empty(64, device="cuda")
    W = S.upload_weights(make_case(cfg).w).struct()
    ws = S.new_workspace(dims, S.SWIMBA_OP_SUMMARY)
    assert S.swimba_scan_summary(dims, None, t, t, t, t, W, t, t, ws, ws.numel()) == 1
    assert S.swimba_scan_summary(dims, t, t, t, t, t, W, t, t, ws, 16) == 4
    assert S.swimba_scan_summary(dims, t.data_ptr() + 4, t, t, t, t, W, t, t, ws, ws.numel()) == 3
    assert S.swimba_scan_chain(dims, 0, t, t, None, t) == 1
    assert S.swimba_scan_chain(dims, 2, None, t, None, t) == 1
