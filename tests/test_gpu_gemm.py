"""The block's projection GEMM (swimba_block_gemm) against the plain definition C = A B (+ R) in
fp64 on the same stored operands ("Mamba y las SSMs: el retorno del estado persistente", section
"Mamba", Figura 3: the in- and out-projections; section "Estado interno puramente lineal": the
residual connection).

bf16: every output within one bf16 spacing of the exact value plus 2^-13 sum_k |A_mk B_kn| (the
fp32 accumulation: K u_32 for K = 2048); fp32: within 1e-5 (1 + sum_k |A_mk B_kn|). Shapes are ragged in M, N and K
against the 128 x 256 x 64 tile, persistent CTAs run several tiles (both tensor-memory
accumulators and the smem ring wrap), the [x_pre | z] column split and the in-place residual
(C0 == R) are covered; the full in-projection of the Mamba-1.4B-like block is checked on sampled
rows."""
from __future__ import annotations

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


def bf16_spacing(v):
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return np.ldexp(1.0, np.floor(np.log2(a)).astype(int) - 7)


def draw(rng, shape, tdtype, scale=1.0):
    return (torch.from_numpy(rng.standard_normal(shape) * scale).float()).to(tdtype)


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def check(got, A, B, R, bf16, rows=None):
    a = A if rows is None else A[rows]
    ref = a @ B + (0.0 if R is None else (R if rows is None else R[rows]))
    mag = np.abs(a) @ np.abs(B)
    if bf16:
        bound = bf16_spacing(ref) + 2.0 ** -13 * mag + 1e-30
    else:
        bound = 1e-5 * (1.0 + mag)
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"worst {np.max(err / bound):.3f} of the bound"


SHAPES = [
    # M, N, K, split, residual
    (1, 8, 8, 8, False),              # one row, K below one 64-wide k-block
    (130, 264, 72, 264, True),        # ragged M, N, K: one partial tile in every direction
    (300, 520, 200, 256, False),      # split inside the second N tile
    (1000, 2048, 512, 1024, True),    # 8 x 8 tiles, split at the tile edge
    (4100, 2048, 136, 2048, False),   # 33 x 8 = 264 tiles: CTAs run two tiles
    (8192, 4096, 256, 2048, True),    # 1024 tiles: both accumulators wrap several times
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "M{}N{}K{}s{}r{}".format(*s))
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_block_gemm_matches_the_product(S, shape, io):
    M, N, K, split, res = shape
    if io == "f32" and M * N * K > 2 ** 31:
        pytest.skip("the fp32 SIMT kernel is for small blocks")
    bf16 = io == "bf16"
    td = torch.bfloat16 if bf16 else torch.float32
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    A = draw(rng, (M, K), td).cuda()
    B = draw(rng, (K, N), td, K ** -0.5).cuda()
    R = draw(rng, (M, N), td).cuda() if res else None
    C0 = torch.full((M, split), float("nan"), dtype=td, device="cuda")
    C1 = torch.full((M, N - split), float("nan"), dtype=td, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    st = S.swimba_block_gemm(S.dtype_code(io), M, N, K, A, K, B, N, C0, split, C1 if split < N else None,
                             max(N - split, 0), split, R, N, ws, 256)
    assert st == 0, S.swimba_status_string(st)
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(ws) == 0
    got = np.concatenate([host(C0), host(C1)], axis=1)
    Ah, Bh = host(A), host(B)
    Rh = host(R) if res else None
    rows = None if M <= 1024 else np.r_[0:64, M - 64:M, rng.integers(0, M, 128)]
    check(got if rows is None else got[rows], Ah, Bh, Rh, bf16, rows)


def test_block_gemm_in_place_residual(S):
    M, N, K = 520, 264, 96
    rng = np.random.default_rng(3)
    A = draw(rng, (M, K), torch.bfloat16).cuda()
    B = draw(rng, (K, N), torch.bfloat16, K ** -0.5).cuda()
    R = draw(rng, (M, N), torch.bfloat16).cuda()
    Rh = host(R)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert S.swimba_block_gemm(S.SWIMBA_BF16, M, N, K, A, K, B, N, R, N, None, 0, N, R, N, ws, 256) == 0
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(ws) == 0
    check(host(R), host(A), host(B), Rh, True)


def test_block_in_projection_full_size_sampled_rows(S):
    """The Mamba-1.4B-like block's in-projection: u [8 x 4096, 2048] times W_in [2048, 8192], split
    at D = 4096, as the block runs it."""
    T, dm, D = 8 * 4096, 2048, 4096
    rng = np.random.default_rng(11)
    u = draw(rng, (T, dm), torch.bfloat16).cuda()
    W = draw(rng, (dm, 2 * D), torch.bfloat16, dm ** -0.5).cuda()
    x_pre = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    z = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert S.swimba_block_gemm(S.SWIMBA_BF16, T, 2 * D, dm, u, dm, W, 2 * D, x_pre, D, z, D, D, None, 0, ws, 256) == 0
    torch.cuda.synchronize()
    assert S.swimba_get_device_status(ws) == 0
    rows = np.r_[0:32, T - 32:T, rng.integers(0, T, 64)]
    rt = torch.from_numpy(rows).cuda()
    got = np.concatenate([host(x_pre[rt]), host(z[rt])], axis=1)
    uh = host(u[rt])
    check(got, uh, host(W), None, True)


def test_block_gemm_rejects_bad_arguments(S):
    t = torch.empty(4096, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    bf = S.SWIMBA_BF16
    assert S.swimba_block_gemm(bf, 8, 8, 0, t, 8, t, 8, t, 8, None, 0, 8, None, 0, ws, 256) == 1  # K = 0
    assert S.swimba_block_gemm(bf, 8, 12, 8, t, 8, t, 12, t, 12, None, 0, 12, None, 0, ws, 256) == 2  # N % 8
    assert S.swimba_block_gemm(bf, 8, 8, 8, t.data_ptr() + 2, 8, t, 8, t, 8, None, 0, 8, None, 0, ws, 256) == 3
    assert S.swimba_block_gemm(bf, 8, 8, 8, t, 8, t, 8, t, 8, None, 0, 8, None, 0, ws, 16) == 4
    assert S.swimba_block_gemm(bf, 8, 16, 8, t, 8, t, 16, t, 8, None, 0, 8, None, 0, ws, 256) == 1  # C1 missing
    assert S.swimba_block_gemm(bf, 0, 8, 8, None, 8, None, 8, None, 8, None, 0, 8, None, 0, ws, 256) == 0
