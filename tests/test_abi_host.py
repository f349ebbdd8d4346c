"""Host-side checks of the C ABI that need no GPU: the library loads, exports every function
include/swimba.h declares, sizes workspaces, and rejects bad arguments before any launch."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import build

    build.build()
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


def declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(swimba_\w+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_function(S):
    names = declared_functions()
    assert len(names) >= 7
    for n in names:
        assert hasattr(S._lib, n), n
    assert set(names) == set(S.EXPORTED)


def test_status_strings(S):
    assert S.swimba_status_string(0) == "ok"
    for code in range(1, 7):
        assert S.swimba_status_string(code) not in ("ok", "unknown status")
    assert S.swimba_status_string(99) == "unknown status"


def test_workspace_sizes(S):
    from parameter_space_moe_swimba_b200.configs import CONFIGS

    for cfg in CONFIGS.values():
        dims = S.make_dims(cfg, seqlen=1 if cfg.decode_steps else None)
        for op in range(5):
            assert S.swimba_workspace_size(dims, op) >= 256
        assert S.swimba_workspace_size(dims, 4) == max(S.swimba_workspace_size(dims, op) for op in range(4))
    bad = S.make_dims(CONFIGS["tiny_fp32"], top_k=9)
    assert S.swimba_workspace_size(bad, 4) == 0


def test_scan_backward_workspace_holds_its_buffers(S):
    """The scan backward's workspace: the status block, the state at every 16-token chunk start
    (B x ceil(L/16) x D x N fp32), the per-64-channel-tile partial rows (dB | dC | dgates), the
    per-sequence dA and dD partials and the packed kernel's per-CTA sub-block state scratch
    (16 KB per CTA of 64 channels), each rounded up to 256 bytes."""
    from parameter_space_moe_swimba_b200.configs import CONFIGS

    up = lambda v: (v + 255) // 256 * 256
    for name in ("tiny_fp32", "mamba130m_like", "mamba1p4b_like", "long_seq_65536"):
        cfg = CONFIGS[name]
        dims = S.make_dims(cfg)
        B, L, D, N, E, k = cfg.batch, cfg.seqlen, cfg.d_inner, cfg.d_state, cfg.n_experts, cfg.top_k
        tiles, nck = -(-D // 64), -(-L // 16)
        need = (up(B * nck * D * N * 4) + up(tiles * B * L * (2 * N + k) * 4) + up(B * E * D * N * 4) +
                up(B * D * 4) + up(tiles * B * 4 * 2 * 128 * 16))
        got = S.swimba_workspace_size(dims, S.SWIMBA_OP_SCAN_BWD)
        assert need <= got <= need + 4096, (name, need, got)


def test_invalid_arguments_return_before_any_launch(S):
    from parameter_space_moe_swimba_b200.configs import CONFIGS

    cfg = CONFIGS["tiny_fp32"]
    dims = S.make_dims(cfg)
    fake = 1 << 40  # never dereferenced: every case fails validation first
    w = S.swimba_weights(fake, fake, fake, fake, fake, fake)
    assert S.swimba_route(dims, None, fake, fake, fake, 0) == 1
    assert S.swimba_route(S.make_dims(cfg, top_k=5), fake, fake, fake, fake, 0) == 1
    assert S.swimba_route(S.make_dims(cfg, n_experts=17, top_k=2), fake, fake, fake, fake, 0) == 2
    assert S.swimba_route(dims, fake + 8, fake, fake, fake, 0) == 3
    odd = S.make_dims(cfg)
    odd.d_inner = 12
    assert S.swimba_route(odd, fake, fake, fake, fake, 0) == 2
    big_n = S.make_dims(cfg)
    big_n.d_state = 17
    assert S.swimba_scan_fwd(big_n, fake, fake, fake, fake, fake, fake, fake, w, None, fake, None, None, fake,
                             1 << 20, 0) == 2
    assert S.swimba_mixed_proj(dims, fake, fake, fake, w, fake, fake, fake, fake, 8, 0) == 4
    assert S.swimba_mixed_proj(dims, fake, fake, fake, w, fake, fake, fake, None, 1 << 20, 0) == 4
    assert S.swimba_scan_fwd(dims, fake, fake, fake, fake, fake, fake, fake, w, None, None, None, None, fake,
                             1 << 20, 0) == 1
    step_dims = S.make_dims(cfg)  # seqlen 128: a decode step needs seqlen 1
    assert S.swimba_step(step_dims, fake, fake, fake, fake, fake, fake, fake, w, fake, fake, 0) == 1
    assert S.swimba_get_device_status(None, 0) == 1
    assert S.swimba_check_wait_timeout(None, 256, 10**6, 0) == 4
    assert S.swimba_check_wait_timeout(fake, 64, 10**6, 0) == 4
    assert S.swimba_check_wait_timeout(fake + 8, 256, 10**6, 0) == 3
    assert S.swimba_check_wait_timeout(fake, 256, 10, 0) == 1
    assert S.swimba_check_wait_timeout(fake, 256, 2 * 10**9, 0) == 1


def test_block_and_conv_arguments_are_checked_before_any_launch(S):
    from parameter_space_moe_swimba_b200.configs import CONFIGS

    cfg = CONFIGS["mamba1p4b_like"]
    dims = S.make_dims(cfg)
    fake = 1 << 40  # never dereferenced
    bd = S.swimba_block_dims(dims, 2048, 4)
    n = S.swimba_block_workspace_size(bd)
    # layer workspace + x_pre, z, x, layer out (bf16) + idx, gates + delta + B_mix, C_mix
    T, D = cfg.tokens, cfg.d_inner
    assert n >= S.swimba_workspace_size(dims, 4) + 4 * T * D * 2 + 2 * T * 2 * 4 + T * D * 4 + 2 * T * 16 * 4
    for bad in (S.swimba_block_dims(dims, 2047, 4), S.swimba_block_dims(dims, 2048, 9),
                S.swimba_block_dims(dims, 2048, 0), S.swimba_block_dims(dims, 0, 4)):
        assert S.swimba_block_workspace_size(bad) == 0
    mixed = S.make_dims(cfg)
    mixed.io_dtype = 0  # the GEMMs take one operand type
    assert S.swimba_block_workspace_size(S.swimba_block_dims(mixed, 2048, 4)) == 0
    lw = S.swimba_weights(fake, fake, fake, fake, fake, fake)
    w = S.swimba_block_weights(fake, fake, fake, fake, lw)
    assert S.swimba_block_fwd(bd, fake, w, None, None, fake, None, None, fake, n - 256, 0) == 4
    assert S.swimba_block_fwd(bd, fake, w, None, None, fake, None, None, None, n, 0) == 4
    assert S.swimba_block_fwd(bd, None, w, None, None, fake, None, None, fake, n, 0) == 1
    assert S.swimba_block_fwd(bd, fake + 2, w, None, None, fake, None, None, fake, n, 0) == 3
    assert S.swimba_block_fwd(S.swimba_block_dims(dims, 2048, 9), fake, w, None, None, fake, None, None, fake, n,
                              0) == 2
    nw = S.swimba_block_weights(fake, None, fake, fake, lw)
    assert S.swimba_block_fwd(bd, fake, nw, None, None, fake, None, None, fake, n, 0) == 1
    # the layer's and the states' arguments are checked before the in-projection is queued
    no_A = S.swimba_block_weights(fake, fake, fake, fake, S.swimba_weights(fake, fake, fake, fake, None, fake))
    assert S.swimba_block_fwd(bd, fake, no_A, None, None, fake, None, None, fake, n, 0) == 1
    odd_A = S.swimba_block_weights(fake, fake, fake, fake, S.swimba_weights(fake, fake, fake, fake, fake + 4, fake))
    assert S.swimba_block_fwd(bd, fake, odd_A, None, None, fake, None, None, fake, n, 0) == 3
    assert S.swimba_block_fwd(bd, fake, w, None, fake, fake, None, fake, fake, n, 0) == 1  # conv state in == out
    assert S.swimba_block_fwd(bd, fake, w, fake + 4, None, fake, None, None, fake, n, 0) == 3  # h0
    assert S.swimba_block_fwd(bd, fake, w, None, fake + 8, fake, None, None, fake, n, 0) == 3  # conv state in
    assert S.swimba_block_step(bd, fake, w, fake, fake, fake, fake, n, 0) == 1  # seqlen != 1
    sd = S.swimba_block_dims(S.make_dims(cfg, seqlen=1), 2048, 4)
    assert S.swimba_block_step(sd, fake, w, None, fake, fake, fake, n, 0) == 1  # no state
    assert S.swimba_block_step(sd, fake, w, fake, None, fake, fake, n, 0) == 1  # no conv state
    assert S.swimba_block_step(sd, fake, w, fake + 4, fake, fake, fake, n, 0) == 3  # h
    assert S.swimba_block_step(sd, fake, w, fake, fake + 8, fake, fake, n, 0) == 3  # conv state
    # the convolution alone
    assert S.swimba_conv1d_fwd(dims, 9, fake, fake, fake, None, fake, None, 0) == 2
    assert S.swimba_conv1d_fwd(dims, 4, None, fake, fake, None, fake, None, 0) == 1
    assert S.swimba_conv1d_fwd(dims, 4, fake, fake, fake, fake, fake, fake, 0) == 1  # state in == out
    assert S.swimba_conv1d_fwd(dims, 4, fake + 4, fake, fake, None, fake, None, 0) == 3
    assert S.swimba_conv1d_fwd(dims, 4, fake, fake, fake, fake + 8, fake, None, 0) == 3
    assert S.swimba_conv1d_step(dims, 4, fake, fake, fake, fake, fake, 0) == 1  # seqlen != 1
    step = S.make_dims(cfg, seqlen=1)
    assert S.swimba_conv1d_step(step, 4, fake, fake, fake, None, fake, 0) == 1
    assert S.swimba_conv1d_step(step, 4, fake, fake, fake, fake + 2, fake, 0) == 3
