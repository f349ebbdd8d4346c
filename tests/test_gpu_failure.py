"""Failure reporting on the GPU without a fault: a bounded device wait that runs out must end with
SWIMBA_ERR_TIMEOUT in the workspace status block (not a hang), and the context must stay usable.

The wait is made to run out on purpose through swimba_check_wait_timeout (an mbarrier that nothing
completes, a 20 ms limit); nothing here faults, traps or hangs the GPU."""
import time

import numpy as np
import pytest

from swimba_cases import make_case, oracle_layer

pytestmark = pytest.mark.gpu

OK, TIMEOUT = 0, 6


@pytest.fixture(scope="module")
def S():
    from parameter_space_moe_swimba_b200 import swimba

    return swimba


def test_stalled_wait_reports_timeout_and_the_context_survives(S):
    import torch

    from parameter_space_moe_swimba_b200.configs import CONFIGS

    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert S.swimba_get_device_status(ws) == OK
    t0 = time.time()
    assert S.swimba_check_wait_timeout(ws, ws.numel(), 20_000_000) == OK  # launched
    assert S.swimba_get_device_status(ws) == TIMEOUT                     # reported
    assert time.time() - t0 < 10.0                                       # and it ended
    assert S.swimba_get_device_status(ws) == OK                          # reading clears it

    # the same context still computes a correct layer
    case = make_case(CONFIGS["tiny_fp32"])
    cfg = case.cfg
    dims = S.make_dims(cfg)
    W = S.upload_weights(case.w)
    buf = S.LayerBuffers(dims, torch.float32, with_y=True)
    S.layer_forward(dims, S.to_device(case.x, cfg.io_dtype), S.to_device(case.z, cfg.io_dtype), W.struct(), buf)
    assert S.swimba_get_device_status(buf.ws) == OK
    ref = oracle_layer(case)
    np.testing.assert_array_equal(buf.idx.cpu().numpy(), ref["idx"])
    y = buf.y.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(y - ref["y"]) / (1 + np.abs(ref["y"]))) <= 1e-4
