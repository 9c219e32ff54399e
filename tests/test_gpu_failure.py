"""Failure detection without a GPU fault (needs a B200).

The kernels' mbarrier waits are bounded; an expired wait records
LH_ERR_TIMEOUT in the workspace header, which the host reads with
lh_workspace_status. Here the wait runs out on a barrier that nothing
arrives on, the status comes back, and the context keeps working.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives(cuda_ok):
    import scale_calibration_b200 as lh
    from scale_calibration_b200._binding import LH_ERR_TIMEOUT, LH_OK
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    lh.lh_debug_wait_timeout(ws, 256, 100000, 0)           # 100 ms, nothing arrives
    assert lh.lh_workspace_status(ws) == LH_ERR_TIMEOUT     # synchronises
    assert time.perf_counter() - t0 >= 0.09
    assert "bounded wait" in lh.lh_last_error_message()
    lh.lh_debug_wait_timeout(ws, 256, 100000, 1)           # barrier completed: no timeout
    assert lh.lh_workspace_status(ws) == LH_OK
    # the same context still runs the real path correctly
    layer = synth.make_layer(32, 64, 100, seed=30)
    res = gu.run_library(layer)
    per, _, _ = gu.hessian_rel_errors(res["H"], oracle.hessian(layer.X))
    assert per <= gu.HESSIAN_RTOL
