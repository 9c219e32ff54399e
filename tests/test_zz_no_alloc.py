"""The allocation-free Hessian entry point against the workspace one (needs a B200).

lh_accumulate_hessian_noalloc serves callers that cannot allocate device
memory when they calibrate (processes whose HBM is already reserved by their
own pools, plugins whose host owns every allocation, callers avoiding the
device-wide synchronisation of cudaMalloc/cudaFree). It must give the same H
as lh_accumulate_hessian with a caller workspace, call after call, although
every call reuses the library's one fixed scratch array. This file sorts last
so that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest
import torch

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _hessians(layer):
    import scale_calibration_b200 as lh
    _, X, off = gu.to_device(layer)
    n_groups = layer.n_mats if off is not None else 1
    J = layer.c_in // 16
    H_ws = torch.zeros(n_groups, J, 16, 16, dtype=torch.float32, device="cuda")
    wsb = lh.lh_hessian_workspace_bytes(layer.n_tok, layer.c_in, n_groups)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    lh.lh_accumulate_hessian(X, lh.LH_BF16, layer.n_tok, layer.c_in, X.stride(0), off, n_groups, H_ws, ws, wsb)
    assert lh.lh_workspace_status(ws) == 0
    H_na = torch.zeros_like(H_ws)
    lh.lh_accumulate_hessian_noalloc(X, lh.LH_BF16, layer.n_tok, layer.c_in, X.stride(0), off, n_groups, H_na)
    assert lh.lh_noalloc_status() == 0  # no kernel-side error left in the scratch header
    torch.cuda.synchronize()
    return H_ws.cpu().numpy(), H_na.cpu().numpy()


def test_noalloc_matches_workspace_entry_on_consecutive_calls(cuda_ok):
    layers = [
        synth.make_layer(8, 128, 2552, seed=21, n_mats=8, counts=[0, 5, 1, 300, 0, 17, 129, 2100]),
        synth.make_layer(4, 4096, 2048, seed=22),      # attention-projection-sized X
    ]
    for layer in layers:   # two calls in a row, different shapes, on the shared scratch array
        H_ws, H_na = _hessians(layer)
        per, whole, bad = gu.hessian_rel_errors(H_na, H_ws.astype(np.float64))
        assert per <= gu.HESSIAN_RTOL and whole <= gu.HESSIAN_RTOL and bad == 0, (per, whole, bad)
        assert np.array_equal(H_ws, H_na)  # same kernels, deterministic order


def test_noalloc_reports_kernel_side_errors_through_its_status(cuda_ok):
    # decreasing offsets (two groups over the same 1000 tokens): the kernel stays in bounds
    # and records the error in the scratch's status word, which lh_noalloc_status reads; the
    # next valid call leaves no error
    import scale_calibration_b200 as lh
    layer = synth.make_layer(8, 128, 1000, seed=32)
    _, X, _ = gu.to_device(layer)
    off = torch.tensor([0, 1000, 0, 1000], dtype=torch.int64, device="cuda")
    H = torch.zeros(3, 8, 16, 16, device="cuda")
    lh.lh_accumulate_hessian_noalloc(X, lh.LH_BF16, 1000, 128, 128, off, 3, H)
    assert lh.lh_noalloc_status() == 1  # LH_ERR_INVALID_ARG
    assert "overlap" in lh.lh_last_error_message()
    H1 = torch.zeros(1, 8, 16, 16, device="cuda")
    lh.lh_accumulate_hessian_noalloc(X, lh.LH_BF16, 1000, 128, 128, None, 1, H1)
    assert lh.lh_noalloc_status() == 0
