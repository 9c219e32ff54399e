"""The sweep's measurement build (liblh_counters.so: the same sources with work
counters compiled in) gives the library's codes and plausible counts (needs a B200)."""
import ctypes
import os

import numpy as np
import pytest
import torch

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_counting_build_matches_and_counts(cuda_ok):
    import scale_calibration_b200 as lh
    path = os.path.join(ROOT, "scale_calibration_b200", "liblh_counters.so")
    if not os.path.exists(path):
        pytest.skip("measurement build not built (scale_calibration_b200/build.py --counters)")
    layer = synth.make_layer(700, 256, 900, seed=41)
    res = gu.run_library(layer)
    W, _, _ = gu.to_device(layer)
    lib = ctypes.CDLL(path)
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.lh_sweep_scales_ws.argtypes = [P, I32, I64, I64, I64, I64, P, P, P, P, P, SZ, P]
    lib.lh_debug_sweep_counts.argtypes = [P, I32]
    J = 16
    amax = torch.from_numpy(res["amax"]).cuda()
    H = torch.from_numpy(res["H"]).cuda()
    codes = torch.empty(1, 700, J, dtype=torch.uint8, device="cuda")
    bam = torch.empty(1, 700, J, dtype=torch.float32, device="cuda")
    ws = torch.empty(J * 16, dtype=torch.uint8, device="cuda")
    assert lib.lh_debug_sweep_counts(None, 1) == 0
    s = torch.cuda.current_stream().cuda_stream
    assert lib.lh_sweep_scales_ws(W.data_ptr(), lh.LH_BF16, 1, 700, 256, 256, amax.data_ptr(), H.data_ptr(),
                                  bam.data_ptr(), codes.data_ptr(), ws.data_ptr(), J * 16, s) == 0
    torch.cuda.synchronize()
    cnt = (ctypes.c_uint64 * 9)()
    assert lib.lh_debug_sweep_counts(cnt, 0) == 0
    chunks, blocks, cand, forms, need, below, resweep, classes, pairs = (int(x) for x in cnt)
    assert np.array_equal(codes.cpu().numpy(), res["codes"])
    assert blocks == 700 * J and classes == 8 * chunks
    assert 0 < forms <= cand <= 126 * chunks and need <= 32 * forms and resweep + pairs <= blocks
