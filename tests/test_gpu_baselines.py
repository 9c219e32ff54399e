"""Baseline scalers through the C ABI vs the oracle (needs a B200): max scaling
and four-over-six bit-exact on every block (codes and best amax); the weight-MSE
sweep (lh_sweep_scales with H = NULL) under the sweep's rule, with H = I on the
oracle side."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _baseline(layer, method):
    import scale_calibration_b200 as lh
    W, _, _ = gu.to_device(layer)
    n_mats, c_out, c_in = W.shape
    J = c_in // 16
    amax = torch.empty(n_mats, dtype=torch.float32, device="cuda")
    lh.lh_absmax(W, W, n_mats, c_out, c_in, W.stride(1), amax)
    codes = torch.empty(n_mats, c_out, J, dtype=torch.uint8, device="cuda")
    bam = torch.empty(n_mats, c_out, J, dtype=torch.float32, device="cuda")
    lh.lh_baseline_scales(W, W, n_mats, c_out, c_in, W.stride(1), amax, method, bam, codes)
    torch.cuda.synchronize()
    return amax.cpu().numpy(), codes.cpu().numpy(), bam.cpu().numpy()


@pytest.mark.parametrize("cfg", [0, 1, 4])
def test_max_and_four_over_six_every_block(cuda_ok, cfg):
    import scale_calibration_b200 as lh
    layer = synth.make_config(cfg)
    Wf = layer.W_f32()
    for method, om in [(lh.LH_SCALE_MAX, oracle.BASELINE_MAX),
                       (lh.LH_SCALE_FOUR_OVER_SIX, oracle.BASELINE_FOUR_OVER_SIX)]:
        amax, codes, bam = _baseline(layer, method)
        co, ao = oracle.baseline_scales(Wf, amax, om)
        assert np.array_equal(codes, co.reshape(codes.shape)), method
        assert np.array_equal(bam, ao.reshape(bam.shape)), method


def test_ragged_and_zero_layers(cuda_ok):
    import scale_calibration_b200 as lh
    layers = [synth.make_layer(200, 48, 16, seed=41, w_dtype="f32", outlier_frac=0.01),
              synth.make_layer(3, 16, 16, seed=42, w_dtype="bf16")]
    for layer in layers:
        Wf = layer.W_f32()
        for method, om in [(lh.LH_SCALE_MAX, 0), (lh.LH_SCALE_FOUR_OVER_SIX, 1)]:
            amax, codes, bam = _baseline(layer, method)
            co, ao = oracle.baseline_scales(Wf, amax, om)
            assert np.array_equal(codes, co.reshape(codes.shape)) and np.array_equal(bam, ao.reshape(bam.shape))
    z = synth.make_layer(4, 32, 16, seed=43, w_dtype="f32")
    z.W[...] = 0
    amax, codes, bam = _baseline(z, lh.LH_SCALE_FOUR_OVER_SIX)
    assert np.all(codes == 1) and np.all(bam == 0)


@pytest.mark.parametrize("cfg", [0, 1])
def test_mse_sweep_identity_hessian(cuda_ok, cfg):
    import scale_calibration_b200 as lh
    layer = synth.make_config(cfg)
    amax, codes, bam = _baseline(layer, lh.LH_SCALE_MSE)
    Wf = layer.W_f32()
    W3 = Wf if Wf.ndim == 3 else Wf[None]
    n_mats, c_out, c_in = W3.shape
    Hid = np.broadcast_to(np.eye(16), (n_mats, c_in // 16, 16, 16))
    if cfg == 0:
        ex, tol, fail, worst = gu.check_codes(W3, amax, Hid, codes, bam)
    else:
        rng = np.random.default_rng(44)
        n = 6000
        mats, rows, cols = (np.zeros(n, np.int64), rng.integers(0, c_out, n), rng.integers(0, c_in // 16, n))
        ex, tol, fail, worst = gu.check_codes(W3, amax, Hid, codes, bam, mats, rows, cols)
    assert fail == 0, (ex, tol, fail, worst)
