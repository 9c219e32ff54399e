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


def _search(layer, H_dev, rows=None, **kw):
    import scale_calibration_b200 as lh
    W, _, _ = gu.to_device(layer)
    n_mats, c_out, c_in = W.shape
    J = c_in // 16
    amax = torch.empty(n_mats, dtype=torch.float32, device="cuda")
    lh.lh_absmax(W, W, n_mats, c_out, c_in, W.stride(1), amax)
    codes = torch.empty(n_mats, c_out, J, dtype=torch.uint8, device="cuda")
    bam = torch.empty(n_mats, c_out, J, dtype=torch.float32, device="cuda")
    lh.lh_search_amax(W, W, n_mats, c_out, c_in, W.stride(1), amax, H_dev, bam, codes, **kw)
    torch.cuda.synchronize()
    return amax.cpu().numpy(), codes.cpu().numpy(), bam.cpu().numpy()


def _check_search(layer, H_np, codes, bam, amax, rows, **kw):
    Wf = layer.W_f32()
    W3 = (Wf if Wf.ndim == 3 else Wf[None])[:, :rows, :]
    co, ao, eo = oracle.amax_search(W3, amax, H_np, **kw)
    cg = codes[:, :rows, :]
    bad = 0
    for m, r, j in zip(*np.nonzero(cg != co)):
        g = oracle.global_scale(amax[m])
        e = oracle.candidate_error(W3[m, r, 16 * j:16 * j + 16], g, int(cg[m, r, j]), H_np[m, j])
        if not (e - eo[m, r, j] <= gu.CODE_RTOL * abs(eo[m, r, j])):
            bad += 1
    assert bad == 0
    g_all = [oracle.global_scale(a) for a in amax]
    exp = np.array([[[np.float32(6.0) * oracle.candidate_scale(int(c), g_all[m]) for c in row] for row in cg[m]]
                    for m in range(cg.shape[0])], np.float32)
    assert np.array_equal(bam[:, :rows, :], exp)


@pytest.mark.parametrize("cfg,rows", [(0, 64), (1, 192), (4, 48)])
def test_amax_search_with_hessian(cuda_ok, cfg, rows):
    import scale_calibration_b200 as lh
    layer = synth.make_config(cfg)
    _, X, off = gu.to_device(layer)
    n_mats, c_in = layer.n_mats, layer.c_in
    G = n_mats if off is not None else 1
    H = torch.zeros(G, c_in // 16, 16, 16, device="cuda")
    wsb = lh.lh_hessian_workspace_bytes(X.shape[0], c_in, G)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    lh.lh_accumulate_hessian(X, lh.LH_BF16, X.shape[0], c_in, X.stride(0), off, G, H, ws, wsb)
    torch.cuda.synchronize()
    Hn = H.cpu().numpy().astype(np.float64)
    Hn = np.broadcast_to(Hn, (n_mats,) + Hn.shape[1:])
    amax, codes, bam = _search(layer, H)
    _check_search(layer, Hn, codes, bam, amax, rows)


def test_amax_search_identity_and_other_grids(cuda_ok):
    layer = synth.make_config(1)
    c_in = layer.c_in
    Hid = np.broadcast_to(np.eye(16), (1, c_in // 16, 16, 16))
    for kw in (dict(), dict(start=0.5, step=0.05, n_mult=31), dict(start=1.0, step=0.0, n_mult=1)):
        amax, codes, bam = _search(layer, None, **kw)
        _check_search(layer, Hid, codes, bam, amax, 96, **kw)
