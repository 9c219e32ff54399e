"""Pins of the oracle's baseline scalers and its E4M3 rounding (CPU).

E4M3 round-to-nearest-even is checked against torch's float8_e4m3fn conversion
(values up to 448; saturation above it separately); max scaling and
four-over-six are restated here with numpy FP32 steps, torch's FP8 cast and the
exhaustive-distance E2M1 quantiser of tests/indep.py."""
import numpy as np
import torch

import oracle
import synth
from tests import indep


def torch_e4m3(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(int)


def test_e4m3_rne_matches_torch_including_ties():
    vals = np.array([oracle.e4m3_value(c) for c in range(0, 127)], np.float64)
    mids = (vals[:-1] + vals[1:]) / 2
    xs = [vals, mids, np.nextafter(mids.astype(np.float32), 0), np.nextafter(mids.astype(np.float32), 1000)]
    rng = np.random.default_rng(7)
    xs.append(rng.uniform(0, 448, 20000))
    xs.append(np.exp2(rng.uniform(-12, np.log2(448), 20000)))
    x = np.concatenate([np.asarray(a, np.float32) for a in xs])
    x = x[(x >= 0) & (x <= 448)]
    ours = np.array([oracle.e4m3_rne(float(v)) for v in x])
    assert np.array_equal(ours, torch_e4m3(x))
    assert oracle.e4m3_rne(448.0) == 0x7E and oracle.e4m3_rne(1e6) == 0x7E and oracle.e4m3_rne(0.0) == 0


def _layer():
    L = synth.make_config(0)
    W = L.W_f32()
    W = (W if W.ndim == 3 else W[None]).copy()
    W[0, 0, :16] = 0.0                  # an all-zero block
    W[0, 1, 5] = np.float32(0.9)        # an outlier block
    return W


def _codes_for(W, g, d):
    a = np.abs(W.reshape(W.shape[0], W.shape[1], -1, 16)).max(-1).astype(np.float32)
    x = ((a / np.float32(d)).astype(np.float32) / np.float32(g)).astype(np.float32)
    return np.clip(torch_e4m3(np.minimum(x, np.float32(448))), 1, 126)


def test_max_scaling_restated():
    W = _layer()
    amax = np.array([oracle.absmax(W[0])], np.float32)
    g = oracle.global_scale(amax[0])
    codes, bam = oracle.baseline_scales(W, amax, oracle.BASELINE_MAX)
    assert np.array_equal(codes, _codes_for(W, g, 6.0))
    exp = np.array([np.float32(6.0) * oracle.candidate_scale(int(c), g) for c in codes.ravel()], np.float32)
    assert np.array_equal(bam.ravel(), exp)


def test_four_over_six_restated():
    W = _layer()
    amax = np.array([oracle.absmax(W[0])], np.float32)
    g = oracle.global_scale(amax[0])
    vals = indep.e4m3_values_torch()
    codes, _ = oracle.baseline_scales(W, amax, oracle.BASELINE_FOUR_OVER_SIX)
    c6s, c4s = _codes_for(W, g, 6.0), _codes_for(W, g, 4.0)
    n_four = 0
    for r in range(W.shape[1]):
        for j in range(W.shape[2] // 16):
            w = W[0, r, 16 * j:16 * j + 16]
            c6, c4 = int(c6s[0, r, j]), int(c4s[0, r, j])
            e6 = float(np.sum(indep.candidate_dw(w, g, vals[c6])[0] ** 2))
            e4 = float(np.sum(indep.candidate_dw(w, g, vals[c4])[0] ** 2))
            want = c4 if (e4 < e6 or (e4 == e6 and c4 < c6)) else c6
            assert codes[0, r, j] == want, (r, j, c6, c4, e6, e4)
            n_four += want == c4 and c4 != c6
    assert n_four > 0  # both candidates win somewhere on this layer


def test_zero_global_amax_gives_code_one():
    W = np.zeros((1, 2, 32), np.float32)
    for m in (oracle.BASELINE_MAX, oracle.BASELINE_FOUR_OVER_SIX):
        codes, bam = oracle.baseline_scales(W, np.array([0.0], np.float32), m)
        assert np.all(codes == 1) and np.all(bam == 0)
