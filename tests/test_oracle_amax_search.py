"""Pins of the oracle's amax multiplier search (CPU): an independent
restatement (torch's FP8 conversion for the candidate codes, numpy FP64 for the
errors), its relation to max scaling (one multiplier of 1.0), and that it never
beats the full 126-code sweep (its candidates are a subset)."""
import numpy as np
import torch

import oracle
import synth
from tests import indep


def _layer():
    L = synth.make_config(0)
    W = L.W_f32()
    W = W if W.ndim == 3 else W[None]
    H = oracle.hessian(L.X, c_in=W.shape[2])
    amax = np.array([oracle.absmax(W[0])], np.float32)
    return W, H, amax


def test_restated_with_torch_fp8_and_numpy():
    W, H, amax = _layer()
    g = oracle.global_scale(amax[0])
    vals = indep.e4m3_values_torch()
    codes, _, errs = oracle.amax_search(W, amax, H)
    mult = np.array([np.float32(0.25 + 0.1 * k) for k in range(38)], np.float32)
    for r in range(0, W.shape[1], 3):
        for j in range(W.shape[2] // 16):
            w = W[0, r, 16 * j:16 * j + 16]
            a = np.float32(np.abs(w).max())
            x = (((mult * a).astype(np.float32) / np.float32(6)).astype(np.float32) / g).astype(np.float32)
            cands = np.clip(torch.from_numpy(np.minimum(x, np.float32(448))).to(torch.float8_e4m3fn)
                            .view(torch.uint8).numpy().astype(int), 1, 126)
            best, be = None, None
            for c in sorted(set(cands.tolist())):
                dw, _ = indep.candidate_dw(w, g, vals[c])
                e = float(dw @ H[0, j] @ dw)
                if be is None or e < be:
                    best, be = c, e
            if codes[0, r, j] != best:  # only a rounding-order tie may differ
                e_o = oracle.candidate_error(w, g, int(codes[0, r, j]), H[0, j])
                assert abs(e_o - be) <= 1e-12 * abs(be), (r, j, codes[0, r, j], best)


def test_single_unit_multiplier_is_max_scaling():
    W, H, amax = _layer()
    c1, a1, _ = oracle.amax_search(W, amax, H, start=1.0, step=0.0, n_mult=1)
    cm, am = oracle.baseline_scales(W, amax, oracle.BASELINE_MAX)
    assert np.array_equal(c1, cm) and np.array_equal(a1, am)


def test_never_beats_the_full_sweep():
    W, H, amax = _layer()
    _, _, e_search = oracle.amax_search(W, amax, H)
    _, _, e_sweep = oracle.sweep(W, amax, H)
    assert np.all(e_search >= e_sweep)
    assert np.mean(e_search > e_sweep) > 0.05  # a strict subset of candidates: it loses on some blocks
