"""Golden fixtures: format facts from the pages and the oracle's tiny-layer result."""
import os

import numpy as np

import oracle
import synth

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _kv(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            k, *v = line.split()
            out[k] = v
    return out


def test_format_fixture():
    kv = _kv(os.path.join(HERE, "nvfp4_format.txt"))
    grid = [float(x) for x in kv["e2m1_grid"]]
    # every grid value is a fixed point of the oracle's rounding, nothing else is
    assert [oracle.e2m1_rne(x) for x in grid] == grid
    assert max(grid) == float(kv["e2m1_max"][0]) == oracle.e2m1_rne(100.0)
    codes = [c for c in range(128) if np.isfinite(oracle.e4m3_value(c)) and oracle.e4m3_value(c) > 0]
    assert len(codes) == int(kv["e4m3_candidates"][0])
    assert codes[0] == int(kv["e4m3_first_code"][0]) and codes[-1] == int(kv["e4m3_last_code"][0])
    assert oracle.e4m3_value(codes[0]) == float(kv["e4m3_min_candidate"][0])
    assert oracle.e4m3_value(codes[-1]) == float(kv["e4m3_max_candidate"][0])
    assert float(kv["global_divisor"][0]) == max(grid) * oracle.e4m3_value(codes[-1])
    assert oracle.global_scale(2688.0) == 1.0


def test_tiny_sweep_fixture():
    lines = [l for l in open(os.path.join(HERE, "tiny_sweep.txt")) if not l.startswith("#")]
    A_ref = float.fromhex(lines[0].split()[1])
    err_ref = float.fromhex(lines[1].split()[1])
    codes_ref = np.array([[int(x) for x in l.split()] for l in lines[2:]], np.uint8)
    L = synth.make_config(0)
    W = L.W_f32()[0]
    A = oracle.absmax(W)
    assert float(A) == A_ref
    codes, _, err = oracle.sweep(W, [A], oracle.hessian(L.X))
    assert np.array_equal(codes[0], codes_ref)
    assert float(err.sum()) == err_ref
