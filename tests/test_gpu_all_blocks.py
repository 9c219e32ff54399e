"""Every block of every full-size layer, CUDA library vs oracle (needs a B200).

The library runs the whole path on the layer; the oracle then sweeps every block
with the GPU's H ("sweep-only": the Hessians are checked separately in
test_gpu_parity.py), sharded by row range over the host's cores in spawned
processes. Codes must be bit-exact except where the oracle's FP64 error of the
GPU's code is within 1e-6 relative of the oracle minimum; best_amax must equal
fp32(6 * s(code)) for every block.
"""
import multiprocessing as mp
import os

import numpy as np
import pytest

import oracle
import synth
from tests import gpu_util as gu
from tests import oracle_shard

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_every_block_matches_oracle(cuda_ok, cfg, tmp_path):
    layer = synth.make_config(cfg)
    res = gu.run_library(layer)
    W = layer.W_f32()
    if W.ndim == 2:
        W = W[None]
    n_mats, c_out, c_in = W.shape
    H = res["H"].astype(np.float32)
    if H.shape[0] != n_mats:  # one H shared by the matrices of a layer
        H = np.broadcast_to(H, (n_mats,) + H.shape[1:])
    np.save(tmp_path / "W.npy", W)
    np.save(tmp_path / "H.npy", np.ascontiguousarray(H))
    np.save(tmp_path / "amax.npy", res["amax"])
    np.save(tmp_path / "codes.npy", res["codes"])

    # best_amax = fp32(6 * fp32(v(code) * g)) for every block
    table = np.zeros((n_mats, 127), np.float32)
    for m in range(n_mats):
        g = oracle.global_scale(res["amax"][m])
        table[m, 1:] = [np.float32(6.0) * oracle.candidate_scale(c, g) for c in range(1, 127)]
    assert res["codes"].min() >= 1 and res["codes"].max() <= 126
    expect = np.take_along_axis(table[:, None, :], res["codes"].astype(np.int64).reshape(n_mats, 1, -1), axis=2)
    assert np.array_equal(expect.reshape(res["best_amax"].shape), res["best_amax"])

    workers = max(1, min(os.cpu_count() or 1, 96))
    step = max(1, -(-c_out // (4 * workers)))
    tasks = [(str(tmp_path), r0, min(c_out, r0 + step), gu.CODE_RTOL) for r0 in range(0, c_out, step)]
    with mp.get_context("spawn").Pool(workers) as pool:
        out = pool.map(oracle_shard.check_rows, tasks)
    exact = sum(o[0] for o in out)
    tol = sum(o[1] for o in out)
    fail = sum(o[2] for o in out)
    worst = max(o[3] for o in out)
    firsts = [o[4] for o in out if o[4] is not None]
    n = n_mats * c_out * (c_in // 16)
    assert exact + tol + fail == n
    assert fail == 0, (exact, tol, fail, worst, firsts[:3])
