"""Worker for the all-blocks parity test: sweeps a row range of a saved layer
with the oracle and compares it with the GPU's codes. Imports only numpy and
the oracle, so spawned processes start quickly."""
from __future__ import annotations

import os

import numpy as np

import oracle


def check_rows(args):
    """args = (directory, first row, end row, relative tolerance). The directory
    holds W.npy (FP32 [n_mats, c_out, c_in]), H.npy (the GPU's H, [n_mats, J, 16, 16]),
    amax.npy and codes.npy (the GPU's codes). Returns (#exact, #within tolerance,
    #failures, worst relative gap, first failure or None)."""
    d, r0, r1, rtol = args
    W = np.load(os.path.join(d, "W.npy"), mmap_mode="r")
    H = np.load(os.path.join(d, "H.npy"), mmap_mode="r")
    amax = np.load(os.path.join(d, "amax.npy"))
    codes = np.load(os.path.join(d, "codes.npy"), mmap_mode="r")
    Ws = np.ascontiguousarray(W[:, r0:r1, :])
    Hd = np.asarray(H, np.float64)
    co, _, eo = oracle.sweep(Ws, amax, Hd)
    cg = np.asarray(codes[:, r0:r1, :])
    diff = np.nonzero(co != cg)
    n_tol = n_fail = 0
    worst = 0.0
    first = None
    for m, r, j in zip(*diff):
        g = oracle.global_scale(amax[m])
        e_gpu = oracle.candidate_error(Ws[m, r, 16 * j:16 * j + 16], g, int(cg[m, r, j]), Hd[m, j])
        e_min = eo[m, r, j]
        gap = (e_gpu - e_min) / e_min if e_min > 0 else (0.0 if e_gpu == e_min else np.inf)
        worst = max(worst, gap)
        if gap <= rtol:
            n_tol += 1
        else:
            n_fail += 1
            if first is None:
                first = (int(m), int(r0 + r), int(j), int(cg[m, r, j]), int(co[m, r, j]), float(gap))
    return int(co.size - len(diff[0])), n_tol, n_fail, worst, first
