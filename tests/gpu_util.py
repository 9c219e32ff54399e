"""Helpers for the GPU parity tests: run the CUDA library through its C ABI on
a synthetic layer, and compare against the oracle with the stated rules."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

HESSIAN_RTOL = 1e-5       # relative Frobenius error, per block and whole tensor
CODE_RTOL = 1e-6          # a differing code passes if its FP64 error is within 1e-6 of the minimum


def to_device(layer: synth.Layer):
    if layer.w_dtype == "bf16":
        W = torch.from_numpy(layer.W.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        W = torch.from_numpy(np.ascontiguousarray(layer.W)).cuda()
    X = torch.from_numpy(layer.X.view(np.int16)).view(torch.bfloat16).cuda()
    off = torch.from_numpy(layer.offsets).cuda() if layer.offsets is not None else None
    return W, X, off


def run_library(layer: synth.Layer, out_dtype=None, W=None, X=None, off=None):
    """absmax -> Hessian -> sweep (with its workspace) -> fake-quant through the C ABI; numpy results."""
    import scale_calibration_b200 as lh
    if W is None:
        W, X, off = to_device(layer)
    n_mats, c_out, c_in = W.shape
    n_groups = n_mats if off is not None else 1
    J = c_in // 16
    amax = torch.empty(n_mats, dtype=torch.float32, device="cuda")
    lh.lh_absmax(W, W, n_mats, c_out, c_in, W.stride(1), amax)
    H = torch.zeros(n_groups, J, 16, 16, dtype=torch.float32, device="cuda")
    wsb = lh.lh_hessian_workspace_bytes(X.shape[0], c_in, n_groups)
    ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device="cuda")
    lh.lh_accumulate_hessian(X, lh.LH_BF16, X.shape[0], c_in, X.stride(0), off, n_groups, H, ws, wsb)
    assert lh.lh_workspace_status(ws) == 0
    codes = torch.empty(n_mats, c_out, J, dtype=torch.uint8, device="cuda")
    bamax = torch.empty(n_mats, c_out, J, dtype=torch.float32, device="cuda")
    # the product path takes the sweep's workspace; the call without one must agree bit for bit
    swsb = lh.lh_sweep_workspace_bytes(n_mats, c_in)
    sws = torch.empty(max(swsb, 16), dtype=torch.uint8, device="cuda")
    lh.lh_sweep_scales_ws(W, W, n_mats, c_out, c_in, W.stride(1), amax, H, bamax, codes, sws, swsb)
    codes2 = torch.empty_like(codes)
    bamax2 = torch.empty_like(bamax)
    lh.lh_sweep_scales(W, W, n_mats, c_out, c_in, W.stride(1), amax, H, bamax2, codes2)
    assert torch.equal(codes, codes2) and torch.equal(bamax.view(torch.int32), bamax2.view(torch.int32))
    od = out_dtype or W.dtype
    Wq = torch.empty(n_mats, c_out, c_in, dtype=od, device="cuda")
    lh.lh_fake_quant(W, W, n_mats, c_out, c_in, W.stride(1), amax, codes, Wq, Wq)
    torch.cuda.synchronize()
    Wq_np = Wq.view(torch.int16).cpu().numpy().view(np.uint16) if od == torch.bfloat16 else Wq.cpu().numpy()
    return dict(amax=amax.cpu().numpy(), H=H.cpu().numpy(), codes=codes.cpu().numpy(),
                best_amax=bamax.cpu().numpy(), Wq=Wq_np)


def hessian_rel_errors(H_gpu: np.ndarray, H_ref: np.ndarray):
    """(worst per-block relative Frobenius error, whole-tensor error, #nonzero where ref is exactly zero)."""
    d = H_gpu.astype(np.float64) - H_ref
    nb = np.sqrt(np.sum(d * d, axis=(-1, -2)))
    nr = np.sqrt(np.sum(H_ref * H_ref, axis=(-1, -2)))
    zero = nr == 0
    per = np.where(zero, 0.0, nb / np.where(zero, 1.0, nr))
    whole = float(np.sqrt(np.sum(d * d)) / max(np.sqrt(np.sum(H_ref * H_ref)), 1e-300))
    bad_zero = int(np.count_nonzero(nb[zero]))
    return float(per.max(initial=0.0)), whole, bad_zero


def check_codes(W_f32, amax, H, codes_gpu, best_amax_gpu, mats=None, rows=None, cols=None):
    """Sweep parity against the oracle on all blocks, or on the listed (mat, row, col) blocks.
    Returns (#exact, #within-tolerance, #failures, worst relative gap)."""
    W3 = W_f32 if W_f32.ndim == 3 else W_f32[None]
    n_mats, c_out, c_in = W3.shape
    if mats is None:
        co, ao, eo = oracle.sweep(W3, amax, H)
        mats, rows, cols = (a.ravel() for a in np.meshgrid(np.arange(n_mats), np.arange(c_out),
                                                               np.arange(c_in // 16), indexing="ij"))
        co, ao, eo = co.ravel(), ao.ravel(), eo.ravel()
    else:
        co, ao, eo = oracle.sweep_blocks(W3, amax, H, mats, rows, cols)
    cg = codes_gpu[mats, rows, cols]
    ag = best_amax_gpu[mats, rows, cols]
    exact = cg == co
    n_tol, n_fail, worst = 0, 0, 0.0
    Hd = np.asarray(H, np.float64)
    for i in np.nonzero(~exact)[0]:
        m, r, j = int(mats[i]), int(rows[i]), int(cols[i])
        g = oracle.global_scale(amax[m])
        e_gpu = oracle.candidate_error(W3[m, r, 16 * j:16 * j + 16], g, int(cg[i]), Hd[m, j])
        gap = (e_gpu - eo[i]) / eo[i] if eo[i] > 0 else (0.0 if e_gpu == 0 else np.inf)
        worst = max(worst, gap)
        if gap <= CODE_RTOL:
            n_tol += 1
        else:
            n_fail += 1
    # amax is bit-exact given the code
    exp_amax = np.array([np.float32(6.0) * oracle.candidate_scale(int(c), oracle.global_scale(amax[int(m)]))
                         for c, m in zip(cg, mats)], np.float32)
    assert np.array_equal(ag, exp_amax), "best_amax differs from 6*s(code)"
    return int(exact.sum()), n_tol, n_fail, worst
