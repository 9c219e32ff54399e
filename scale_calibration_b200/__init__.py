"""Local-Hessian NVFP4 block-scale calibration for B200 (sm_100a).

The work happens in liblh.so (C ABI in include/lh.h); this package is its
ctypes binding plus `calibrate`, which chains the four calls of the hot path
for one layer:

    lh_absmax -> lh_accumulate_hessian -> lh_sweep_scales_ws -> lh_fake_quant

Method: "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块
权重缩放算法实战指南" (xxmr.cn/news/266017), sections "算法原理" and
"入口 API 与校准流程".
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    EXPORTS, LH_BF16, LH_F32, LH_OK, LHError, lh_absmax, lh_accumulate_hessian, lh_fake_quant,
    lh_accumulate_hessian_noalloc, lh_noalloc_status, lh_debug_wait_timeout, lh_hessian_workspace_bytes, lh_last_error_message, lh_status_string,
    lh_quantize_nvfp4, lh_sweep_scales, lh_workspace_status, lh_baseline_scales, LH_SCALE_MAX,
    LH_SCALE_FOUR_OVER_SIX, LH_SCALE_MSE, lh_search_amax, lh_sweep_scales_ws, lh_sweep_workspace_bytes,
    lh_probe_fma, lh_probe_fma_flop,
)


class Calibrator:
    """Device buffers for calibrating one layer shape; `run` launches the
    whole hot path on the current stream. Inputs are torch CUDA tensors:
    W [n_mats, c_out, c_in] (bf16 or f32), X [n_tok, c_in] bf16, optional
    offsets int64 [n_mats + 1] on the device (one token group per matrix)."""

    def __init__(self, n_mats: int, c_out: int, c_in: int, n_tok: int, grouped: bool, out_dtype=None,
                 device="cuda"):
        import torch
        self.n_mats, self.c_out, self.c_in, self.n_tok = n_mats, c_out, c_in, n_tok
        self.grouped = grouped
        if not grouped and n_mats > 1:
            raise ValueError("several matrices need grouped tokens (offsets, one group per matrix)")
        J = c_in // 16
        n_groups = n_mats if grouped else 1
        self.n_groups = n_groups
        self.out_dtype = out_dtype
        self.amax = torch.empty(n_mats, dtype=torch.float32, device=device)
        self.H = torch.zeros(n_groups, J, 16, 16, dtype=torch.float32, device=device)
        self.ws_bytes = lh_hessian_workspace_bytes(n_tok, c_in, n_groups)
        self.ws = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=device)
        self.sweep_ws_bytes = lh_sweep_workspace_bytes(n_mats, c_in)
        self.sweep_ws = torch.empty(max(self.sweep_ws_bytes, 16), dtype=torch.uint8, device=device)
        self.best_amax = torch.empty(n_mats, c_out, J, dtype=torch.float32, device=device)
        self.best_code = torch.empty(n_mats, c_out, J, dtype=torch.uint8, device=device)
        self.Wq = None

    def run(self, W, X, offsets=None, stream=None, zero_h: bool = True):
        import torch
        n_mats, c_out, c_in = self.n_mats, self.c_out, self.c_in
        if self.Wq is None or self.Wq.dtype != (self.out_dtype or W.dtype):
            self.Wq = torch.empty(n_mats, c_out, c_in, dtype=self.out_dtype or W.dtype, device=W.device)
        if zero_h:
            self.H.zero_()
        lh_absmax(W, W, n_mats, c_out, c_in, W.stride(-2), self.amax, stream)
        lh_accumulate_hessian(X, LH_BF16, X.shape[0], c_in, X.stride(0), offsets if self.grouped else None,
                              self.n_groups, self.H, self.ws, self.ws_bytes, stream)
        lh_sweep_scales_ws(W, W, n_mats, c_out, c_in, W.stride(-2), self.amax, self.H, self.best_amax,
                           self.best_code, self.sweep_ws, self.sweep_ws_bytes, stream)
        lh_fake_quant(W, W, n_mats, c_out, c_in, W.stride(-2), self.amax, self.best_code, self.Wq, self.Wq, stream)
        return self.best_code, self.best_amax, self.Wq


def calibrate(W, X, offsets=None, out_dtype=None, stream=None):
    """One-shot Local-Hessian calibration of a layer (see Calibrator)."""
    if W.dim() == 2:
        W = W.unsqueeze(0)
    cal = Calibrator(W.shape[0], W.shape[1], W.shape[2], X.shape[0], offsets is not None, out_dtype,
                     device=W.device)
    codes, amax, Wq = cal.run(W, X, offsets, stream)
    return dict(codes=codes, best_amax=amax, Wq=Wq, H=cal.H, global_amax=cal.amax)
