"""ctypes binding of liblh.so (include/lh.h): argument marshalling only.

Every function here has the name of the C entry point it calls and takes
device pointers either as torch CUDA tensors or as integers. Nothing here
computes any part of the calibration: all arithmetic runs in the library's
kernels. If liblh.so is missing the import fails; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblh.so")

LH_OK, LH_ERR_INVALID_ARG, LH_ERR_UNSUPPORTED, LH_ERR_ALIGNMENT, LH_ERR_WORKSPACE, LH_ERR_CUDA, LH_ERR_TIMEOUT = range(7)
LH_BF16, LH_F32 = 0, 1

EXPORTS = [
    "lh_status_string", "lh_last_error_message", "lh_absmax", "lh_hessian_workspace_bytes",
    "lh_accumulate_hessian", "lh_workspace_status", "lh_sweep_scales", "lh_fake_quant",
    "lh_accumulate_hessian_noalloc", "lh_noalloc_status", "lh_debug_wait_timeout", "lh_quantize_nvfp4", "lh_baseline_scales",
    "lh_search_amax", "lh_sweep_workspace_bytes", "lh_sweep_scales_ws", "lh_probe_fma", "lh_probe_fma_flop", "lh_debug_sweep_counts",
]
LH_SCALE_MAX, LH_SCALE_FOUR_OVER_SIX, LH_SCALE_MSE = range(3)


class LHError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {lh_status_string(status)}: {detail}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"liblh.so not built ({LIB_PATH}); run python scale_calibration_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sig = {
        "lh_status_string": (ctypes.c_char_p, [I32]),
        "lh_last_error_message": (ctypes.c_char_p, []),
        "lh_absmax": (I32, [P, I32, I64, I64, I64, I64, P, P]),
        "lh_hessian_workspace_bytes": (ctypes.c_size_t, [I64, I64, I64]),
        "lh_accumulate_hessian": (I32, [P, I32, I64, I64, I64, P, I64, P, P, ctypes.c_size_t, P]),
        "lh_workspace_status": (I32, [P, P]),
        "lh_accumulate_hessian_noalloc": (I32, [P, I32, I64, I64, I64, P, I64, P, P]),
        "lh_noalloc_status": (I32, [P]),
        "lh_debug_wait_timeout": (I32, [P, ctypes.c_size_t, I64, I32, P]),
        "lh_sweep_scales": (I32, [P, I32, I64, I64, I64, I64, P, P, P, P, P]),
        "lh_sweep_workspace_bytes": (ctypes.c_size_t, [I64, I64]),
        "lh_sweep_scales_ws": (I32, [P, I32, I64, I64, I64, I64, P, P, P, P, P, ctypes.c_size_t, P]),
        "lh_fake_quant": (I32, [P, I32, I64, I64, I64, I64, P, P, P, I32, P]),
        "lh_quantize_nvfp4": (I32, [P, I32, I64, I64, I64, I64, P, P, P, P, P, P, I32, P]),
        "lh_baseline_scales": (I32, [P, I32, I64, I64, I64, I64, P, I32, P, P, P]),
        "lh_search_amax": (I32, [P, I32, I64, I64, I64, I64, P, P, ctypes.c_double, ctypes.c_double, I64, P, P, P]),
        "lh_probe_fma_flop": (I64, [I64, I64]),
        "lh_probe_fma": (I32, [I32, I64, I64, P, P]),
        "lh_debug_sweep_counts": (I32, [P, I32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype(t) -> int:
    if isinstance(t, int):
        return t
    import torch
    if t.dtype == torch.bfloat16:
        return LH_BF16
    if t.dtype == torch.float32:
        return LH_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check(status: int, where: str) -> None:
    if status != LH_OK:
        raise LHError(status, where, lh_last_error_message())


def lh_status_string(status: int) -> str:
    return _lib.lh_status_string(status).decode()


def lh_last_error_message() -> str:
    return _lib.lh_last_error_message().decode()


def lh_absmax(W, w_dtype, n_mats, rows, cols, ld, out_amax, stream=None, check=True) -> int:
    s = _lib.lh_absmax(_ptr(W), _dtype(w_dtype), n_mats, rows, cols, ld, _ptr(out_amax), _stream(stream))
    if check:
        _check(s, "lh_absmax")
    return s


def lh_hessian_workspace_bytes(n_tokens_total, c_in, n_groups) -> int:
    return int(_lib.lh_hessian_workspace_bytes(n_tokens_total, c_in, n_groups))


def lh_accumulate_hessian(X, x_dtype, n_tokens_total, c_in, ld_x, offsets, n_groups, H, workspace,
                          workspace_bytes, stream=None, check=True) -> int:
    s = _lib.lh_accumulate_hessian(_ptr(X), _dtype(x_dtype), n_tokens_total, c_in, ld_x, _ptr(offsets), n_groups,
                                   _ptr(H), _ptr(workspace), workspace_bytes, _stream(stream))
    if check:
        _check(s, "lh_accumulate_hessian")
    return s


def lh_accumulate_hessian_noalloc(X, x_dtype, n_tokens_total, c_in, ld_x, offsets, n_groups, H, stream=None,
                                  check=True) -> int:
    """lh_accumulate_hessian with the workspace taken from the library's own
    fixed 8 MiB device array, for callers that cannot allocate device memory."""
    s = _lib.lh_accumulate_hessian_noalloc(_ptr(X), _dtype(x_dtype), n_tokens_total, c_in, ld_x, _ptr(offsets),
                                           n_groups, _ptr(H), _stream(stream))
    if check:
        _check(s, "lh_accumulate_hessian_noalloc")
    return s


def lh_debug_wait_timeout(workspace, workspace_bytes, timeout_us, arrive, stream=None, check=True) -> int:
    s = _lib.lh_debug_wait_timeout(_ptr(workspace), workspace_bytes, timeout_us, arrive, _stream(stream))
    if check:
        _check(s, "lh_debug_wait_timeout")
    return s


def lh_workspace_status(workspace, stream=None) -> int:
    return _lib.lh_workspace_status(_ptr(workspace), _stream(stream))


def lh_probe_fma_flop(blocks: int, iters: int) -> int:
    return _lib.lh_probe_fma_flop(blocks, iters)


def lh_probe_fma(packed: bool, blocks: int, iters: int, out, stream=None, check=True) -> int:
    """FP32 FMA throughput probe (diagnostics): time the launch with CUDA events."""
    s = _lib.lh_probe_fma(1 if packed else 0, blocks, iters, _ptr(out), _stream(stream))
    if check:
        _check(s, "lh_probe_fma")
    return s


def lh_noalloc_status(stream=None) -> int:
    return _lib.lh_noalloc_status(_stream(stream))


def lh_sweep_scales(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, H, best_amax, best_code, stream=None,
                    check=True) -> int:
    s = _lib.lh_sweep_scales(_ptr(W), _dtype(w_dtype), n_mats, c_out, c_in, ld_w, _ptr(global_amax), _ptr(H),
                             _ptr(best_amax), _ptr(best_code), _stream(stream))
    if check:
        _check(s, "lh_sweep_scales")
    return s


def lh_sweep_workspace_bytes(n_mats, c_in) -> int:
    return int(_lib.lh_sweep_workspace_bytes(n_mats, c_in))


def lh_sweep_scales_ws(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, H, best_amax, best_code, workspace,
                       workspace_bytes, stream=None, check=True) -> int:
    s = _lib.lh_sweep_scales_ws(_ptr(W), _dtype(w_dtype), n_mats, c_out, c_in, ld_w, _ptr(global_amax), _ptr(H),
                                _ptr(best_amax), _ptr(best_code), _ptr(workspace), workspace_bytes, _stream(stream))
    if check:
        _check(s, "lh_sweep_scales_ws")
    return s


def lh_fake_quant(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, codes, W_out, out_dtype, stream=None,
                  check=True) -> int:
    s = _lib.lh_fake_quant(_ptr(W), _dtype(w_dtype), n_mats, c_out, c_in, ld_w, _ptr(global_amax), _ptr(codes),
                           _ptr(W_out), _dtype(out_dtype), _stream(stream))
    if check:
        _check(s, "lh_fake_quant")
    return s


def lh_quantize_nvfp4(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, codes, packed, block_scales=None,
                      global_scale=None, W_out=None, out_dtype=LH_BF16, stream=None, check=True) -> int:
    s = _lib.lh_quantize_nvfp4(_ptr(W), _dtype(w_dtype), n_mats, c_out, c_in, ld_w, _ptr(global_amax), _ptr(codes),
                               _ptr(packed), _ptr(block_scales), _ptr(global_scale), _ptr(W_out),
                               _dtype(out_dtype), _stream(stream))
    if check:
        _check(s, "lh_quantize_nvfp4")
    return s


def lh_baseline_scales(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, method, best_amax, best_code, stream=None,
                       check=True) -> int:
    s = _lib.lh_baseline_scales(_ptr(W), _dtype(w_dtype), n_mats, c_out, c_in, ld_w, _ptr(global_amax), int(method),
                                _ptr(best_amax), _ptr(best_code), _stream(stream))
    if check:
        _check(s, "lh_baseline_scales")
    return s


def lh_search_amax(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, H, best_amax, best_code, start=0.25, step=0.1,
                   n_mult=38, stream=None, check=True) -> int:
    s = _lib.lh_search_amax(_ptr(W), _dtype(w_dtype), n_mats, c_out, c_in, ld_w, _ptr(global_amax), _ptr(H),
                            float(start), float(step), int(n_mult), _ptr(best_amax), _ptr(best_code), _stream(stream))
    if check:
        _check(s, "lh_search_amax")
    return s
