"""Oracle for Local-Hessian NVFP4 block-scale calibration (test infrastructure).

This package is the plain, slow, single-threaded FP64 CPU statement of the
calibration hot path (``lh_oracle.cpp``) plus a ctypes wrapper. It exists to
check the CUDA library; only the tests, the smoke check and the CPU-baseline
leg of ``bench.py`` may import it. It shares no code with
``scale_calibration_b200`` and imports nothing from it.

Sources: "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4
逐块权重缩放算法实战指南" (xxmr.cn/news/266017), sections "Local-Hessian 是什么"
and "算法原理"; see ``lh_oracle.cpp`` for the function-by-function citations.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lh_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile lh_oracle.cpp into liboracle.so (plain g++, no GPU code)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *_CXXFLAGS, _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_int]
        lib.oracle_e2m1_rne.restype = F
        lib.oracle_e2m1_rne.argtypes = [F]
        lib.oracle_float_to_bf16.restype = ctypes.c_uint16
        lib.oracle_float_to_bf16.argtypes = [F]
        lib.oracle_absmax.restype = F
        lib.oracle_absmax.argtypes = [P, I64, I64, I64]
        lib.oracle_global_scale.restype = F
        lib.oracle_global_scale.argtypes = [F]
        lib.oracle_candidate_scale.restype = F
        lib.oracle_candidate_scale.argtypes = [ctypes.c_int, F]
        lib.oracle_hessian.restype = None
        lib.oracle_hessian.argtypes = [P, I64, I64, I64, P, I64, P]
        lib.oracle_candidate_error.restype = ctypes.c_double
        lib.oracle_candidate_error.argtypes = [P, F, ctypes.c_int, P]
        lib.oracle_block_errors.restype = None
        lib.oracle_block_errors.argtypes = [P, F, P, P]
        lib.oracle_block_argmin.restype = ctypes.c_int
        lib.oracle_block_argmin.argtypes = [P, F, P, P, P]
        lib.oracle_sweep.restype = None
        lib.oracle_sweep.argtypes = [P, I64, I64, I64, I64, P, P, P, P, P]
        lib.oracle_sweep_blocks.restype = None
        lib.oracle_sweep_blocks.argtypes = [P, I64, I64, I64, P, P, P, P, P, I64, P, P, P]
        lib.oracle_fake_quant_f32.restype = None
        lib.oracle_fake_quant_f32.argtypes = [P, I64, I64, I64, I64, P, P, P]
        lib.oracle_fake_quant_bf16.restype = None
        lib.oracle_fake_quant_bf16.argtypes = [P, I64, I64, I64, I64, P, P, P]
        lib.oracle_pack_nvfp4.restype = None
        lib.oracle_pack_nvfp4.argtypes = [P, I64, I64, I64, I64, P, P, P, P, P]
        lib.oracle_e4m3_rne.restype = ctypes.c_int
        lib.oracle_e4m3_rne.argtypes = [F]
        lib.oracle_baseline_scales.restype = None
        lib.oracle_baseline_scales.argtypes = [P, I64, I64, I64, I64, P, ctypes.c_int, P, P]
        D = ctypes.c_double
        lib.oracle_amax_search.restype = None
        lib.oracle_amax_search.argtypes = [P, I64, I64, I64, I64, P, P, D, D, I64, P, P, P]
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- formats
def e4m3_value(code: int) -> float:
    return _L().oracle_e4m3_value(int(code))


def e2m1_rne(u: float) -> float:
    return _L().oracle_e2m1_rne(float(np.float32(u)))


def float_to_bf16_bits(x: float) -> int:
    return int(_L().oracle_float_to_bf16(float(np.float32(x))))


def global_scale(amax: float) -> np.float32:
    return np.float32(_L().oracle_global_scale(float(np.float32(amax))))


def candidate_scale(code: int, g: float) -> np.float32:
    return np.float32(_L().oracle_candidate_scale(int(code), float(np.float32(g))))


# --------------------------------------------------------------------------- steps
def absmax(W: np.ndarray) -> np.float32:
    """max |W| of a 2-D FP32 matrix."""
    W = _c(W, np.float32)
    return np.float32(_L().oracle_absmax(_p(W), W.shape[0], W.shape[1], W.shape[1]))


def hessian(X_bf16_bits: np.ndarray, c_in: int | None = None, offsets=None) -> np.ndarray:
    """Local Hessians in FP64. X: uint16 bf16 bits [n_tok, ld]. Returns
    [n_groups, c_in/16, 16, 16] (n_groups = 1 when offsets is None)."""
    X = _c(X_bf16_bits, np.uint16)
    n_tok, ld = X.shape
    c_in = ld if c_in is None else c_in
    J = c_in // 16
    if offsets is None:
        H = np.zeros((1, J, 16, 16), np.float64)
        _L().oracle_hessian(_p(X), n_tok, c_in, ld, None, 1, _p(H))
    else:
        off = _c(offsets, np.int64)
        G = off.shape[0] - 1
        H = np.zeros((G, J, 16, 16), np.float64)
        _L().oracle_hessian(_p(X), n_tok, c_in, ld, _p(off), G, _p(H))
    return H


def candidate_error(w16, g, code, H16) -> float:
    w = _c(w16, np.float32)
    H = _c(H16, np.float64)
    return _L().oracle_candidate_error(_p(w), float(np.float32(g)), int(code), _p(H))


def block_errors(w16, g, H16) -> np.ndarray:
    w = _c(w16, np.float32)
    H = _c(H16, np.float64)
    out = np.zeros(126, np.float64)
    _L().oracle_block_errors(_p(w), float(np.float32(g)), _p(H), _p(out))
    return out


def sweep(W: np.ndarray, global_amax, H: np.ndarray):
    """W: FP32 [n_mats, c_out, c_in] (or 2-D); global_amax [n_mats];
    H: [n_mats, c_in/16, 16, 16] (any float dtype, promoted to FP64).
    Returns (codes u8, amax f32, err f64) of shape [n_mats, c_out, c_in/16]."""
    W = _c(W, np.float32)
    if W.ndim == 2:
        W = W[None]
    n_mats, c_out, c_in = W.shape
    J = c_in // 16
    ga = _c(np.atleast_1d(global_amax), np.float32)
    Hd = _c(H, np.float64).reshape(n_mats, J, 16, 16)
    code = np.zeros((n_mats, c_out, J), np.uint8)
    amax = np.zeros((n_mats, c_out, J), np.float32)
    err = np.zeros((n_mats, c_out, J), np.float64)
    _L().oracle_sweep(_p(W), n_mats, c_out, c_in, c_in, _p(ga), _p(Hd), _p(code), _p(amax), _p(err))
    return code, amax, err


def sweep_blocks(W: np.ndarray, global_amax, H: np.ndarray, mats, rows, cols):
    """Sweep only the listed blocks (mat, row, block column)."""
    W = _c(W, np.float32)
    if W.ndim == 2:
        W = W[None]
    n_mats, c_out, c_in = W.shape
    J = c_in // 16
    ga = _c(np.atleast_1d(global_amax), np.float32)
    Hd = _c(H, np.float64).reshape(n_mats, J, 16, 16)
    mats, rows, cols = (_c(a, np.int64) for a in (mats, rows, cols))
    n = mats.shape[0]
    code = np.zeros(n, np.uint8)
    amax = np.zeros(n, np.float32)
    err = np.zeros(n, np.float64)
    _L().oracle_sweep_blocks(_p(W), c_out, c_in, c_in, _p(ga), _p(Hd), _p(mats), _p(rows), _p(cols),
                             n, _p(code), _p(amax), _p(err))
    return code, amax, err


def fake_quant(W: np.ndarray, global_amax, codes: np.ndarray, out_bf16: bool = False) -> np.ndarray:
    """Fake-quantised W with the given codes. Returns FP32 values, or uint16
    bf16 bits when out_bf16."""
    W = _c(W, np.float32)
    squeeze = W.ndim == 2
    if squeeze:
        W = W[None]
    n_mats, c_out, c_in = W.shape
    ga = _c(np.atleast_1d(global_amax), np.float32)
    cd = _c(codes, np.uint8).reshape(n_mats, c_out, c_in // 16)
    if out_bf16:
        out = np.zeros(W.shape, np.uint16)
        _L().oracle_fake_quant_bf16(_p(W), n_mats, c_out, c_in, c_in, _p(ga), _p(cd), _p(out))
    else:
        out = np.zeros(W.shape, np.float32)
        _L().oracle_fake_quant_f32(_p(W), n_mats, c_out, c_in, c_in, _p(ga), _p(cd), _p(out))
    return out[0] if squeeze else out


def e4m3_rne(x: float) -> int:
    """E4M3 code of x >= 0, round to nearest even, saturating at 448."""
    return int(_L().oracle_e4m3_rne(float(x)))


BASELINE_MAX, BASELINE_FOUR_OVER_SIX = 0, 1


def baseline_scales(W: np.ndarray, global_amax, method: int):
    """Max scaling (method 0) or four-over-six (method 1): (codes u8, amax f32)
    of shape [n_mats, c_out, c_in/16]. The MSE baseline is sweep() with H = I."""
    W = _c(W, np.float32)
    if W.ndim == 2:
        W = W[None]
    n_mats, c_out, c_in = W.shape
    ga = _c(np.atleast_1d(global_amax), np.float32)
    code = np.zeros((n_mats, c_out, c_in // 16), np.uint8)
    amax = np.zeros((n_mats, c_out, c_in // 16), np.float32)
    _L().oracle_baseline_scales(_p(W), n_mats, c_out, c_in, c_in, _p(ga), int(method), _p(code), _p(amax))
    return code, amax


def amax_search(W: np.ndarray, global_amax, H: np.ndarray, start=0.25, step=0.1, n_mult=38):
    """Amax multiplier search with the Hessian metric: (codes u8, amax f32, err f64)
    of shape [n_mats, c_out, c_in/16]."""
    W = _c(W, np.float32)
    if W.ndim == 2:
        W = W[None]
    n_mats, c_out, c_in = W.shape
    J = c_in // 16
    ga = _c(np.atleast_1d(global_amax), np.float32)
    Hd = _c(H, np.float64).reshape(n_mats, J, 16, 16)
    code = np.zeros((n_mats, c_out, J), np.uint8)
    amax = np.zeros((n_mats, c_out, J), np.float32)
    err = np.zeros((n_mats, c_out, J), np.float64)
    _L().oracle_amax_search(_p(W), n_mats, c_out, c_in, c_in, _p(ga), _p(Hd), float(start), float(step), int(n_mult),
                            _p(code), _p(amax), _p(err))
    return code, amax, err


def pack_nvfp4(W: np.ndarray, global_amax, codes: np.ndarray):
    """Packed NVFP4 of W with the given codes: (packed u8 [n_mats, c_out, c_in/2],
    block scale bytes u8 [n_mats, c_out, c_in/16], global scale f32 [n_mats])."""
    W = _c(W, np.float32)
    if W.ndim == 2:
        W = W[None]
    n_mats, c_out, c_in = W.shape
    ga = _c(np.atleast_1d(global_amax), np.float32)
    cd = _c(codes, np.uint8).reshape(n_mats, c_out, c_in // 16)
    packed = np.zeros((n_mats, c_out, c_in // 2), np.uint8)
    scales = np.zeros((n_mats, c_out, c_in // 16), np.uint8)
    gs = np.zeros(n_mats, np.float32)
    _L().oracle_pack_nvfp4(_p(W), n_mats, c_out, c_in, c_in, _p(ga), _p(cd), _p(packed), _p(scales), _p(gs))
    return packed, scales, gs


def errors_for_codes(W: np.ndarray, global_amax, H: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """FP64 error E(code) of given codes, per block (slow; small inputs)."""
    W = _c(W, np.float32)
    if W.ndim == 2:
        W = W[None]
    n_mats, c_out, c_in = W.shape
    J = c_in // 16
    ga = np.atleast_1d(np.asarray(global_amax, np.float32))
    Hd = _c(H, np.float64).reshape(n_mats, J, 16, 16)
    cd = np.asarray(codes).reshape(n_mats, c_out, J)
    out = np.zeros((n_mats, c_out, J), np.float64)
    lib = _L()
    for m in range(n_mats):
        g = float(global_scale(ga[m]))
        for r in range(c_out):
            for j in range(J):
                w = np.ascontiguousarray(W[m, r, 16 * j:16 * j + 16])
                h = np.ascontiguousarray(Hd[m, j])
                out[m, r, j] = lib.oracle_candidate_error(_p(w), g, int(cd[m, r, j]), _p(h))
    return out
