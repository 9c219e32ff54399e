"""Independent restatements used to pin the oracle (test helpers only).

Nothing here is shared with the oracle or with the CUDA library: these are
second, differently written statements of the format definitions (nearest
grid point by exhaustive distance, FP8 decoding by torch's float8 dtype) used
only to check the oracle against something other than itself.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import torch

# E2M1 magnitudes in code order 0..7 (sign-magnitude nibble 0.EE.M).
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float64)


def e4m3_values_torch() -> np.ndarray:
    """Values of all 256 E4M3 bytes decoded by torch.float8_e4m3fn."""
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def e2m1_nearest(u: np.ndarray) -> np.ndarray:
    """Nearest E2M1 grid value by exhaustive distance over the 8 magnitudes;
    on an exact tie the magnitude with an even code (mantissa bit 0) wins.
    Values beyond 6 land on 6 since it is the nearest grid point."""
    u = np.asarray(u, np.float32)
    x = np.abs(u.astype(np.float64))
    d = np.abs(x[..., None] - E2M1_GRID)            # exact in float64
    dmin = d.min(axis=-1, keepdims=True)
    hit = d == dmin
    idx = np.arange(8)
    even_hit = hit & (idx % 2 == 0)
    choose = np.where(even_hit.any(axis=-1), np.argmax(even_hit, axis=-1), np.argmax(hit, axis=-1))
    q = E2M1_GRID[choose]
    return np.where(np.signbit(u), -q, q)


def e2m1_nearest_fraction(u: float) -> float:
    """Slow exact-rational version of e2m1_nearest for single values."""
    x = abs(Fraction(float(np.float32(u))))
    best = None
    for k, gv in enumerate(E2M1_GRID):
        d = abs(x - Fraction(gv))
        key = (d, k % 2)          # smaller distance first, then even code
        if best is None or key < best[0]:
            best = (key, gv)
    q = best[1]
    return -q if np.signbit(np.float32(u)) else q


def candidate_dw(w16: np.ndarray, g: np.float32, v: float) -> tuple[np.ndarray, np.float32]:
    """dw = q*s - w for one candidate with value v (numpy FP32 ops for s and u)."""
    w = np.asarray(w16, np.float32)
    s = np.float32(np.float32(v) * np.float32(g))
    if s == 0:
        q = np.zeros(16)
    else:
        with np.errstate(divide="ignore", invalid="ignore"):
            u = (w / s).astype(np.float32)
        q = e2m1_nearest(u)
    return q * np.float64(s) - w.astype(np.float64), s


def mse_sweep_block(w16: np.ndarray, g: np.float32) -> int:
    """Plain weight-MSE 126-candidate sweep (sum of squared dw), lowest code wins ties."""
    vals = e4m3_values_torch()
    best, best_e = None, None
    for c in range(1, 127):
        dw, _ = candidate_dw(w16, g, vals[c])
        e = float(np.sum(dw * dw))
        if best_e is None or e < best_e:
            best, best_e = c, e
    return best


def max_scaling_code(block_amax: float, g: np.float32) -> int:
    """FP8 E4M3 code of amax_b / (6 g), rounded to nearest even by torch's
    float8 conversion after clamping to 448, then clamped to [1, 126]."""
    x = np.float32(np.float32(block_amax) / (np.float32(6.0) * np.float32(g)))
    x = min(float(x), 448.0)
    b = int(torch.tensor([x], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).item())
    return min(max(b, 1), 126)
