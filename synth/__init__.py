"""Seeded synthetic inputs for Local-Hessian calibration tests and benchmarks.

This module only draws random numbers: it holds none of the method's
arithmetic (no amax, no scales, no rounding to FP4/FP8). Both the oracle
tests and the CUDA parity tests feed its arrays to each side.

Weights and activations are drawn in FP32 with numpy's PCG64 generator and
rounded to bfloat16 (round to nearest even) where the layer is bf16. The five
layer recipes stand in for the layer shapes the calibration is run on (an
attention projection, MLP up/gate and down projections, a mixture-of-experts
expert bank); no dataset is involved.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 1000


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """FP32 -> bfloat16 bit patterns (uint16), round to nearest even; finite input."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    b = a.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> FP32 values (exact)."""
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Layer:
    """One calibration problem: n_mats weight matrices [c_out, c_in] that share
    the token axis layout of X [n_tok, c_in]; group g owns tokens
    [offsets[g], offsets[g+1]) and calibrates matrix g (offsets None: one group)."""
    name: str
    W: np.ndarray            # [n_mats, c_out, c_in]: uint16 bf16 bits, or float32 values
    w_dtype: str             # "bf16" | "f32"
    X: np.ndarray            # [n_tok, c_in] uint16 bf16 bits
    offsets: np.ndarray | None = None   # int64 [n_mats + 1] or None
    meta: dict = field(default_factory=dict)

    @property
    def n_mats(self) -> int:
        return self.W.shape[0]

    @property
    def c_out(self) -> int:
        return self.W.shape[1]

    @property
    def c_in(self) -> int:
        return self.W.shape[2]

    @property
    def n_tok(self) -> int:
        return self.X.shape[0]

    @property
    def n_blocks(self) -> int:
        return self.n_mats * self.c_out * (self.c_in // 16)

    def W_f32(self) -> np.ndarray:
        return bf16_bits_to_f32(self.W) if self.w_dtype == "bf16" else self.W


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _normal(rng, shape, scale=1.0):
    return rng.standard_normal(size=shape, dtype=np.float32) * np.float32(scale)


def zipf_counts(total: int, n: int, a: float) -> np.ndarray:
    """Deterministic proportional allocation of `total` tokens over n experts
    with weights k^-a (k = 1..n): floor of the shares, then the remainder to the
    largest fractional parts (ties to the lower rank)."""
    w = np.arange(1, n + 1, dtype=np.float64) ** (-a)
    share = total * w / w.sum()
    base = np.floor(share).astype(np.int64)
    rem = total - int(base.sum())
    frac = share - base
    order = np.lexsort((np.arange(n), -frac))
    base[order[:rem]] += 1
    return base


CONFIG_NAMES = ["tiny", "attn_proj", "mlp_up", "mlp_down", "moe_experts"]


def config_shapes(idx: int) -> dict:
    """Shapes of the five standard layers without drawing any data."""
    return [
        dict(name="tiny", n_mats=1, c_out=64, c_in=128, n_tok=256, w_dtype="f32"),
        dict(name="attn_proj", n_mats=1, c_out=4096, c_in=4096, n_tok=2048, w_dtype="bf16"),
        dict(name="mlp_up", n_mats=1, c_out=12288, c_in=4096, n_tok=8192, w_dtype="bf16"),
        dict(name="mlp_down", n_mats=1, c_out=5120, c_in=17408, n_tok=16384, w_dtype="bf16"),
        dict(name="moe_experts", n_mats=64, c_out=1536, c_in=2048, n_tok=32768, w_dtype="bf16"),
    ][idx]


def make_config(idx: int, seed: int | None = None) -> Layer:
    """The five standard layers, seeded with SEED_BASE + idx by default.

    0 tiny:        W [64,128] fp32 ~N(0,0.02); X [256,128] ~N(0,1), 4 channels x20.
    1 attn_proj:   W [4096,4096] ~N(0,0.02), round(0.001*numel) entries x8;
                   X [2048,4096] = N(0,1) * l_c, l_c ~ lognormal(0,1) per channel.
    2 mlp_up:      W [12288,4096] ~ Student-t(4) * 0.015;
                   X [8192,4096] = N(0,1) * l_c, l_c ~ lognormal(0,1.5); 8 channels x50.
    3 mlp_down:    W [5120,17408] ~N(0,0.01); X [16384,17408]: 0 with p=0.6, else
                   |N(0,1)| * l_c, l_c ~ lognormal(0,1).
    4 moe_experts: 64 x W [1536,2048] ~N(0,0.02); X [32768,2048] ~N(0,1) sorted by
                   expert, counts from zipf_counts(32768, 64, 1.1).
    """
    rng = _rng(SEED_BASE + idx if seed is None else seed)
    sh = config_shapes(idx)
    name = sh["name"]
    if idx == 0:
        W = _normal(rng, (1, 64, 128), 0.02)
        X = _normal(rng, (256, 128))
        ch = rng.choice(128, size=4, replace=False)
        X[:, ch] *= np.float32(20.0)
        return Layer(name, W, "f32", f32_to_bf16_bits(X), None, dict(outlier_channels=ch.tolist()))
    if idx == 1:
        W = _normal(rng, (4096 * 4096,), 0.02)
        n_out = int(round(0.001 * W.size))
        pos = rng.choice(W.size, size=n_out, replace=False)
        W[pos] *= np.float32(8.0)
        lc = rng.lognormal(0.0, 1.0, size=4096).astype(np.float32)
        X = _normal(rng, (2048, 4096)) * lc[None, :]
        return Layer(name, f32_to_bf16_bits(W.reshape(1, 4096, 4096)), "bf16", f32_to_bf16_bits(X),
                     None, dict(n_outliers=n_out))
    if idx == 2:
        W = (rng.standard_t(4.0, size=(1, 12288, 4096)) * 0.015).astype(np.float32)
        lc = rng.lognormal(0.0, 1.5, size=4096).astype(np.float32)
        ch = rng.choice(4096, size=8, replace=False)
        lc[ch] *= np.float32(50.0)
        X = _normal(rng, (8192, 4096)) * lc[None, :]
        return Layer(name, f32_to_bf16_bits(W), "bf16", f32_to_bf16_bits(X), None,
                     dict(outlier_channels=ch.tolist()))
    if idx == 3:
        W = _normal(rng, (1, 5120, 17408), 0.01)
        lc = rng.lognormal(0.0, 1.0, size=17408).astype(np.float32)
        Xb = np.empty((16384, 17408), np.uint16)
        step = 1024
        for t0 in range(0, 16384, step):
            z = rng.random(size=(step, 17408), dtype=np.float32) < np.float32(0.6)
            v = np.abs(_normal(rng, (step, 17408))) * lc[None, :]
            v[z] = 0.0
            Xb[t0:t0 + step] = f32_to_bf16_bits(v)
        return Layer(name, f32_to_bf16_bits(W), "bf16", Xb, None, {})
    if idx == 4:
        W = _normal(rng, (64, 1536, 2048), 0.02)
        counts = zipf_counts(32768, 64, 1.1)
        X = _normal(rng, (32768, 2048))
        off = np.zeros(65, np.int64)
        off[1:] = np.cumsum(counts)
        return Layer(name, f32_to_bf16_bits(W), "bf16", f32_to_bf16_bits(X), off,
                     dict(counts=counts.tolist()))
    raise ValueError(idx)


def make_layer(c_out: int, c_in: int, n_tok: int, seed: int, n_mats: int = 1, w_dtype: str = "bf16",
               w_std: float = 0.02, counts=None, x_lognormal: float = 1.0, sparse: float = 0.0,
               outlier_frac: float = 0.0) -> Layer:
    """A small random layer for parity cases (ragged sizes, groups, sparsity)."""
    rng = _rng(seed)
    W = _normal(rng, (n_mats, c_out, c_in), w_std)
    if outlier_frac > 0:
        k = max(1, int(round(outlier_frac * W.size)))
        pos = rng.choice(W.size, size=k, replace=False)
        W.reshape(-1)[pos] *= np.float32(8.0)
    lc = rng.lognormal(0.0, x_lognormal, size=c_in).astype(np.float32) if x_lognormal > 0 else \
        np.ones(c_in, np.float32)
    X = _normal(rng, (n_tok, c_in)) * lc[None, :]
    if sparse > 0:
        X = np.abs(X)
        X[rng.random(size=X.shape) < sparse] = 0.0
    off = None
    if counts is not None:
        counts = np.asarray(counts, np.int64)
        assert counts.sum() == n_tok and len(counts) == n_mats
        off = np.zeros(n_mats + 1, np.int64)
        off[1:] = np.cumsum(counts)
    Wout = f32_to_bf16_bits(W) if w_dtype == "bf16" else W
    return Layer(f"layer_{c_out}x{c_in}_t{n_tok}_s{seed}", Wout, w_dtype, f32_to_bf16_bits(X), off, {})
