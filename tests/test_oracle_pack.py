"""Pins of the oracle's packed NVFP4 export (CPU).

The decoder here is written from the OCP E2M1 definition alone (1 sign bit, 2
exponent bits with bias 1, 1 mantissa bit; exponent field 0 is subnormal with
value m * 0.5), independent of the oracle: decoding the oracle's packed bytes
and scaling by fp32(e4m3(scale byte) * g) must give the oracle's fake-quantised
weights bit for bit (the fake-quant itself is pinned in test_oracle_pins.py)."""
import numpy as np

import oracle
import synth


def e2m1_decode(nib: np.ndarray) -> np.ndarray:
    s = (nib >> 3) & 1
    e = (nib >> 1) & 3
    m = nib & 1
    mag = np.where(e == 0, m * 0.5, np.ldexp(1.0 + m / 2.0, e.astype(np.int64) - 1))
    return np.where(s == 1, -mag, mag).astype(np.float32)


def unpack(packed: np.ndarray) -> np.ndarray:
    lo = packed & 0xF
    hi = packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * 2,))


def check(W, amax, codes):
    p, sc, gs = oracle.pack_nvfp4(W, amax, codes)
    W3 = W if W.ndim == 3 else W[None]
    n_mats, c_out, c_in = W3.shape
    assert np.array_equal(sc, codes.reshape(sc.shape))
    assert np.array_equal(gs, np.array([oracle.global_scale(a) for a in amax], np.float32))
    q = e2m1_decode(unpack(p))
    s = np.zeros(codes.shape, np.float32)
    for m in range(n_mats):
        for c in np.unique(codes[m]):
            s[m][codes[m] == c] = oracle.candidate_scale(int(c), gs[m])
    out = (q * np.repeat(s, 16, axis=-1)).astype(np.float32)
    ref = oracle.fake_quant(W3, amax, codes)
    assert np.array_equal(out.view(np.uint32), ref.reshape(out.shape).view(np.uint32))  # signed zeros too
    return p


def test_decode_table_is_the_e2m1_grid():
    vals = e2m1_decode(np.arange(16, dtype=np.uint8))
    assert list(vals[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(vals[8:]) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_pack_tiny_layer_random_codes():
    L = synth.make_config(0)
    W = L.W_f32()
    W3 = W if W.ndim == 3 else W[None]
    amax = np.array([oracle.absmax(W3[0])], np.float32)
    codes = np.random.default_rng(3).integers(1, 127, size=(1, W3.shape[1], W3.shape[2] // 16)).astype(np.uint8)
    check(W3, amax, codes)


def test_pack_every_code_and_sign():
    # one block per grid value and sign, with the scale chosen so w/s lands on it
    g_amax = np.float32(2688.0)          # g = 1
    vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)
    row = np.concatenate([vals, -vals]).astype(np.float32)
    W = np.tile(row, (1, 3, 1)).reshape(1, 3, 16)
    codes = np.array([[[0x38]], [[0x40]], [[0x30]]], np.uint8).reshape(1, 3, 1)  # s = 1, 2, 0.5
    p = check(W, np.array([g_amax]), codes)
    nibs = unpack(p)[0, 0]
    assert list(nibs) == list(range(8)) + [8 + i for i in range(8)]


def test_pack_zero_amax_keeps_the_sign_of_w():
    W = np.array([[[0.5, -0.25] * 8]], np.float32)
    p = check(W, np.array([0.0], np.float32), np.ones((1, 1, 1), np.uint8))
    assert list(unpack(p)[0, 0]) == [0, 8] * 8


def test_pack_nibble_order_even_column_low():
    W = np.zeros((1, 1, 16), np.float32)
    W[0, 0, 0] = 6.0   # column 0 -> low nibble of byte 0
    W[0, 0, 3] = -1.0  # column 3 -> high nibble of byte 1
    p = check(W, np.array([2688.0], np.float32), np.full((1, 1, 1), 0x38, np.uint8))
    assert p[0, 0, 0] == 0x07 and p[0, 0, 1] == 0xA0
