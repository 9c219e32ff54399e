"""Pins of the oracle to what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: a library
decoder, an exhaustive or exact-rational restatement, a closed form, a brute
force over tiny inputs, or an invariance of the method. Sources: "NVIDIA
Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块权重缩放算法实战指南"
(xxmr.cn/news/266017), sections "Local-Hessian 是什么" and "算法原理".
"""
import itertools

import numpy as np
import pytest

import oracle
import synth
from tests import indep


# ----------------------------------------------------------------------------- formats
def test_e4m3_decode_matches_torch_float8():
    ref = indep.e4m3_values_torch()
    ours = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ref[~nan], ours[~nan])


def test_e4m3_candidate_set():
    # "Local-Hessian 是什么": the sweep covers the 126 positive, non-zero finite
    # FP8 values; E4M3 has 128 positive bit patterns, 0x00 is zero, 0x7F NaN.
    v = np.array([oracle.e4m3_value(c) for c in range(128)])
    cand = [c for c in range(128) if np.isfinite(v[c]) and v[c] > 0]
    assert cand == list(range(1, 127))
    assert v[1] == 2.0 ** -9 and v[0x7E] == 448.0
    assert np.all(np.diff(v[1:127]) > 0)


def _tie_points():
    pts = []
    for t in [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5, 1.0, 2.0, 4.0]:
        t32 = np.float32(t)
        pts += [t32, np.nextafter(t32, np.float32(0)), np.nextafter(t32, np.float32(10))]
    return np.array(pts, np.float32)


def test_e2m1_rne_exact_rational_on_ties():
    vals = np.concatenate([_tie_points(), -_tie_points(), np.float32([0.0, -0.0, 7.0, 1e30, 1e-30])])
    for u in vals:
        assert oracle.e2m1_rne(u) == indep.e2m1_nearest_fraction(u), u


def test_e2m1_rne_dense_against_exhaustive_distance():
    rng = np.random.default_rng(0)
    u = np.concatenate([np.linspace(-8, 8, 40001, dtype=np.float32),
                        rng.uniform(-7, 7, 20000).astype(np.float32), _tie_points()])
    ours = np.array([oracle.e2m1_rne(x) for x in u])
    assert np.array_equal(ours, indep.e2m1_nearest(u))
    # signs of zero follow the input
    assert np.signbit(oracle.e2m1_rne(np.float32(-0.1)))


def test_e2m1_tie_directions():
    # ties go to the even E2M1 code: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    exp = {0.25: 0, 0.75: 1, 1.25: 1, 1.75: 2, 2.5: 2, 3.5: 4, 5.0: 4}
    for t, q in exp.items():
        assert oracle.e2m1_rne(t) == q and oracle.e2m1_rne(-t) == -q


def test_global_scale_is_one_fp32_division():
    rng = np.random.default_rng(1)
    for a in rng.uniform(1e-6, 100, 1000).astype(np.float32):
        assert oracle.global_scale(a) == np.float32(a) / np.float32(2688.0)
    assert oracle.global_scale(0.0) == 0.0


def test_candidate_scale_is_fp32_product():
    vals = indep.e4m3_values_torch()
    g = np.float32(0.0123456)
    for c in range(1, 127):
        assert oracle.candidate_scale(c, g) == np.float32(np.float32(vals[c]) * g)


def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        np.float32([1.00390625, 1.01171875, -3.0e-3])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([oracle.float_to_bf16_bits(v) for v in x], np.uint16)
    assert np.array_equal(ref, ours)


# ----------------------------------------------------------------------------- Hessian
def _bits(x):
    return synth.f32_to_bf16_bits(np.asarray(x, np.float32))


def test_hessian_one_hot_tokens_give_counts():
    rng = np.random.default_rng(3)
    c_in, n = 48, 500
    idx = rng.integers(0, c_in, n)
    X = np.zeros((n, c_in), np.float32)
    X[np.arange(n), idx] = 1.0
    H = oracle.hessian(_bits(X))[0]
    counts = np.bincount(idx, minlength=c_in)
    for j in range(c_in // 16):
        assert np.array_equal(H[j], np.diag(counts[16 * j:16 * j + 16]).astype(np.float64))


def test_hessian_constant_token_is_rank_one():
    rng = np.random.default_rng(4)
    x = synth.bf16_bits_to_f32(_bits(rng.standard_normal(32)))
    X = np.tile(x, (37, 1))
    H = oracle.hessian(_bits(X))[0]
    for j in range(2):
        xb = x[16 * j:16 * j + 16].astype(np.float64)
        assert np.allclose(H[j], 37 * np.outer(xb, xb), rtol=1e-15, atol=0)


def test_hessian_matches_numpy_gram_groups_and_ld():
    rng = np.random.default_rng(5)
    n, c_in, ld = 300, 64, 80
    Xf = synth.bf16_bits_to_f32(_bits(rng.standard_normal((n, ld)) * rng.lognormal(0, 1, ld)))
    off = np.array([0, 7, 7, 150, 300])
    H = oracle.hessian(_bits(Xf), c_in=c_in, offsets=off)
    assert H.shape == (4, 4, 16, 16)
    for g in range(4):
        Xg = Xf[off[g]:off[g + 1], :c_in].astype(np.float64)
        for j in range(4):
            B = Xg[:, 16 * j:16 * j + 16]
            assert np.allclose(H[g, j], B.T @ B, rtol=1e-13, atol=1e-300)
    assert np.all(H[1] == 0)  # empty group


def test_hessian_token_permutation_invariant_and_psd():
    rng = np.random.default_rng(6)
    X = _bits(rng.standard_normal((200, 32)))
    H1 = oracle.hessian(X)[0]
    H2 = oracle.hessian(X[rng.permutation(200)])[0]
    assert np.allclose(H1, H2, rtol=1e-14)
    for j in range(2):
        assert np.allclose(H1[j], H1[j].T)
        assert np.linalg.eigvalsh(H1[j]).min() > -1e-9 * np.abs(H1[j]).max()


# ----------------------------------------------------------------------------- error E(s)
def _tiny_layer(seed, c_out, c_in, n_tok, disjoint=False):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((c_out, c_in)) * 0.02).astype(np.float32)
    Xf = (rng.standard_normal((n_tok, c_in)) * rng.lognormal(0, 1, c_in)).astype(np.float32)
    if disjoint:  # each token touches only one 16-channel block
        blk = np.arange(n_tok) % (c_in // 16)
        mask = (np.arange(c_in)[None, :] // 16) == blk[:, None]
        Xf = np.where(mask, Xf, 0).astype(np.float32)
    Xb = _bits(Xf)
    return W, Xb, synth.bf16_bits_to_f32(Xb).astype(np.float64)


def test_candidate_error_equals_output_error_of_one_block():
    # "算法原理": E(s) = ||Delta X||_F^2 = tr(Delta (X X^T) Delta^T); for one block
    # the local Hessian is X_b X_b^T. dw here is recomputed independently.
    W, Xb, X = _tiny_layer(7, 1, 16, 64)
    H = oracle.hessian(Xb)[0, 0]
    g = oracle.global_scale(np.abs(W).max())
    vals = indep.e4m3_values_torch()
    for c in range(1, 127):
        dw, _ = indep.candidate_dw(W[0], g, vals[c])
        direct = float(np.sum((X @ dw) ** 2))
        assert oracle.candidate_error(W[0], g, c, H) == pytest.approx(direct, rel=1e-12, abs=1e-300)


def test_blockwise_sum_equals_full_error_when_cross_terms_vanish():
    # With tokens that touch one block each, ||Delta X||_F^2 = sum_b dw_b^T H_b dw_b.
    W, Xb, X = _tiny_layer(8, 3, 64, 96, disjoint=True)
    H = oracle.hessian(Xb)[0]
    A = np.abs(W).max()
    codes, _, err = oracle.sweep(W, [A], H)
    g = oracle.global_scale(A)
    vals = indep.e4m3_values_torch()
    D = np.zeros(W.shape, np.float64)
    for r in range(3):
        for j in range(4):
            D[r, 16 * j:16 * j + 16], _ = indep.candidate_dw(W[r, 16 * j:16 * j + 16], g, vals[codes[0, r, j]])
    full = float(np.sum((D @ X.T) ** 2))
    assert err.sum() == pytest.approx(full, rel=1e-12)


def test_full_error_is_blockwise_plus_cross_terms():
    W, Xb, X = _tiny_layer(9, 2, 32, 80)
    H = oracle.hessian(Xb)[0]
    A = np.abs(W).max()
    codes, _, err = oracle.sweep(W, [A], H)
    g = oracle.global_scale(A)
    vals = indep.e4m3_values_torch()
    full = 0.0
    for r in range(2):
        d = [indep.candidate_dw(W[r, 16 * j:16 * j + 16], g, vals[codes[0, r, j]])[0] for j in range(2)]
        dfull = np.concatenate(d)
        cross = 2 * float((X[:, :16] @ d[0]) @ (X[:, 16:] @ d[1]))
        full_r = float(np.sum((X @ dfull) ** 2))
        assert full_r == pytest.approx(err[0, r].sum() + cross, rel=1e-10, abs=1e-18)
        full += full_r
    assert full > 0


def test_joint_brute_force_on_1x32_layer():
    # "算法原理": the joint search over all M^(C_in/16) scale combinations is what
    # the block-diagonal approximation replaces. On a 1x32 layer whose tokens
    # touch one block each, the joint argmin of ||Delta X||^2 over all 126^2
    # pairs equals the pair of per-block argmins.
    W, Xb, X = _tiny_layer(10, 1, 32, 64, disjoint=True)
    H = oracle.hessian(Xb)[0]
    A = np.abs(W).max()
    codes, _, _ = oracle.sweep(W, [A], H)
    g = oracle.global_scale(A)
    vals = indep.e4m3_values_torch()
    P = [np.stack([X[:, 16 * j:16 * j + 16] @ indep.candidate_dw(W[0, 16 * j:16 * j + 16], g, vals[c])[0]
                   for c in range(1, 127)]) for j in range(2)]        # [126, n_tok]
    tot = np.sum((P[0][:, None, :] + P[1][None, :, :]) ** 2, axis=-1)  # [126, 126]
    i0, i1 = np.unravel_index(np.argmin(tot), tot.shape)  # row-major: lowest codes on exact ties
    assert (i0 + 1, i1 + 1) == (codes[0, 0, 0], codes[0, 0, 1])


def test_joint_brute_force_bounds_blockwise_choice_generic_x():
    W, Xb, X = _tiny_layer(11, 1, 32, 64)
    H = oracle.hessian(Xb)[0]
    A = np.abs(W).max()
    codes, _, _ = oracle.sweep(W, [A], H)
    g = oracle.global_scale(A)
    vals = indep.e4m3_values_torch()
    P = [np.stack([X[:, 16 * j:16 * j + 16] @ indep.candidate_dw(W[0, 16 * j:16 * j + 16], g, vals[c])[0]
                   for c in range(1, 127)]) for j in range(2)]
    tot = np.sum((P[0][:, None, :] + P[1][None, :, :]) ** 2, axis=-1)
    assert tot.min() <= tot[codes[0, 0, 0] - 1, codes[0, 0, 1] - 1] * (1 + 1e-12)


def test_rank_one_hessian_closed_form():
    rng = np.random.default_rng(12)
    w = (rng.standard_normal(16) * 0.02).astype(np.float32)
    h = rng.standard_normal(16)
    H = np.outer(h, h)
    g = oracle.global_scale(np.abs(w).max())
    vals = indep.e4m3_values_torch()
    for c in range(1, 127, 5):
        dw, _ = indep.candidate_dw(w, g, vals[c])
        assert oracle.candidate_error(w, g, c, H) == pytest.approx(float(h @ dw) ** 2, rel=1e-10, abs=1e-300)


# ----------------------------------------------------------------------------- sweep
def test_identity_hessian_is_weight_mse_sweep():
    # "Local-Hessian 是什么": the MSE method sweeps the same 126 candidates on the
    # weight error; with H = I the Local-Hessian objective is that error.
    rng = np.random.default_rng(13)
    W = (rng.standard_t(4, (8, 64)) * 0.015).astype(np.float32)
    A = np.abs(W).max()
    H = np.broadcast_to(np.eye(16), (1, 4, 16, 16)).copy()
    codes, _, _ = oracle.sweep(W, [A], H)
    g = oracle.global_scale(A)
    for r in range(8):
        for j in range(4):
            assert codes[0, r, j] == indep.mse_sweep_block(W[r, 16 * j:16 * j + 16], g)


def test_never_worse_than_max_scaling_on_tiny_config():
    L = synth.make_config(0)
    W = L.W_f32()[0]
    A = oracle.absmax(W)
    H = oracle.hessian(L.X)
    codes, _, err = oracle.sweep(W, [A], H)
    g = oracle.global_scale(A)
    viol = 0
    for r in range(W.shape[0]):
        for j in range(W.shape[1] // 16):
            wb = W[r, 16 * j:16 * j + 16]
            cmax = indep.max_scaling_code(np.abs(wb).max(), g)
            e_max = oracle.candidate_error(wb, g, cmax, H[0, j])
            viol += err[0, r, j] > e_max
    assert viol == 0


def test_argmin_is_min_over_all_candidates_and_lowest_code_on_ties():
    L = synth.make_layer(4, 64, 64, seed=14, w_dtype="f32")
    W = L.W_f32()[0]
    A = oracle.absmax(W)
    H = oracle.hessian(L.X)
    codes, amax, err = oracle.sweep(W, [A], H)
    g = oracle.global_scale(A)
    for r, j in itertools.product(range(4), range(4)):
        e = oracle.block_errors(W[r, 16 * j:16 * j + 16], g, H[0, j])
        assert codes[0, r, j] == int(np.argmin(e)) + 1
        assert err[0, r, j] == e.min()
        assert amax[0, r, j] == np.float32(6.0) * oracle.candidate_scale(codes[0, r, j], g)
    # H = 0: every candidate has error 0, the lowest code wins
    c0, a0, _ = oracle.sweep(W, [A], np.zeros_like(H))
    assert np.all(c0 == 1) and np.all(a0 == np.float32(6.0) * oracle.candidate_scale(1, g))


def test_zero_matrix_gives_code_one_and_zero_amax():
    W = np.zeros((2, 32), np.float32)
    H = np.broadcast_to(np.eye(16), (1, 2, 16, 16)).copy()
    codes, amax, err = oracle.sweep(W, [0.0], H)
    assert np.all(codes == 1) and np.all(amax == 0) and np.all(err == 0)


def test_invariances_scale_of_h_power_of_two_w_row_permutation():
    L = synth.make_layer(6, 32, 128, seed=15, w_dtype="f32")
    W = L.W_f32()[0]
    A = oracle.absmax(W)
    H = oracle.hessian(L.X)
    c1, a1, _ = oracle.sweep(W, [A], H)
    c2, _, _ = oracle.sweep(W, [A], 3.7 * H)              # normalised H: any positive factor
    assert np.array_equal(c1, c2)
    c3, a3, _ = oracle.sweep(W * np.float32(8.0), [A * np.float32(8.0)], H)   # W -> 2^3 W
    assert np.array_equal(c1, c3) and np.array_equal(a3, a1 * np.float32(8.0))
    perm = np.random.default_rng(0).permutation(6)
    c4, _, _ = oracle.sweep(W[perm], [A], H)
    assert np.array_equal(c4[0], c1[0][perm])


# ----------------------------------------------------------------------------- fake quant
def test_fake_quant_matches_independent_q_times_s():
    L = synth.make_layer(4, 48, 64, seed=16, w_dtype="f32")
    W = L.W_f32()[0]
    A = oracle.absmax(W)
    H = oracle.hessian(L.X)
    codes, _, _ = oracle.sweep(W, [A], H)
    g = oracle.global_scale(A)
    vals = indep.e4m3_values_torch()
    out = oracle.fake_quant(W, [A], codes[0])
    out_bf = oracle.fake_quant(W, [A], codes[0], out_bf16=True)
    import torch
    for r in range(4):
        for j in range(3):
            s = np.float32(np.float32(vals[codes[0, r, j]]) * g)
            u = (W[r, 16 * j:16 * j + 16] / s).astype(np.float32)
            ref = (indep.e2m1_nearest(u).astype(np.float32) * s).astype(np.float32)
            assert np.array_equal(out[r, 16 * j:16 * j + 16], ref)
            refb = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(out_bf[r, 16 * j:16 * j + 16], refb)


@pytest.mark.parametrize("g", [1.0, 2.0 ** -95])
def test_fake_quant_ties_at_tiny_and_unit_scales(g):
    # every E2M1 tie and its FP32 neighbours, saturation, quotients below 2^-5 and signed
    # zeros, at block scales f g for f in {1, 2, 0.5, 1.5}: the oracle equals the
    # independent fp32(w / s) -> nearest E2M1 (ties to even) -> fp32(q s)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1, 1.5, 2, 3, 4, 6, 6.5, 7, 100,
                     1e-30, 2.0 ** -6, 0.02, 0], np.float32)
    vals = np.concatenate([ties, np.nextafter(ties, np.float32(0)), np.nextafter(ties, np.float32(1e9))])
    vals = np.concatenate([vals, -vals, [np.float32(-0.0)]]).astype(np.float32)
    n = ((len(vals) + 15) // 16) * 16
    W = np.zeros((4, n), np.float32)
    W[:, :len(vals)] = vals
    for r, f in enumerate((1.0, 2.0, 0.5, 1.5)):
        W[r] *= np.float32(f * g)
    codes = np.repeat(np.array([0x38, 0x40, 0x30, 0x3C], np.uint8)[:, None], n // 16, axis=1)
    A = np.float32(2688.0 * g)
    out = oracle.fake_quant(W, [A], codes)
    gs = oracle.global_scale(A)
    ev = indep.e4m3_values_torch()
    for r in range(4):
        s = np.float32(np.float32(ev[codes[r, 0]]) * gs)
        u = (W[r] / s).astype(np.float32)
        ref = (indep.e2m1_nearest(u).astype(np.float32) * s).astype(np.float32)
        assert np.array_equal(out[r].view(np.uint32), ref.view(np.uint32)), r


def test_fake_quant_error_is_the_swept_dw():
    L = synth.make_layer(3, 32, 64, seed=17, w_dtype="f32")
    W = L.W_f32()[0]
    A = oracle.absmax(W)
    H = oracle.hessian(L.X)
    codes, _, err = oracle.sweep(W, [A], H)
    D = oracle.fake_quant(W, [A], codes[0]).astype(np.float64) - W
    for r in range(3):
        for j in range(2):
            d = D[r, 16 * j:16 * j + 16]
            assert float(d @ H[0, j] @ d) == pytest.approx(err[0, r, j], rel=1e-6)
