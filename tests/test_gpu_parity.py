"""CUDA library vs oracle, element by element, through the C ABI (needs a B200).

Rules: Hessians within 1e-5 relative Frobenius error (per block and whole
tensor; all-zero blocks exactly zero); codes bit-exact except where the
oracle's FP64 error of the GPU's code is within 1e-6 relative of the oracle's
minimum ("sweep-only" mode: the oracle sweeps with the GPU's H); best amax
bit-exact given the code; fake-quant output bit-exact given the codes.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _full_parity(layer, out_dtype=None, e2e_max_frac=1e-3):
    res = gu.run_library(layer, out_dtype=out_dtype)
    W = layer.W_f32()
    n_mats = layer.n_mats
    # a1: global amax, exact
    for m in range(n_mats):
        assert res["amax"][m] == oracle.absmax(W[m]), m
    # a2: Hessian vs FP64 oracle
    Hr = oracle.hessian(layer.X, c_in=layer.c_in, offsets=layer.offsets)
    per, whole, bad_zero = gu.hessian_rel_errors(res["H"], Hr)
    assert per <= gu.HESSIAN_RTOL and whole <= gu.HESSIAN_RTOL and bad_zero == 0, (per, whole, bad_zero)
    # a3: sweep-only parity with the GPU's H
    Hg = res["H"].astype(np.float64)
    ex, tol, fail, worst = gu.check_codes(W, res["amax"], Hg, res["codes"], res["best_amax"])
    assert fail == 0, (ex, tol, fail, worst)
    # end-to-end: oracle's own H (reported; differences come from H rounding only)
    co, _, _ = oracle.sweep(W, res["amax"], Hr)
    e2e_mismatch = int(np.count_nonzero(co != res["codes"]))
    assert e2e_mismatch <= e2e_max_frac * co.size + 2, e2e_mismatch
    # a4: fake-quant, bit-exact given the GPU codes
    bf = res["Wq"].dtype == np.uint16
    ref = oracle.fake_quant(W, res["amax"], res["codes"], out_bf16=bf)
    assert np.array_equal(ref.reshape(res["Wq"].shape), res["Wq"])
    return res


def test_tiny_layer_full_parity(cuda_ok):
    res = _full_parity(synth.make_config(0))
    assert res["codes"].min() >= 1 and res["codes"].max() <= 126


def test_tiny_layer_bf16_output(cuda_ok):
    _full_parity(synth.make_config(0), out_dtype=torch.bfloat16)


@pytest.mark.parametrize("c_out,c_in,n_tok,w_dtype,seed", [
    (200, 48, 300, "f32", 1),      # ragged rows, slab wider than c_in, ragged token tail
    (130, 144, 129, "bf16", 2),    # one token past a stage
    (64, 272, 1000, "bf16", 3),    # c_in not a multiple of 128
    (3, 16, 17, "f32", 4),         # smallest block count, one MMA step plus one row
    (257, 256, 4096, "bf16", 5),   # many token tiles per slab, split over CTA ranges
])
def test_ragged_layers(cuda_ok, c_out, c_in, n_tok, w_dtype, seed):
    _full_parity(synth.make_layer(c_out, c_in, n_tok, seed=seed, w_dtype=w_dtype, outlier_frac=0.001))


def test_grouped_experts_with_empty_and_tiny_groups(cuda_ok):
    counts = [0, 5, 1, 300, 0, 17, 129, 2100]
    layer = synth.make_layer(96, 128, sum(counts), seed=6, n_mats=len(counts), counts=counts)
    res = _full_parity(layer)
    assert np.all(res["H"][0] == 0) and np.all(res["H"][4] == 0)
    assert np.all(res["codes"][0] == 1) and np.all(res["codes"][4] == 1)  # H = 0: lowest code


def test_hessian_many_ragged_groups(cuda_ok):
    # 70 groups (three empty) over 16 slabs: CTA ranges start and end inside groups and slabs
    import scale_calibration_b200 as lh
    rng = np.random.default_rng(31)
    counts = rng.integers(0, 300, size=70)
    counts[[3, 10, 11]] = 0
    layer = synth.make_layer(8, 2048, int(counts.sum()), seed=31, n_mats=70, counts=counts.tolist())
    _, X, off = gu.to_device(layer)
    H = torch.zeros(70, 128, 16, 16, device="cuda")
    wsb = lh.lh_hessian_workspace_bytes(layer.n_tok, 2048, 70)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    lh.lh_accumulate_hessian(X, lh.LH_BF16, layer.n_tok, 2048, X.stride(0), off, 70, H, ws, wsb)
    assert lh.lh_workspace_status(ws) == 0
    Hg = H.cpu().numpy()
    per, whole, bad = gu.hessian_rel_errors(Hg, oracle.hessian(layer.X, c_in=2048, offsets=layer.offsets))
    assert per <= gu.HESSIAN_RTOL and whole <= gu.HESSIAN_RTOL and bad == 0, (per, whole, bad)
    assert np.all(Hg[[3, 10, 11]] == 0)


def test_hessian_pile_of_empty_groups(cuda_ok):
    # 48 empty groups at one offset: the bands charge every group a share of work, so
    # several bands start at that token and hold none; the big group after it spans
    # five bands whose parts its last band sums
    import scale_calibration_b200 as lh
    counts = [700, 40] + [0] * 48 + [3000, 5, 1200, 0, 0, 900]
    G = len(counts)
    layer = synth.make_layer(8, 256, int(sum(counts)), seed=33, n_mats=G, counts=counts)
    _, X, off = gu.to_device(layer)
    H = torch.zeros(G, 16, 16, 16, device="cuda")
    wsb = lh.lh_hessian_workspace_bytes(layer.n_tok, 256, G)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    lh.lh_accumulate_hessian(X, lh.LH_BF16, layer.n_tok, 256, X.stride(0), off, G, H, ws, wsb)
    assert lh.lh_workspace_status(ws) == 0
    Hg = H.cpu().numpy()
    per, whole, bad = gu.hessian_rel_errors(Hg, oracle.hessian(layer.X, c_in=256, offsets=layer.offsets))
    assert per <= gu.HESSIAN_RTOL and whole <= gu.HESSIAN_RTOL and bad == 0, (per, whole, bad)
    assert np.all(Hg[[c == 0 for c in counts]] == 0)


def test_hessian_overlapping_offsets_are_reported(cuda_ok):
    # two groups over the same 1000 tokens hold more tiles than the workspace bound: the call
    # stays in bounds and the workspace status says the offsets are invalid
    import scale_calibration_b200 as lh
    layer = synth.make_layer(8, 128, 1000, seed=32)
    _, X, _ = gu.to_device(layer)
    off = torch.tensor([0, 1000, 0, 1000], dtype=torch.int64, device="cuda")
    H = torch.zeros(3, 8, 16, 16, device="cuda")
    wsb = lh.lh_hessian_workspace_bytes(1000, 128, 3)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    lh.lh_accumulate_hessian(X, lh.LH_BF16, 1000, 128, 128, off, 3, H, ws, wsb)
    assert lh.lh_workspace_status(ws) == 1  # LH_ERR_INVALID_ARG
    assert "overlap" in lh.lh_last_error_message()


def _packed_parity(layer, out_dtype):
    import scale_calibration_b200 as lh
    W, X, off = gu.to_device(layer)
    res = gu.run_library(layer, W=W, X=X, off=off, out_dtype=out_dtype)
    n_mats, c_out, c_in = W.shape
    codes = torch.from_numpy(res["codes"]).cuda()
    amax = torch.from_numpy(res["amax"]).cuda()
    packed = torch.empty(n_mats, c_out, c_in // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(n_mats, c_out, c_in // 16, dtype=torch.uint8, device="cuda")
    gs = torch.empty(n_mats, dtype=torch.float32, device="cuda")
    Wq = torch.empty(n_mats, c_out, c_in, dtype=out_dtype, device="cuda")
    dt = lh.LH_BF16 if out_dtype == torch.bfloat16 else lh.LH_F32
    lh.lh_quantize_nvfp4(W, W, n_mats, c_out, c_in, W.stride(1), amax, codes, packed, scales, gs, Wq, dt)
    torch.cuda.synchronize()
    p_ref, s_ref, g_ref = oracle.pack_nvfp4(layer.W_f32(), res["amax"], res["codes"])
    assert np.array_equal(packed.cpu().numpy(), p_ref)
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(gs.cpu().numpy(), g_ref)
    wq = Wq.view(torch.int16).cpu().numpy().view(np.uint16) if out_dtype == torch.bfloat16 else Wq.cpu().numpy()
    assert np.array_equal(wq, res["Wq"])  # the fused pass writes what lh_fake_quant writes
    # packed only: no optional outputs
    packed2 = torch.zeros_like(packed)
    lh.lh_quantize_nvfp4(W, W, n_mats, c_out, c_in, W.stride(1), amax, codes, packed2)
    torch.cuda.synchronize()
    assert torch.equal(packed2, packed)


def test_packed_nvfp4_export_tiny(cuda_ok):
    _packed_parity(synth.make_config(0), torch.float32)


def test_packed_nvfp4_export_ragged_and_grouped(cuda_ok):
    _packed_parity(synth.make_layer(130, 144, 129, seed=2, w_dtype="bf16", outlier_frac=0.001), torch.bfloat16)
    counts = [0, 5, 1, 300, 0, 17, 129, 2100]
    _packed_parity(synth.make_layer(96, 128, sum(counts), seed=6, n_mats=len(counts), counts=counts), torch.bfloat16)


def test_signed_zero_weights_keep_their_sign(cuda_ok):
    # -0 weights quantise to -0: W_q and the packed sign bit, compared as bits
    import scale_calibration_b200 as lh
    for w_dtype, out_dtype in (("f32", torch.float32), ("bf16", torch.bfloat16)):
        layer = synth.make_layer(64, 128, 256, seed=51, w_dtype=w_dtype)
        if w_dtype == "f32":
            layer.W[0, ::3, ::5] = np.float32(-0.0)
        else:
            layer.W[0, ::3, ::5] = np.uint16(0x8000)
        W, X, off = gu.to_device(layer)
        res = gu.run_library(layer, W=W, X=X, off=off, out_dtype=out_dtype)
        n_mats, c_out, c_in = W.shape
        bf = out_dtype == torch.bfloat16
        ref = oracle.fake_quant(layer.W_f32(), res["amax"], res["codes"], out_bf16=bf).reshape(res["Wq"].shape)
        got = res["Wq"]
        if not bf:
            ref, got = ref.view(np.uint32), got.view(np.uint32)
        assert np.array_equal(ref, got)
        packed = torch.empty(n_mats, c_out, c_in // 2, dtype=torch.uint8, device="cuda")
        lh.lh_quantize_nvfp4(W, W, n_mats, c_out, c_in, W.stride(1), torch.from_numpy(res["amax"]).cuda(),
                             torch.from_numpy(res["codes"]).cuda(), packed)
        torch.cuda.synchronize()
        p_ref, _, _ = oracle.pack_nvfp4(layer.W_f32(), res["amax"], res["codes"])
        assert np.array_equal(packed.cpu().numpy(), p_ref)


@pytest.mark.parametrize("g", [1.0, 2.0 ** -95])
def test_e2m1_ties_and_saturation_through_fake_quant_and_export(cuda_ok, g):
    # every E2M1 rounding tie, its FP32 neighbours, grid points, saturation, tiny values and
    # signed zeros, at four block scales: W_q bits and packed bytes equal the oracle's.
    # g = 2^-95 puts the block scales on both sides of 2^-95 (s = 2^-96 .. 2^-94), where
    # the kernel switches between the reciprocal quotient and IEEE division.
    import scale_calibration_b200 as lh
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1, 1.5, 2, 3, 4, 6, 6.5, 7, 100,
                     1e-30, 2.0 ** -6, 0.02, 0], np.float32)
    vals = np.concatenate([ties, np.nextafter(ties, np.float32(0)), np.nextafter(ties, np.float32(1e9))])
    vals = np.concatenate([vals, -vals, [np.float32(-0.0)]]).astype(np.float32)
    n = ((len(vals) + 15) // 16) * 16
    Wn = np.zeros((1, 4, n), np.float32)
    Wn[0, :, :len(vals)] = vals
    for r, f in enumerate((1.0, 2.0, 0.5, 1.5)):
        Wn[0, r] *= np.float32(f * g)
    cd = np.repeat(np.array([0x38, 0x40, 0x30, 0x3C], np.uint8)[:, None], n // 16, axis=1)[None]  # s = f g
    amax = np.array([2688.0 * g], np.float32)
    W, A, C = (torch.from_numpy(a).cuda() for a in (Wn, amax, cd))
    out = torch.empty_like(W)
    pk = torch.zeros(1, 4, n // 2, dtype=torch.uint8, device="cuda")
    lh.lh_fake_quant(W, lh.LH_F32, 1, 4, n, n, A, C, out, lh.LH_F32)
    lh.lh_quantize_nvfp4(W, lh.LH_F32, 1, 4, n, n, A, C, pk)
    torch.cuda.synchronize()
    ref = oracle.fake_quant(Wn, amax, cd).reshape(Wn.shape)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(pk.cpu().numpy(), oracle.pack_nvfp4(Wn, amax, cd)[0])


def test_sparse_nonnegative_activations(cuda_ok):
    _full_parity(synth.make_layer(128, 256, 777, seed=7, sparse=0.6))


def test_strided_inputs(cuda_ok):
    import scale_calibration_b200 as lh
    layer = synth.make_layer(40, 64, 333, seed=8, w_dtype="bf16")
    W, X, _ = gu.to_device(layer)
    Wp = torch.zeros(1, 40, 88, dtype=torch.bfloat16, device="cuda")
    Wp[:, :, :64] = W
    Xp = torch.zeros(333, 72, dtype=torch.bfloat16, device="cuda")
    Xp[:, :64] = X
    Xp[:, 64:] = 1e3  # padding columns must not leak into H
    ref = gu.run_library(layer)
    amax = torch.empty(1, device="cuda")
    lh.lh_absmax(Wp, Wp, 1, 40, 64, 88, amax)
    H = torch.zeros(1, 4, 16, 16, device="cuda")
    wsb = lh.lh_hessian_workspace_bytes(333, 64, 1)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    lh.lh_accumulate_hessian(Xp, lh.LH_BF16, 333, 64, 72, None, 1, H, ws, wsb)
    codes = torch.empty(1, 40, 4, dtype=torch.uint8, device="cuda")
    bam = torch.empty(1, 40, 4, device="cuda")
    lh.lh_sweep_scales(Wp, Wp, 1, 40, 64, 88, amax, H, bam, codes)
    torch.cuda.synchronize()
    assert np.array_equal(H.cpu().numpy(), ref["H"])
    assert np.array_equal(codes.cpu().numpy(), ref["codes"])


def test_hessian_accumulates_across_calls(cuda_ok):
    import scale_calibration_b200 as lh
    layer = synth.make_layer(8, 128, 1500, seed=9)
    _, X, _ = gu.to_device(layer)
    H = torch.zeros(1, 8, 16, 16, device="cuda")
    for t0, t1 in [(0, 700), (700, 1500)]:
        Xs = X[t0:t1]
        wsb = lh.lh_hessian_workspace_bytes(t1 - t0, 128, 1)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        lh.lh_accumulate_hessian(Xs, lh.LH_BF16, t1 - t0, 128, 128, None, 1, H, ws, wsb)
    torch.cuda.synchronize()
    per, whole, _ = gu.hessian_rel_errors(H.cpu().numpy(), oracle.hessian(layer.X))
    assert per <= gu.HESSIAN_RTOL


def test_degenerate_zero_weights_and_zero_hessian(cuda_ok):
    layer = synth.make_layer(16, 64, 50, seed=10, w_dtype="f32")
    layer.W[...] = 0
    res = gu.run_library(layer)
    assert np.all(res["codes"] == 1) and np.all(res["best_amax"] == 0) and np.all(res["Wq"] == 0)
    layer = synth.make_layer(16, 64, 50, seed=11, w_dtype="f32")
    layer.X[...] = 0
    res = gu.run_library(layer)
    assert np.all(res["H"] == 0) and np.all(res["codes"] == 1)


def test_tiny_global_scale_takes_exact_path(cuda_ok):
    # amax ~ 1e-33: the smallest candidate scales are FP32 subnormals; the
    # kernel must fall back to per-candidate division and still match.
    layer = synth.make_layer(32, 64, 200, seed=12, w_dtype="f32")
    layer.W = (layer.W * np.float32(2.0 ** -105)).astype(np.float32)
    _full_parity(layer)


def test_invariances_on_gpu(cuda_ok):
    layer = synth.make_layer(64, 128, 400, seed=13, w_dtype="f32")
    base = gu.run_library(layer)
    l2 = synth.make_layer(64, 128, 400, seed=13, w_dtype="f32")
    l2.W = (l2.W * np.float32(16.0)).astype(np.float32)
    r2 = gu.run_library(l2)
    assert np.array_equal(base["codes"], r2["codes"])
    assert np.array_equal(base["best_amax"] * np.float32(16.0), r2["best_amax"])
    perm = np.random.default_rng(0).permutation(64)
    l3 = synth.make_layer(64, 128, 400, seed=13, w_dtype="f32")
    l3.W = np.ascontiguousarray(l3.W[:, perm])
    r3 = gu.run_library(l3)
    assert np.array_equal(base["codes"][:, perm], r3["codes"])


def _full_size_parity(idx, n_sample=6000, seed=0):
    layer = synth.make_config(idx)
    res = gu.run_library(layer)
    W = layer.W_f32()
    for m in range(layer.n_mats):
        assert res["amax"][m] == oracle.absmax(W[m])
    rng = np.random.default_rng(seed)
    J = layer.c_in // 16
    # Hessian: every block column of every group against the oracle's FP64 sums
    Hr = oracle.hessian(layer.X, c_in=layer.c_in, offsets=layer.offsets)
    per, whole, bad = gu.hessian_rel_errors(res["H"], Hr)
    assert per <= gu.HESSIAN_RTOL and whole <= gu.HESSIAN_RTOL and bad == 0, (per, whole, bad)
    # sweep-only parity on sampled blocks plus two full rows
    n = n_sample
    mats = rng.integers(0, layer.n_mats, n)
    rows = rng.integers(0, layer.c_out, n)
    cols = rng.integers(0, J, n)
    for r in (0, layer.c_out - 1):
        mats = np.concatenate([mats, np.zeros(J, np.int64) + layer.n_mats - 1])
        rows = np.concatenate([rows, np.full(J, r)])
        cols = np.concatenate([cols, np.arange(J)])
    ex, tol, fail, worst = gu.check_codes(W, res["amax"], res["H"].astype(np.float64), res["codes"],
                                          res["best_amax"], mats, rows, cols)
    assert fail == 0, (ex, tol, fail, worst)
    # fake-quant: sampled rows, bit-exact
    for m, r in zip(mats[:64], rows[:64]):
        ref = oracle.fake_quant(W[m, r:r + 1], res["amax"][m:m + 1], res["codes"][m, r:r + 1], out_bf16=True)
        assert np.array_equal(ref, res["Wq"][m, r:r + 1])
    # invariant at any size: never worse than the candidate max scaling picks
    return res


def test_attention_projection_full_size(cuda_ok):
    _full_size_parity(1)


@pytest.mark.slow
def test_mlp_up_full_size(cuda_ok):
    _full_size_parity(2)


@pytest.mark.slow
def test_mlp_down_full_size(cuda_ok):
    _full_size_parity(3)


@pytest.mark.slow
def test_moe_experts_full_size(cuda_ok):
    _full_size_parity(4)


def test_tiny_weights_inside_normal_blocks(cuda_ok):
    # weights far below the global scale (down to 1e-37) next to normal ones: the
    # quotients w/s stay exact where the sweep divides by a reciprocal and
    # fall back to IEEE division for blocks holding such tiny values
    layer = synth.make_layer(256, 64, 300, seed=14, w_dtype="f32")
    rng = np.random.default_rng(14)
    W = layer.W
    idx = rng.choice(W.size, size=W.size // 8, replace=False)
    W.reshape(-1)[idx] *= np.float32(10.0) ** rng.integers(-36, -2, size=idx.size).astype(np.float32)
    _full_parity(layer)


def test_indefinite_hessian_gets_exact_argmin(cuda_ok):
    # a symmetric but indefinite H (errors can be negative): no pruning may apply,
    # the sweep must still return the oracle's argmin
    import scale_calibration_b200 as lh
    layer = synth.make_layer(96, 64, 10, seed=15, w_dtype="f32")
    W, _, _ = gu.to_device(layer)
    rng = np.random.default_rng(15)
    Hn = np.zeros((1, 4, 16, 16), np.float32)
    for j in range(4):
        A = rng.standard_normal((16, 16)).astype(np.float32)
        Hn[0, j] = (A + A.T) * np.float32(0.5)
    H = torch.from_numpy(Hn).cuda()
    amax = torch.empty(1, device="cuda")
    lh.lh_absmax(W, W, 1, 96, 64, 64, amax)
    codes = torch.empty(1, 96, 4, dtype=torch.uint8, device="cuda")
    bam = torch.empty(1, 96, 4, device="cuda")
    lh.lh_sweep_scales(W, W, 1, 96, 64, 64, amax, H, bam, codes)
    torch.cuda.synchronize()
    ex, tol, fail, worst = gu.check_codes(layer.W_f32(), amax.cpu().numpy(), Hn.astype(np.float64),
                                          codes.cpu().numpy(), bam.cpu().numpy())
    assert fail == 0, (ex, tol, fail, worst)


@pytest.mark.parametrize("kind", ["dominant_channel", "correlated", "near_collinear_pairs"])
def test_sweep_error_bound_on_conditioned_hessians(cuda_ok, kind):
    # Hessians whose normalised form C = D^-1/2 H D^-1/2 spans the range the FP32
    # error bound depends on: one channel ~5000x the others (diagonal ratio ~1e7,
    # many near ties), channels sharing a common factor (|C| row sums near 16), and
    # pairs of almost equal channels (lambda_min(C) small); sweep-only parity
    import scale_calibration_b200 as lh
    rng = np.random.default_rng({"dominant_channel": 21, "correlated": 22, "near_collinear_pairs": 23}[kind])
    c_out, c_in, n_tok = 1024, 64, 4096
    X = rng.standard_normal((n_tok, c_in))
    if kind == "dominant_channel":
        X[:, rng.choice(c_in, size=4, replace=False)] *= 5000.0
    elif kind == "correlated":
        X = 0.3 * X + rng.standard_normal((n_tok, 1))
    else:
        X[:, 1::2] = X[:, 0::2] + 1e-3 * rng.standard_normal((n_tok, c_in // 2))
    Hn = np.einsum("tja,tjb->jab", X.reshape(n_tok, c_in // 16, 16), X.reshape(n_tok, c_in // 16, 16))
    Hn = Hn.astype(np.float32)[None]
    Wn = (rng.standard_t(4.0, size=(c_out, c_in)) * 0.015).astype(np.float32)
    W = torch.from_numpy(Wn).cuda()
    H = torch.from_numpy(Hn).cuda()
    amax = torch.empty(1, device="cuda")
    lh.lh_absmax(W, W, 1, c_out, c_in, c_in, amax)
    codes = torch.empty(1, c_out, c_in // 16, dtype=torch.uint8, device="cuda")
    bam = torch.empty(1, c_out, c_in // 16, device="cuda")
    lh.lh_sweep_scales(W, W, 1, c_out, c_in, c_in, amax, H, bam, codes)
    torch.cuda.synchronize()
    ex, tol, fail, worst = gu.check_codes(Wn[None], amax.cpu().numpy(), Hn.astype(np.float64),
                                          codes.cpu().numpy(), bam.cpu().numpy())
    assert fail == 0, (ex, tol, fail, worst)


@pytest.mark.parametrize("c_out,c_in,n_mats,h_none", [(1, 16, 1, False), (700, 48, 3, False), (2100, 32, 1, True),
                                                     (4096, 2560, 1, False)])
def test_sweep_workspace_variant_matches(cuda_ok, c_out, c_in, n_mats, h_none):
    # the workspace path (column bounds from a first kernel) returns what the path
    # without a workspace returns, on shapes where every tile or only the last wave
    # of tiles is halved, ragged tiles, several matrices and the identity H; stale
    # workspace contents do not matter
    import scale_calibration_b200 as lh
    rng = np.random.default_rng(c_out + c_in)
    Wn = (rng.standard_t(4.0, size=(n_mats, c_out, c_in)) * 0.015).astype(np.float32)
    W = torch.from_numpy(Wn).cuda().to(torch.bfloat16)
    X = rng.standard_normal((512, c_in)) * rng.lognormal(0.0, 1.0, size=c_in)
    Hn = np.einsum("tja,tjb->jab", X.reshape(512, c_in // 16, 16), X.reshape(512, c_in // 16, 16)).astype(np.float32)
    H = None if h_none else torch.from_numpy(np.broadcast_to(Hn, (n_mats,) + Hn.shape).copy()).cuda()
    amax = torch.empty(n_mats, device="cuda")
    lh.lh_absmax(W, W, n_mats, c_out, c_in, c_in, amax)
    J = c_in // 16
    out = []
    for use_ws in (False, True):
        codes = torch.empty(n_mats, c_out, J, dtype=torch.uint8, device="cuda")
        bam = torch.empty(n_mats, c_out, J, device="cuda")
        if use_ws:
            wsb = lh.lh_sweep_workspace_bytes(n_mats, c_in)
            ws = torch.full((wsb,), 0x7F, dtype=torch.uint8, device="cuda")
            lh.lh_sweep_scales_ws(W, W, n_mats, c_out, c_in, c_in, amax, H, bam, codes, ws, wsb)
        else:
            lh.lh_sweep_scales(W, W, n_mats, c_out, c_in, c_in, amax, H, bam, codes)
        torch.cuda.synchronize()
        out.append((codes.cpu().numpy(), bam.cpu().numpy()))
    assert np.array_equal(out[0][0], out[1][0])
    assert np.array_equal(out[0][1].view(np.int32), out[1][1].view(np.int32))
    if c_out * J * n_mats <= 20000:
        Hd = (np.broadcast_to(np.eye(16), (n_mats, J, 16, 16)) if h_none
              else np.broadcast_to(Hn, (n_mats,) + Hn.shape)).astype(np.float64)
        Wf = W.float().cpu().numpy()
        ex, tol, fail, worst = gu.check_codes(Wf, amax.cpu().numpy(), Hd, out[1][0], out[1][1])
        assert fail == 0, (ex, tol, fail, worst)
