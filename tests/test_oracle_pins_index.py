"""Pins of the oracle's indexing: the global amax over a strided matrix, the
sampled-block sweep against the whole-layer sweep, and the per-matrix offsets
of a batched sweep (CPU only).

"NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块权重缩放算法实战指南"
(xxmr.cn/news/266017), section "算法原理", kernel contract: the kernel receives
the global FP32 amax of the weight, weights as [N_BLOCKS, 16] in (cout, cin/16)
order and H as [cin/16, 16, 16]. These tests check that the oracle reads the
elements those layouts name, and only those: numpy's reductions and slicing
serve as the independent statement.
"""
import ctypes

import numpy as np
import pytest

import oracle


def _absmax_strided(buf: np.ndarray, rows: int, cols: int) -> np.float32:
    """oracle_absmax over the first `cols` columns of a [rows, ld] buffer."""
    buf = np.ascontiguousarray(buf, np.float32)
    lib = oracle._L()
    return np.float32(lib.oracle_absmax(buf.ctypes.data_as(ctypes.c_void_p), rows, cols, buf.shape[1]))


@pytest.mark.parametrize("where", ["first", "last_col", "last_row", "last_row_last_col", "last_row_first_col"])
def test_absmax_reads_every_element_and_skips_padding(where):
    rng = np.random.default_rng(7)
    rows, cols, ld = 37, 45, 56
    buf = rng.standard_normal((rows, ld)).astype(np.float32) * np.float32(0.02)
    buf[:, cols:] = np.float32(1e30)  # padding past cols must be ignored
    r, c = dict(first=(0, 0), last_col=(11, cols - 1), last_row=(rows - 1, 17),
                last_row_last_col=(rows - 1, cols - 1), last_row_first_col=(rows - 1, 0))[where]
    buf[r, c] = np.float32(-3.75)  # the largest magnitude, negative
    ref = np.abs(buf[:, :cols]).max()
    assert ref == np.float32(3.75)
    assert _absmax_strided(buf, rows, cols) == ref


def test_absmax_signed_zero_and_subnormal():
    z = np.full((3, 8), -0.0, np.float32)
    a = _absmax_strided(z, 3, 8)
    assert a == 0.0 and not np.signbit(a)
    sub = np.zeros((4, 16), np.float32)
    tiny = np.float32(np.finfo(np.float32).smallest_subnormal) * np.float32(3)
    sub[2, 5] = -tiny
    sub[1, 1] = np.float32(np.finfo(np.float32).smallest_subnormal)
    assert _absmax_strided(sub, 4, 16) == tiny
    # the wrapper on a contiguous matrix agrees with numpy
    rng = np.random.default_rng(3)
    W = rng.standard_t(4, (64, 80)).astype(np.float32)
    assert oracle.absmax(W) == np.abs(W).max()


def _layer(n_mats=3, c_out=5, c_in=48, seed=11):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((n_mats, c_out, c_in)) * 0.02).astype(np.float32)
    W[1, 2, 7] = np.float32(0.3)  # matrices get different global amaxes
    amax = np.abs(W).max(axis=(1, 2)).astype(np.float32)
    J = c_in // 16
    X = rng.standard_normal((n_mats, J, 40, 16))
    H = np.einsum("mjta,mjtb->mjab", X, X)  # a distinct PSD H per matrix and column
    return W, amax, H


def test_sweep_blocks_equals_full_sweep_at_listed_indices():
    W, amax, H = _layer()
    n_mats, c_out, c_in = W.shape
    J = c_in // 16
    code, bam, err = oracle.sweep(W, amax, H)
    rng = np.random.default_rng(5)
    mats = np.concatenate([rng.integers(0, n_mats, 40), [0, n_mats - 1, n_mats - 1, 0, 1, 1]])
    rows = np.concatenate([rng.integers(0, c_out, 40), [0, c_out - 1, c_out - 1, c_out - 1, 2, 2]])
    cols = np.concatenate([rng.integers(0, J, 40), [0, J - 1, 0, J - 1, 1, 1]])  # repeats and boundaries
    c2, a2, e2 = oracle.sweep_blocks(W, amax, H, mats, rows, cols)
    assert np.array_equal(c2, code[mats, rows, cols])
    assert np.array_equal(a2.view(np.uint32), bam[mats, rows, cols].view(np.uint32))
    assert np.array_equal(e2, err[mats, rows, cols])


def test_sweep_of_every_block_through_sweep_blocks():
    W, amax, H = _layer(n_mats=2, c_out=4, c_in=64, seed=2)
    n_mats, c_out, c_in = W.shape
    J = c_in // 16
    m, r, j = (a.ravel() for a in np.meshgrid(np.arange(n_mats), np.arange(c_out), np.arange(J), indexing="ij"))
    code, bam, err = oracle.sweep(W, amax, H)
    c2, a2, e2 = oracle.sweep_blocks(W, amax, H, m, r, j)
    assert np.array_equal(c2.reshape(code.shape), code)
    assert np.array_equal(a2.reshape(bam.shape), bam)
    assert np.array_equal(e2.reshape(err.shape), err)


def test_batched_sweep_equals_per_matrix_sweeps():
    # matrix m is swept with its own global amax and its own H[m]: a batched call
    # equals n_mats one-matrix calls, and the blocks of row r, column j are the 16
    # weights W[m, r, 16j:16j+16]
    W, amax, H = _layer()
    code, bam, err = oracle.sweep(W, amax, H)
    for m in range(W.shape[0]):
        c1, a1, e1 = oracle.sweep(W[m], amax[m:m + 1], H[m:m + 1])
        assert np.array_equal(code[m], c1[0])
        assert np.array_equal(bam[m], a1[0])
        assert np.array_equal(err[m], e1[0])
    # one block, against the single-block error of every candidate
    m, r, j = 1, 2, 0
    errs = oracle.block_errors(W[m, r, 16 * j:16 * j + 16], oracle.global_scale(amax[m]), H[m, j])
    c = int(np.argmin(errs)) + 1
    assert code[m, r, j] == c and err[m, r, j] == errs.min()
