"""The C ABI on the host: the library loads without a GPU, exports every
symbol include/lh.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lh():
    import scale_calibration_b200 as lh
    return lh


def declared_functions():
    src = open(os.path.join(ROOT, "include", "lh.h")).read()
    return sorted(set(re.findall(r"LH_API\s+[\w\s\*]*?\b(lh_\w+)\s*\(", src)))


def test_exports_every_declared_symbol():
    lh = _lh()
    names = declared_functions()
    assert len(names) >= 8
    lib = ctypes.CDLL(lh._binding.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(lh.EXPORTS) == names


def test_status_strings():
    lh = _lh()
    assert lh.lh_status_string(0) == "LH_OK"
    assert lh.lh_status_string(6) == "LH_ERR_TIMEOUT"
    assert lh.lh_status_string(99) == "LH_ERR_UNKNOWN"


FAKE = 0x10000000  # a 256-byte-aligned address that is never dereferenced: validation fails first


def test_sweep_rejects_bad_arguments():
    lh = _lh()
    ok = dict(W=FAKE, w_dtype=lh.LH_BF16, n_mats=1, c_out=64, c_in=128, ld_w=128, global_amax=FAKE, H=FAKE,
              best_amax=FAKE, best_code=FAKE, stream=0, check=False)
    cases = [
        (dict(W=0), 1), (dict(global_amax=0), 1), (dict(best_code=0), 1), (dict(n_mats=0), 1), (dict(c_out=-1), 1),
        (dict(c_in=24, ld_w=24), 2), (dict(ld_w=120), 1), (dict(W=FAKE + 2), 3), (dict(ld_w=132), 3),
        (dict(w_dtype=7), 2), (dict(c_in=16 * 70000, ld_w=16 * 70000), 2),
    ]
    for over, want in cases:
        a = dict(ok, **over)
        assert lh.lh_sweep_scales(**a) == want, over
        assert lh.lh_last_error_message() != ""


def test_sweep_ws_rejects_bad_arguments():
    lh = _lh()
    need = lh.lh_sweep_workspace_bytes(2, 128)
    assert need == 16 * 2 * 8
    assert lh.lh_sweep_workspace_bytes(0, 128) == 0 and lh.lh_sweep_workspace_bytes(1, 24) == 0
    ok = dict(W=FAKE, w_dtype=lh.LH_BF16, n_mats=2, c_out=64, c_in=128, ld_w=128, global_amax=FAKE, H=FAKE,
              best_amax=FAKE, best_code=FAKE, workspace=FAKE, workspace_bytes=need, stream=0, check=False)
    cases = [
        (dict(workspace=0), 4), (dict(workspace_bytes=need - 1), 4), (dict(workspace=FAKE + 8), 3),
        (dict(W=0), 1), (dict(n_mats=0), 1), (dict(c_in=24, ld_w=24), 2), (dict(W=FAKE + 2), 3), (dict(w_dtype=7), 2),
    ]
    for over, want in cases:
        a = dict(ok, **over)
        assert lh.lh_sweep_scales_ws(**a) == want, over
        assert lh.lh_last_error_message() != ""
    # nothing to sweep: no launch, whatever the sizes
    assert lh.lh_sweep_scales_ws(**dict(ok, c_out=0)) == 0


def test_sweep_empty_is_noop():
    lh = _lh()
    assert lh.lh_sweep_scales(FAKE, lh.LH_BF16, 1, 0, 128, 128, FAKE, FAKE, FAKE, FAKE, 0, check=False) == 0


def test_hessian_rejects_bad_arguments():
    lh = _lh()
    need = lh.lh_hessian_workspace_bytes(300, 64, 1)
    ok = dict(X=FAKE, x_dtype=lh.LH_BF16, n_tokens_total=300, c_in=64, ld_x=64, offsets=None, n_groups=1, H=FAKE,
              workspace=FAKE, workspace_bytes=need, stream=0, check=False)
    cases = [
        (dict(x_dtype=lh.LH_F32), 2), (dict(X=0), 1), (dict(H=0), 1), (dict(n_groups=2), 1),
        (dict(c_in=40, ld_x=40), 2), (dict(ld_x=60), 1), (dict(ld_x=68), 3), (dict(X=FAKE + 8), 3),
        (dict(workspace_bytes=need - 1), 4), (dict(workspace=0), 4), (dict(workspace=FAKE + 16), 3),
        (dict(n_tokens_total=-1), 1), (dict(n_groups=0), 1),
    ]
    for over, want in cases:
        a = dict(ok, **over)
        assert lh.lh_accumulate_hessian(**a) == want, over


def test_hessian_noalloc_checks_arguments_like_the_workspace_entry():
    # the allocation-free entry point returns the same argument errors, before touching any
    # device (no GPU here)
    lh = _lh()
    ok = dict(X=FAKE, x_dtype=lh.LH_BF16, n_tokens_total=300, c_in=64, ld_x=64, offsets=None, n_groups=1, H=FAKE,
              stream=0, check=False)
    cases = [
        (dict(x_dtype=lh.LH_F32), 2), (dict(X=0), 1), (dict(H=0), 1), (dict(n_groups=2), 1),
        (dict(c_in=40, ld_x=40), 2), (dict(ld_x=60), 1), (dict(ld_x=68), 3), (dict(X=FAKE + 8), 3),
        (dict(n_tokens_total=-1), 1), (dict(n_groups=0), 1),
        (dict(n_tokens_total=1 << 24, c_in=40008, ld_x=40008), 2),
        (dict(n_tokens_total=1 << 24, c_in=32768, ld_x=32768, X=0), 1),
    ]
    for over, want in cases:
        a = dict(ok, **over)
        assert lh.lh_accumulate_hessian_noalloc(**a) == want, over
    assert lh.lh_accumulate_hessian_noalloc(**dict(ok, n_tokens_total=0)) == 0


def test_hessian_workspace_is_bounded_and_fits_the_noalloc_scratch():
    # the Hessian kernel runs at most 320 CTAs (token bands x slabs) and the workspace holds at
    # most two parts per CTA: it stops growing with the tokens, never depends on the groups,
    # and the largest one fits the 8 MiB array of the allocation-free entry point
    lh = _lh()
    sizes = [lh.lh_hessian_workspace_bytes(n, c, g) for n in (1, 255, 4096, 1 << 20, (1 << 31) - 1)
             for c in (16, 2048, 4096, 17408, 40960, (1 << 31) - 16) for g in (1, 64, 65535)]
    assert 0 < max(sizes) <= (8 << 20)
    assert lh.lh_hessian_workspace_bytes(1 << 20, 4096, 1) == lh.lh_hessian_workspace_bytes(8192, 4096, 64)
    assert lh.lh_hessian_workspace_bytes(256, 128, 1) < lh.lh_hessian_workspace_bytes(2048, 128, 1)
    # a layer wider than the grid runs as one band: no parts at all
    assert lh.lh_hessian_workspace_bytes(4096, 128 * 400, 1) == 256


def test_hessian_zero_tokens_is_noop():
    lh = _lh()
    assert lh.lh_accumulate_hessian(FAKE, lh.LH_BF16, 0, 64, 64, None, 1, FAKE, 0, 0, 0, check=False) == 0


def test_workspace_size_grows_with_tokens_then_stays_bounded():
    lh = _lh()
    a = lh.lh_hessian_workspace_bytes(256, 128, 1)
    b = lh.lh_hessian_workspace_bytes(2048, 128, 1)
    c = lh.lh_hessian_workspace_bytes(8192, 4096, 64)
    d = lh.lh_hessian_workspace_bytes(16384, 4096, 1)
    assert 0 < a < b <= c == d
    assert lh.lh_hessian_workspace_bytes(100, 0, 1) == 0


def test_fake_quant_and_absmax_reject_bad_arguments():
    lh = _lh()
    ok = dict(W=FAKE, w_dtype=lh.LH_BF16, n_mats=1, c_out=8, c_in=32, ld_w=32, global_amax=FAKE, codes=FAKE,
              W_out=FAKE + 4096, out_dtype=lh.LH_BF16, stream=0, check=False)
    for over, want in [(dict(W_out=FAKE), 1), (dict(codes=0), 1), (dict(c_in=20, ld_w=20), 2),
                       (dict(out_dtype=3), 2), (dict(W_out=FAKE + 4100), 3)]:
        assert lh.lh_fake_quant(**dict(ok, **over)) == want, over
    assert lh.lh_absmax(FAKE, lh.LH_F32, 1, 4, 8, 4, FAKE, 0, check=False) == 1
    assert lh.lh_absmax(0, lh.LH_F32, 1, 4, 8, 8, FAKE, 0, check=False) == 1
    assert lh.lh_absmax(FAKE + 4, lh.LH_F32, 1, 4, 8, 8, FAKE, 0, check=False) == 3


def test_debug_wait_rejects_bad_arguments():
    lh = _lh()
    assert lh.lh_debug_wait_timeout(FAKE, 255, 1000, 0, 0, check=False) == 4
    assert lh.lh_debug_wait_timeout(0, 256, 1000, 0, 0, check=False) == 4
    assert lh.lh_debug_wait_timeout(FAKE + 16, 256, 1000, 0, 0, check=False) == 3
    assert lh.lh_debug_wait_timeout(FAKE, 256, 0, 0, 0, check=False) == 1
    assert lh.lh_debug_wait_timeout(FAKE, 256, 2000000, 0, 0, check=False) == 1


def test_quantize_nvfp4_rejects_bad_arguments():
    lh = _lh()
    ok = dict(W=FAKE, w_dtype=lh.LH_BF16, n_mats=1, c_out=8, c_in=32, ld_w=32, global_amax=FAKE, codes=FAKE,
              packed=FAKE + 4096, block_scales=None, global_scale=None, W_out=None, out_dtype=lh.LH_BF16, stream=0,
              check=False)
    for over, want in [(dict(packed=None), 1), (dict(codes=None), 1), (dict(W=None), 1), (dict(c_in=20, ld_w=20), 2),
                       (dict(packed=FAKE + 4104), 3), (dict(W_out=FAKE + 8200), 3), (dict(packed=FAKE), 1),
                       (dict(W_out=FAKE), 1), (dict(w_dtype=5), 2), (dict(W_out=FAKE + 8192, out_dtype=9), 2)]:
        assert lh.lh_quantize_nvfp4(**dict(ok, **over)) == want, over
        assert lh.lh_last_error_message() != ""


def test_baseline_scales_reject_bad_arguments():
    lh = _lh()
    ok = dict(W=FAKE, w_dtype=lh.LH_BF16, n_mats=1, c_out=64, c_in=128, ld_w=128, global_amax=FAKE,
              method=lh.LH_SCALE_MAX, best_amax=FAKE, best_code=FAKE, stream=0, check=False)
    for over, want in [(dict(W=0), 1), (dict(best_code=0), 1), (dict(method=7), 2), (dict(c_in=24, ld_w=24), 2),
                       (dict(ld_w=120), 1), (dict(W=FAKE + 2), 3), (dict(w_dtype=7), 2),
                       (dict(method=lh.LH_SCALE_FOUR_OVER_SIX, best_amax=0), 1),
                       (dict(method=lh.LH_SCALE_MSE, W=0), 1), (dict(method=lh.LH_SCALE_MSE, ld_w=132), 3)]:
        assert lh.lh_baseline_scales(**dict(ok, **over)) == want, over
        assert lh.lh_last_error_message() != ""
    assert lh.lh_baseline_scales(**dict(ok, c_out=0)) == 0


def test_search_amax_rejects_bad_arguments():
    lh = _lh()
    ok = dict(W=FAKE, w_dtype=lh.LH_BF16, n_mats=1, c_out=64, c_in=128, ld_w=128, global_amax=FAKE, H=FAKE,
              best_amax=FAKE, best_code=FAKE, start=0.25, step=0.1, n_mult=38, stream=0, check=False)
    for over, want in [(dict(W=0), 1), (dict(best_code=0), 1), (dict(start=0.0), 1), (dict(step=-0.1), 1),
                       (dict(n_mult=0), 1), (dict(n_mult=5000), 1), (dict(start=float("nan")), 1),
                       (dict(c_in=24, ld_w=24), 2), (dict(W=FAKE + 2), 3), (dict(w_dtype=7), 2)]:
        assert lh.lh_search_amax(**dict(ok, **over)) == want, over
        assert lh.lh_last_error_message() != ""
    assert lh.lh_search_amax(**dict(ok, c_out=0)) == 0


def test_fma_probe_rejects_bad_arguments():
    lh = _lh()
    assert lh.lh_probe_fma_flop(148, 1000) == 148 * 256 * 1000 * 128
    assert lh.lh_probe_fma_flop(0, 10) == 0
    for packed, blocks, iters, out in [(1, 0, 10, FAKE), (0, 10, 0, FAKE), (1, 10, 10, 0), (0, 1 << 21, 10, FAKE)]:
        assert lh.lh_probe_fma(packed, blocks, iters, out, stream=0, check=False) == 1


def test_sweep_counts_only_in_the_measurement_build():
    lh = _lh()
    assert lh._binding.lib().lh_debug_sweep_counts(None, 1) == 2  # LH_ERR_UNSUPPORTED, no device call
