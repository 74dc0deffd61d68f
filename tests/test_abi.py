"""The C ABI on the host (no GPU needed): the library loads, exports every
function include/nvfp4.h declares, and rejects invalid arguments before it
touches the device."""
import ctypes
import os
import re

import pytest

import nvfp4_block_scaled_12_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_expected_entry_points():
    names = declared_functions()
    for n in ("nvfp4_sf_bytes", "nvfp4_calibrate", "nvfp4_quantize", "nvfp4_swizzle_sf", "nvfp4_gemm",
              "nvfp4_gemm_quant", "nvfp4_quantize_dynamic", "nvfp4_gemm_dynamic", "nvfp4_mxfp8_sf_bytes",
              "nvfp4_mxfp8_quantize", "nvfp4_mxfp8_gemm", "nvfp4_fp8row_quantize", "nvfp4_fp8row_gemm",
              "nvfp4_dequantize", "nvfp4_check_fault", "nvfp4_last_error", "nvfp4_gemm_amax",
              "nvfp4_quantize_from_amax"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(F.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_mirrors_every_entry_point():
    for n in declared_functions():
        assert callable(getattr(F, n, None)), n


@pytest.mark.parametrize("rows,k,want", [(4608, 12288, 4608 * 768), (1, 64, 128 * 4), (129, 16, 256 * 4),
                                         (0, 64, 0), (5, 8, 0), (5, 24, 0)])
def test_sf_bytes(rows, k, want):
    assert F.nvfp4_sf_bytes(rows, k) == want


def _expect(status, fn, *args):
    with pytest.raises(F.NVFP4Error) as e:
        fn(*args)
    assert e.value.status == status, str(e.value)
    assert F.nvfp4_last_error()


P = 1 << 20  # a 16-byte-aligned fake device address: never dereferenced


def test_quantize_rejects_bad_arguments_on_the_host():
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize, 0, 16, 64, 1.0, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize, P, 0, 64, 1.0, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize, P, 4, 48, 1.0, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize, P, 4, 64, float("nan"), P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize, P, 4, 64, 0.0, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize, P, 4, 64, 2.0 ** 70, P, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_quantize, P + 2, 4, 64, 1.0, P, P, 0)


def test_gemm_rejects_bad_arguments_on_the_host():
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm, P, P, P, P, 0, 64, 64, 1.0, 0, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm, P, P, P, P, 16, 12, 64, 1.0, 0, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm, P, P, P, P, 16, 64, 96, 1.0, 0, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm, P, P, P, P, 16, 64, 64, float("inf"), 0, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm, P, 0, P, P, 16, 64, 64, 1.0, 0, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_gemm, P, P, P + 8, P, 16, 64, 64, 1.0, 0, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_gemm, P, P, P, P, 16, 64, 64, 1.0, P + 4, P, 0)


def test_gemm_quant_rejects_bad_ranges_on_the_host():
    R = F.ColRange
    args = lambda rs: (P, P, P, P, 128, 256, 256, 1.0, 0, rs, P, 256, 0.1, P, P, 256, 0)  # noqa: E731
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_quant, *args([R(0, 100, 0, 1, 0)]))
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_quant, *args([R(0, 128, 0, 1, 0), R(64, 192, 0, 0, 0)]))
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_quant, *args([R(0, 128, 7, 1, 0)]))
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_quant, *args([R(0, 128, 0, 9, 0)]))
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_quant, *args([R(0, 512, 0, 1, 0)]))
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_quant, *args([R(0, 256, 0, 1, 64)]))
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_quant, *args([]))
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_quant, *args([R(0, 64, 0, 1, 0)] * 9))


def test_dynamic_entry_points_reject_bad_arguments_on_the_host():
    W = F.NVFP4_DYNAMIC_WORKSPACE_BYTES
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_dynamic, P, 4, 64, P, P, P, 0, W, 0)       # no workspace
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_dynamic, P, 4, 64, P, P, P, P, W - 1, 0)   # too small
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_dynamic, P, 4, 64, P, P, 0, P, W, 0)       # no scale_out
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_dynamic, P, 0, 64, P, P, P, P, W, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_dynamic, P, 4, 96, P, P, P, P, W, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_quantize_dynamic, P + 8, 4, 64, P, P, P, P, W, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_quantize_dynamic, P, 4, 64, P, P, P + 2, P, W, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_dynamic, P, P, P, P, 16, 64, 64, 1.0, 0, 0, P, 0)   # no g_a
    _expect(F.NVFP4_EALIGN, F.nvfp4_gemm_dynamic, P, P, P, P, 16, 64, 64, 1.0, P + 1, 0, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_dynamic, P, P, P, P, 16, 64, 64, float("nan"), P, 0, P, 0)


def test_amax_entry_points_reject_bad_arguments_on_the_host():
    # nvfp4_gemm_amax(a, sfa, b, sfb, M, N, K, g_a, g_a_device, g_b, bias, y, amax_out, stream)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_amax, P, P, P, P, 16, 64, 64, 1.0, 0, 1.0, 0, P, 0, 0)    # no amax_out
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_amax, P, P, P, P, 16, 64, 64, 1.0, 0, 1.0, 0, 0, P, 0)    # no y
    _expect(F.NVFP4_EALIGN, F.nvfp4_gemm_amax, P, P, P, P, 16, 64, 64, 1.0, 0, 1.0, 0, P, P + 2, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_gemm_amax, P, P, P, P, 16, 64, 64, 1.0, P + 1, 1.0, 0, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_amax, P, P, P, P, 16, 64, 64, float("inf"), 0, 1.0, 0, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_amax, P, P, P, P, 16, 64, 64, 3e38, 0, 10.0, 0, P, P, 0)  # product
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_amax, P, P, P, P, 16, 64, 64, 1.0, P, float("nan"), 0, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_amax, P, P, P, P, 16, 12, 64, 1.0, 0, 1.0, 0, P, P, 0)    # N % 8
    # nvfp4_quantize_from_amax(x, M, K, amax, codes, sf, scale_out, stream)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_from_amax, P, 4, 64, 0, P, P, P, 0)      # no amax
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_from_amax, P, 4, 64, P, P, P, 0, 0)      # no scale_out
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_from_amax, P, 4, 96, P, P, P, P, 0)      # K % 64
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_from_amax, P, 0, 64, P, P, P, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_quantize_from_amax, P + 8, 4, 64, P, P, P, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_quantize_from_amax, P, 4, 64, P + 2, P, P, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_quantize_from_amax, P, 4, 64, P, P, P, P + 1, 0)


@pytest.mark.parametrize("rows,k,want", [(4608, 3072, 4608 * 96), (1, 64, 128 * 4), (129, 192, 256 * 8),
                                         (0, 64, 0), (5, 16, 0), (5, 48, 0)])
def test_mxfp8_sf_bytes(rows, k, want):
    assert F.nvfp4_mxfp8_sf_bytes(rows, k) == want


def test_mxfp8_entry_points_reject_bad_arguments_on_the_host():
    _expect(F.NVFP4_EINVAL, F.nvfp4_mxfp8_quantize, 0, 16, 64, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_mxfp8_quantize, P, 16, 96, P, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_mxfp8_quantize, P, 16, 64, P + 4, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_mxfp8_gemm, P, P, P, P, 16, 12, 64, 1.0, 0, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_mxfp8_gemm, P, P, P, P, 16, 64, 32, 1.0, 0, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_mxfp8_gemm, P, P, P + 8, P, 16, 64, 64, 1.0, 0, P, 0)


def test_fp8row_entry_points_reject_bad_arguments_on_the_host():
    _expect(F.NVFP4_EINVAL, F.nvfp4_fp8row_quantize, P, 0, 64, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_fp8row_quantize, P, 4, 96, P, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_fp8row_quantize, P, 4, 64, P, P + 4, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_fp8row_gemm, P, P, P, P, 16, 12, 64, 0, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_fp8row_gemm, P, P, P, P + 4, 16, 64, 64, 0, P, 0)


def test_dequantize_rejects_bad_arguments_on_the_host():
    _expect(F.NVFP4_EINVAL, F.nvfp4_dequantize, P, P, 1.0, 0, 64, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_dequantize, P, P, 1.0, 4, 48, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_dequantize, P, P, float("inf"), 4, 64, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_dequantize, P, P, 1.0, 4, 64, P + 2, 0)


def test_calibrate_and_swizzle_reject_bad_arguments_on_the_host():
    _expect(F.NVFP4_EINVAL, F.nvfp4_calibrate, P, 12, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_calibrate, P + 1, 16, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_swizzle_sf, P, 4, 80, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_swizzle_sf, P, 4, 64, P + 4, 0)


BIG = 1 << 30  # one past the largest row count or K


def test_sizes_past_the_int32_limits_are_rejected_on_the_host():
    W = F.NVFP4_DYNAMIC_WORKSPACE_BYTES
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize, P, BIG, 64, 1.0, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize, P, 4, BIG, 1.0, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_dynamic, P, BIG, 64, P, P, P, P, W, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_quantize_dynamic_noalloc, P, 4, BIG, P, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_mxfp8_quantize, P, BIG, 64, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_fp8row_quantize, P, BIG, 64, P, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm, P, P, P, P, BIG, 64, 64, 1.0, 0, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm, P, P, P, P, 16, BIG, 64, 1.0, 0, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm, P, P, P, P, 16, 64, BIG, 1.0, 0, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_dequantize, P, P, 1.0, BIG, 64, P, 0)
    # rows and K each in range, but a grid of more than 2^31 - 1 blocks
    _expect(F.NVFP4_EINVAL, F.nvfp4_dequantize, P, P, 1.0, BIG - 1, BIG - 64, P, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_swizzle_sf, P, BIG - 1, BIG - 64, P, 0)


def test_valid_arguments_without_a_device_fail_loudly_not_silently():
    # On this CPU-only host a valid call reaches the device check and must
    # report an error: there is no CPU fallback.
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(F.NVFP4Error) as e:
        F.nvfp4_quantize(P, 4, 64, 1.0, P, P, 0)
    assert e.value.status in (F.NVFP4_ECUDA, F.NVFP4_EARCH)


def test_scaled_gemms_reject_bad_scales_on_the_host():
    # the two per-tensor scales must be finite and so must their fp32 product
    for ga, gb in ((float("nan"), 1.0), (1.0, float("inf")), (2.0 ** 100, 2.0 ** 100)):
        _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_scaled, P, P, P, P, 16, 64, 64, ga, gb, 0, P, 0)
        rs = [F.ColRange(0, 64, F.ACT_NONE, F.DST_NVFP4, 0)]
        _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_quant_scaled, P, P, P, P, 16, 64, 64, ga, gb, 0, rs, 0, 0, 0.1, P, P,
                64, 0)
    # sizes and alignment are checked as for nvfp4_gemm
    _expect(F.NVFP4_EINVAL, F.nvfp4_gemm_scaled, P, P, P, P, 16, 12, 64, 1.0, 1.0, 0, P, 0)
    _expect(F.NVFP4_EALIGN, F.nvfp4_gemm_scaled, P, P, P, P, 16, 64, 64, 1.0, 1.0, 0, P + 4, 0)


def test_grid_wait_knob_checks_its_limits_and_resets():
    _expect(F.NVFP4_EINVAL, F.nvfp4_testing_set_grid_wait, 2 * 10 ** 9, 0)
    _expect(F.NVFP4_EINVAL, F.nvfp4_testing_set_grid_wait, 1000, 5000)
    F.nvfp4_testing_set_grid_wait(1000, 1)
    F.nvfp4_testing_set_grid_wait(0, 0)  # back to the defaults
