"""GPU parity of the MXFP8 variant against the oracle: the quantizer bit-exact
(codes, E8M0 scales, padding), the GEMM within the NVFP4 GEMM's tolerance and
bit-exact where fp32 accumulation is exact.

MXFP8: E4M3 elements in 32-element blocks sharing an E8M0 power-of-two scale,
per the OCP microscaling standard ("NVIDIA FP4 format" news page,
paragraph 1).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import mxfp8_ref as X
from oracle import nvfp4_ref as N
from tests.gpu_helpers import assert_bytes_equal, assert_within_tol, f32, gpu_bytes, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    require_gpu()
    import nvfp4_block_scaled_12_b200 as F
    return F


def _check_quant(F, x_bf16: torch.Tensor, what: str, rows=None):
    q = F.quantize_mxfp8(x_bf16.cuda())
    torch.cuda.synchronize()
    x = f32(x_bf16)
    M, K = x.shape
    sel = np.arange(M) if rows is None else rows
    codes, sf = X.quantize_mxfp8(x[sel])
    assert_bytes_equal(gpu_bytes(q.codes)[sel], codes, what + " codes")
    got_sf = gpu_bytes(q.sf)
    assert_bytes_equal(X.unswizzle_sf_mxfp8(got_sf, M, K)[sel], sf, what + " scales")
    if rows is None:  # padding rows and columns are zero
        assert_bytes_equal(got_sf, X.swizzle_sf_mxfp8(X.quantize_mxfp8(x)[1]), what + " scale buffer")
    return q


def test_tiny(F):
    _check_quant(F, synth.TINY.activations(), "tiny")


@pytest.mark.parametrize("m,k", [(1, 64), (7, 192), (127, 320), (129, 64), (300, 4160), (256, 128)])
def test_ragged_shapes_including_padding(F, m, k):
    _check_quant(F, synth.activations_with_outlier_channels(m, k, seed=m * 7 + k), f"ragged {m}x{k}")


def test_every_bf16_value_inside_a_block(F):
    # every finite bf16 value as an element, in blocks whose maximum is 448
    # (scale 2^0) or 448 * 2^20, so each value is converted at many scales
    bits = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    v = bits[np.isfinite(bits)]
    n_blk = (v.size + 30) // 31
    vals = np.zeros(n_blk * 31, np.float32)
    vals[:v.size] = v
    vals = np.clip(vals, -400.0, 400.0)
    for top in (448.0, 448.0 * 2.0 ** 20, 448.0 * 2.0 ** -30):
        blocks = np.concatenate([np.full((n_blk, 1), top, np.float32),
                                 (vals * np.float32(top / 448.0)).reshape(n_blk, 31)], axis=1)
        rows = (n_blk + 1) // 2
        x = np.zeros((rows * 2, 32), np.float32)
        x[:n_blk] = blocks
        x = torch.from_numpy(x.reshape(rows, 64)).to(torch.bfloat16)
        _check_quant(F, x, f"all bf16 values, top {top}")


def test_special_blocks(F):
    x = np.zeros((4, 128), np.float32)
    x[0, 5] = -0.0                           # zero block with a -0
    x[0, 32:64] = np.linspace(-3, 3, 32)
    x[1, :32] = 511.0                        # saturates to 448
    x[1, 32:64] = 2.0 ** -130                # fp32-subnormal block maximum (bf16 subnormal)
    x[2, :] = np.linspace(-1e30, 1e30, 128)
    x[3, :] = -np.logspace(-30, 30, 128)
    _check_quant(F, torch.from_numpy(x).to(torch.bfloat16), "special")


def test_mlp_up_activations_sampled_rows(F):
    x = synth.MLP_UP.activations()
    rows = np.sort(np.random.default_rng(9).choice(x.shape[0], 64, replace=False))
    _check_quant(F, x, "mlp-up", rows=rows)


def _linear(F, wl, rows=None, cols=None):
    x, w = wl.activations(), wl.weight()
    bias = wl.bias_vec()
    xq = F.quantize_mxfp8(x.cuda())
    wq = F.quantize_mxfp8(w.cuda())
    y = F.gemm_mxfp8(xq, wq, bias=bias.cuda() if bias is not None else None)
    torch.cuda.synchronize()
    a_codes, a_sf = X.quantize_mxfp8(f32(x))
    b_codes, b_sf = X.quantize_mxfp8(f32(w))
    r = np.arange(wl.m) if rows is None else rows
    c = np.arange(wl.n) if cols is None else cols
    b_np = f32(bias) if bias is not None else None
    y_ref = X.gemm_ref_mxfp8(a_codes[r], a_sf[r], b_codes[c], b_sf[c], 1.0, None if b_np is None else b_np[c])
    tol = X.gemm_tolerance_mxfp8(a_codes[r], a_sf[r], b_codes[c], b_sf[c], y_ref)
    got = y.float().cpu().numpy()[np.ix_(r, c)]
    assert_within_tol(got, y_ref, tol, wl.name)


def test_gemm_tiny(F):
    _linear(F, synth.TINY)


@pytest.mark.parametrize("m,n,k", [(1, 8, 64), (100, 200, 192), (130, 264, 320), (257, 392, 4160), (512, 768, 3072)])
def test_gemm_ragged(F, m, n, k):
    _linear(F, synth.LinearWorkload(f"mx_{m}x{n}x{k}", m, k, n, seed=m + n + k))


@pytest.mark.parametrize("m,n,k", [(2341, 2056, 3136), (4608, 3072, 1088)])
def test_gemm_wide_tiles_ragged_sampled(F, m, n, k):
    # shapes that take the 256 x 256 tiles: sampled rows and columns, the last
    # ones and those at 128-row / 128-column boundaries included
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert F.nvfp4_gemm_tile_shape(m, n, sms) == (2, 256, 1)
    rng = np.random.default_rng(m + n)
    rows = np.unique(np.r_[rng.choice(m, 40, replace=False), m - 1, 127, 128, 255, 256])
    cols = np.unique(np.r_[rng.choice(n, 64, replace=False), n - 1, 127, 128, 255, 256])
    _linear(F, synth.LinearWorkload(f"mx_wide_{m}x{n}x{k}", m, k, n, seed=m + n + k), rows=rows, cols=cols)


def test_gemm_mlp_up_sampled(F):
    wl = synth.MLP_UP
    rng = np.random.default_rng(10)
    _linear(F, wl, rows=np.sort(rng.choice(wl.m, 48, replace=False)), cols=np.sort(rng.choice(wl.n, 96, replace=False)))


def test_gemm_bit_exact_when_accumulation_is_exact(F):
    # elements in {0, +-1, +-2, +-0.5}, scales 2^0 / 2^1: every product and
    # partial sum is exactly representable in fp32, so the GPU result must
    # equal the oracle's rounded to bf16 exactly
    rng = np.random.default_rng(11)
    M, Nn, K = 130, 264, 256
    choices = np.array([0x00, 0x38, 0xB8, 0x40, 0xC0, 0x30, 0xB0], np.uint8)  # 0, 1, -1, 2, -2, .5, -.5
    a_codes = rng.choice(choices, (M, K))
    b_codes = rng.choice(choices, (Nn, K))
    a_sf = rng.choice(np.array([127, 128], np.uint8), (M, K // 32))
    b_sf = rng.choice(np.array([127, 128], np.uint8), (Nn, K // 32))
    a = F.MXFP8Tensor(torch.from_numpy(a_codes).cuda(), torch.from_numpy(X.swizzle_sf_mxfp8(a_sf)).cuda(), M, K)
    b = F.MXFP8Tensor(torch.from_numpy(b_codes).cuda(), torch.from_numpy(X.swizzle_sf_mxfp8(b_sf)).cuda(), Nn, K)
    y = F.gemm_mxfp8(a, b, alpha=0.25).float().cpu().numpy()
    y_ref = N.round_to_bf16(X.gemm_ref_mxfp8(a_codes, a_sf, b_codes, b_sf, alpha=0.25))
    assert np.array_equal(y, y_ref)


def test_scale_byte_positions(F):
    # one scale 2^1 at a time, for each of the 4 bytes of a scale word (one
    # 32-element block each) and both operands: a wrong scale-byte selector or
    # row-group placement moves the doubled contribution
    M, Nn, K = 256, 192, 256
    a_codes = np.full((M, K), 0x38, np.uint8)   # 1.0
    b_codes = np.full((Nn, K), 0x38, np.uint8)
    for operand in ("a", "b"):
        for blk in range(K // 32):
            for row in (0, 37, 100, 130):
                a_sf = np.full((M, K // 32), 127, np.uint8)
                b_sf = np.full((Nn, K // 32), 127, np.uint8)
                if operand == "a":
                    a_sf[row, blk] = 128
                else:
                    b_sf[row % Nn, blk] = 128
                a = F.MXFP8Tensor(torch.from_numpy(a_codes).cuda(), torch.from_numpy(X.swizzle_sf_mxfp8(a_sf)).cuda(),
                                  M, K)
                b = F.MXFP8Tensor(torch.from_numpy(b_codes).cuda(), torch.from_numpy(X.swizzle_sf_mxfp8(b_sf)).cuda(),
                                  Nn, K)
                y = F.gemm_mxfp8(a, b).float().cpu().numpy()
                y_ref = N.round_to_bf16(X.gemm_ref_mxfp8(a_codes, a_sf, b_codes, b_sf))
                assert np.array_equal(y, y_ref), (operand, blk, row)


def test_no_kernel_reported_a_fault(F):
    F.nvfp4_check_fault()
