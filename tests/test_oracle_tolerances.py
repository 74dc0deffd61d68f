"""Pins for the GEMM tolerances of the three block formats (CPU only).

Each tolerance is ``2e-3 * |alpha| * ||a_hat_m|| * ||b_hat_n|| + 1e-2 * |y_ref|``
around the float64 reference (fp32 accumulation error plus the bf16 output
rounding).  Two properties pin it from outside its own formula:

* it admits what a tensor-core kernel may legitimately return: products of
  the exactly representable block-scaled operands accumulated in fp32 in
  64-element k-chunks taken in any order, the per-tensor or per-row scales
  applied in fp32, the bias added, the result rounded to bf16;
* it rejects the plausible kernel mistakes: one k-block dropped, one block
  scale applied twice, the bias left out, the per-row scales of two rows
  exchanged, the per-tensor scale of one operand forgotten.
"""
import numpy as np
import pytest

from oracle import fp8row_ref as R
from oracle import mxfp8_ref as X
from oracle import nvfp4_ref as O

M, N, K = 24, 40, 512


def _data(seed, m, k, spread):
    rng = np.random.default_rng(seed)
    x = rng.laplace(size=(m, k)) * np.exp(rng.normal(0, spread, (1, k)))  # outlier channels
    return O.round_to_bf16(x).astype(np.float32)


def _fp32_chunked(a32, b32, chunk, seed):
    """sum_k a[m,k] b[n,k]: fp32 products, fp32 sums within each k-chunk,
    the chunk sums added in fp32 in a random order."""
    order = np.random.default_rng(seed).permutation(a32.shape[1] // chunk)
    acc = np.zeros((a32.shape[0], b32.shape[0]), np.float32)
    for c in order:
        part = np.zeros_like(acc)
        for k in range(c * chunk, (c + 1) * chunk):
            part = part + np.outer(a32[:, k], b32[:, k]).astype(np.float32)
        acc = acc + part
    return acc


def _bias(y_ref, seed):
    return O.round_to_bf16(np.random.default_rng(seed).normal(0, 0.5 * np.std(y_ref), y_ref.shape[1]))


def _exceeds(y, y_ref, tol):
    return bool(np.any(np.abs(y - y_ref) > tol))


# ---------------------------------------------------------------- NVFP4

def _nvfp4_case(seed):
    x, w = _data(seed, M, K, 1.0), _data(seed + 1, N, K, 0.5)
    gx, gw = O.global_scale(O.tensor_amax(x)), O.global_scale(O.tensor_amax(w))
    xc, xs = O.quantize_nvfp4(x, gx)
    wc, ws = O.quantize_nvfp4(w, gw)
    a32 = O.dequantize(xc, xs, 1.0).astype(np.float32)   # e2m1 * e4m3: exact in fp32
    b32 = O.dequantize(wc, ws, 1.0).astype(np.float32)
    y0 = O.gemm_ref(xc, xs, gx, wc, ws, gw)
    bias = _bias(y0, seed + 2)
    y_ref = O.gemm_ref(xc, xs, gx, wc, ws, gw, bias)
    tol = O.gemm_tolerance(xc, xs, gx, wc, ws, gw, y_ref)
    alpha = np.float32(gx) * np.float32(gw)
    return a32, b32, alpha, bias, y_ref, tol, gx


def _nvfp4_out(a32, b32, alpha, bias, seed=0):
    acc = _fp32_chunked(a32, b32, 64, seed)
    return O.round_to_bf16((np.float32(alpha) * acc + bias.astype(np.float32)).astype(np.float32))


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_nvfp4_tolerance_admits_fp32_accumulation_in_any_chunk_order(seed):
    a32, b32, alpha, bias, y_ref, tol, _ = _nvfp4_case(seed)
    for order_seed in range(3):
        assert not _exceeds(_nvfp4_out(a32, b32, alpha, bias, order_seed), y_ref, tol)


def test_nvfp4_tolerance_rejects_plausible_kernel_mistakes():
    a32, b32, alpha, bias, y_ref, tol, gx = _nvfp4_case(7)
    dropped = a32.copy()
    dropped[:, 16 * 5:16 * 6] = 0                              # one 16-element block lost
    assert _exceeds(_nvfp4_out(dropped, b32, alpha, bias), y_ref, tol)
    twice = a32.copy()
    twice[:, 16 * 9:16 * 10] *= 2                              # one block scale applied twice
    assert _exceeds(_nvfp4_out(twice, b32, alpha, bias), y_ref, tol)
    assert _exceeds(_nvfp4_out(a32, b32, alpha, np.zeros_like(bias)), y_ref, tol)   # bias left out
    assert _exceeds(_nvfp4_out(a32, b32, np.float32(gx), bias), y_ref, tol)         # g_w forgotten


# ---------------------------------------------------------------- MXFP8

def _mxfp8_case(seed, alpha):
    x, w = _data(seed, M, K, 1.0), _data(seed + 1, N, K, 0.5)
    ac, asf = X.quantize_mxfp8(x)
    bc, bsf = X.quantize_mxfp8(w)
    a32 = X.dequantize_mxfp8(ac, asf).astype(np.float32)  # e4m3 * 2^k: exact in fp32
    b32 = X.dequantize_mxfp8(bc, bsf).astype(np.float32)
    y0 = X.gemm_ref_mxfp8(ac, asf, bc, bsf, alpha)
    bias = _bias(y0, seed + 2)
    y_ref = X.gemm_ref_mxfp8(ac, asf, bc, bsf, alpha, bias)
    tol = X.gemm_tolerance_mxfp8(ac, asf, bc, bsf, y_ref, alpha)
    return a32, b32, bias, y_ref, tol


def _mxfp8_out(a32, b32, alpha, bias, seed=0):
    acc = _fp32_chunked(a32, b32, 64, seed)
    return O.round_to_bf16((np.float32(alpha) * acc + bias.astype(np.float32)).astype(np.float32))


@pytest.mark.parametrize("seed,alpha", [(11, 1.0), (12, 0.25), (13, 3.0)])
def test_mxfp8_tolerance_admits_fp32_accumulation_in_any_chunk_order(seed, alpha):
    a32, b32, bias, y_ref, tol = _mxfp8_case(seed, alpha)
    for order_seed in range(3):
        assert not _exceeds(_mxfp8_out(a32, b32, alpha, bias, order_seed), y_ref, tol)


def test_mxfp8_tolerance_rejects_plausible_kernel_mistakes():
    alpha = 0.5
    a32, b32, bias, y_ref, tol = _mxfp8_case(17, alpha)
    dropped = a32.copy()
    dropped[:, 32 * 3:32 * 4] = 0                              # one 32-element block lost
    assert _exceeds(_mxfp8_out(dropped, b32, alpha, bias), y_ref, tol)
    twice = b32.copy()
    twice[:, 32 * 7:32 * 8] *= 2                               # a block exponent off by one
    assert _exceeds(_mxfp8_out(a32, twice, alpha, bias), y_ref, tol)
    assert _exceeds(_mxfp8_out(a32, b32, alpha, np.zeros_like(bias)), y_ref, tol)
    assert _exceeds(_mxfp8_out(a32, b32, 1.0, bias), y_ref, tol)                    # alpha forgotten


# ---------------------------------------------------------------- row-wise FP8

def _fp8row_case(seed):
    x, w = _data(seed, M, K, 1.0), _data(seed + 1, N, K, 0.5)
    x *= np.float32(2.0) ** np.random.default_rng(seed).integers(-6, 6, (M, 1)).astype(np.float32)
    ac, sa = R.quantize_fp8_rowwise(x)
    bc, sb = R.quantize_fp8_rowwise(w)
    a32 = O.e4m3_decode(ac).astype(np.float32)
    b32 = O.e4m3_decode(bc).astype(np.float32)
    y0 = R.gemm_ref_fp8row(ac, sa, bc, sb)
    bias = _bias(y0, seed + 2)
    y_ref = R.gemm_ref_fp8row(ac, sa, bc, sb, bias)
    tol = R.gemm_tolerance_fp8row(ac, sa, bc, sb, y_ref)
    return a32, b32, sa, sb, bias, y_ref, tol


def _fp8row_out(a32, b32, sa, sb, bias, seed=0):
    acc = _fp32_chunked(a32, b32, 64, seed)
    scale = (sa.astype(np.float32)[:, None] * sb.astype(np.float32)[None, :]).astype(np.float32)
    return O.round_to_bf16((scale * acc + bias.astype(np.float32)).astype(np.float32))


@pytest.mark.parametrize("seed", [21, 22, 23])
def test_fp8row_tolerance_admits_fp32_accumulation_in_any_chunk_order(seed):
    a32, b32, sa, sb, bias, y_ref, tol = _fp8row_case(seed)
    for order_seed in range(3):
        assert not _exceeds(_fp8row_out(a32, b32, sa, sb, bias, order_seed), y_ref, tol)


def test_fp8row_tolerance_rejects_plausible_kernel_mistakes():
    a32, b32, sa, sb, bias, y_ref, tol = _fp8row_case(27)
    dropped = a32.copy()
    dropped[:, 64 * 2:64 * 3] = 0                              # one k-chunk lost
    assert _exceeds(_fp8row_out(dropped, b32, sa, sb, bias), y_ref, tol)
    swapped = sa.copy()
    swapped[[0, 1]] = swapped[[1, 0]]                          # two rows' scales exchanged
    assert sa[0] != sa[1]
    assert _exceeds(_fp8row_out(a32, b32, swapped, sb, bias), y_ref, tol)
    assert _exceeds(_fp8row_out(a32, b32, sa, sb, np.zeros_like(bias)), y_ref, tol)
    assert _exceeds(_fp8row_out(a32, b32, sa, np.ones_like(sb), bias), y_ref, tol)   # weight scales forgotten
