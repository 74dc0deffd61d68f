"""Pins for the oracle's GEMM, dequantization and fused-epilogue math (CPU).

The GEMM is the NVFP4 x NVFP4 linear layer of the "BFL (fp8r / nvfp4)" doc,
section "Kernels" (``mm_fp4`` with ``nvfp4_quantize`` on the activations):
y = alpha * A_hat B_hat^T + bias with alpha = input_scale * weight_scale_2.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def test_closed_form_constant_codes_and_scales():
    # All codes c, all scales s: y = K * (c*s_a*g_a) * (c*s_b*g_b) + bias.
    M, N, K = 3, 5, 128
    c = 0x5  # 3.0
    a_codes = np.full((M, K // 2), c | (c << 4), np.uint8)
    b_codes = np.full((N, K // 2), c | (c << 4), np.uint8)
    a_sf = np.full((M, K // 16), 0x38, np.uint8)  # 1.0
    b_sf = np.full((N, K // 16), 0x30, np.uint8)  # 0.5
    g_a, g_b = np.float32(0.25), np.float32(3.0)
    bias = np.arange(N, dtype=np.float64)
    y = O.gemm_ref(a_codes, a_sf, g_a, b_codes, b_sf, g_b, bias)
    want = K * (3.0 * 1.0 * 0.25) * (3.0 * 0.5 * 3.0) + bias
    assert np.array_equal(y, np.broadcast_to(want, (M, N)))


def test_gemm_equals_triple_loop_brute_force():
    # Independent decode via ml_dtypes and plain Python loops.
    rng = np.random.default_rng(3)
    M, N, K = 3, 4, 64
    a_codes = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    b_codes = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    a_sf = rng.integers(0, 127, (M, K // 16)).astype(np.uint8)
    b_sf = rng.integers(0, 127, (N, K // 16)).astype(np.uint8)
    g_a, g_b = np.float32(0.37), np.float32(1.9)
    bias = rng.standard_normal(N)
    y = O.gemm_ref(a_codes, a_sf, g_a, b_codes, b_sf, g_b, bias)

    def elem(codes, sf, row, k):
        byte = int(codes[row, k // 2])
        nib = byte & 0xF if k % 2 == 0 else byte >> 4
        return float(np.uint8(nib).view(F4)) * float(np.uint8(sf[row, k // 16]).view(F8))

    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += elem(a_codes, a_sf, m, k) * elem(b_codes, b_sf, n, k)
            want = float(g_a) * float(g_b) * acc + bias[n]
            assert abs(y[m, n] - want) <= 1e-12 * max(1.0, abs(want))


def test_dequantize_layout_matches_nibble_order():
    codes = np.array([[0x21, 0x7F]], np.uint8)  # elements: 1(0.5) 2(1.0) F(-6) 7(6)
    sf = np.array([[0x38]], np.uint8)
    x = O.dequantize(np.concatenate([codes, np.zeros((1, 6), np.uint8)], 1), sf, 2.0)
    assert x[0, :4].tolist() == [1.0, 2.0, -12.0, 12.0]


def test_gelu_tanh_matches_torch_and_identities():
    v = np.linspace(-12, 12, 20001)
    ref = torch.nn.functional.gelu(torch.from_numpy(v), approximate="tanh").numpy()
    got = O.gelu_tanh(v)
    assert np.max(np.abs(got - ref)) < 1e-14
    # gelu(v) - gelu(-v) = v (the odd part of GELU is v/2)
    assert np.max(np.abs(O.gelu_tanh(v) - O.gelu_tanh(-v) - v)) < 1e-12
    assert O.gelu_tanh(0.0) == 0.0


def test_epilogue_ref_rounds_applies_act_and_concatenates():
    y = np.array([[1.00390625 + 2 ** -10, -3.0, 0.5, 100.0]])
    out = O.epilogue_ref(y, [(0, 2, O.ACT_NONE), (2, 4, O.ACT_GELU_TANH)])
    assert out[0, 0] == 1.0078125  # rounded up to the next bf16 (tie-free)
    assert out[0, 1] == -3.0
    g = torch.nn.functional.gelu(torch.tensor([0.5, 100.0], dtype=torch.float64), approximate="tanh")
    assert np.array_equal(out[0, 2:], g.to(torch.bfloat16).double().numpy())


def test_w4a4_close_to_bf16_linear():
    # The unquantized-activation fallback "may differ slightly" from the fused
    # W4A4 kernel (BFL doc, section "Kernels"): check the W4A4 result stays
    # within a modest relative error of the plain linear on N(0,1) data.
    rng = np.random.default_rng(4)
    x = O.round_to_bf16(rng.standard_normal((64, 512))).astype(np.float32)
    w = O.round_to_bf16(rng.standard_normal((96, 512)) * 0.02).astype(np.float32)
    gx, gw = O.global_scale(O.tensor_amax(x)), O.global_scale(O.tensor_amax(w))
    xc, xs = O.quantize_nvfp4(x, gx)
    wc, ws = O.quantize_nvfp4(w, gw)
    y = O.gemm_ref(xc, xs, gx, wc, ws, gw)
    y_ref = x.astype(np.float64) @ w.astype(np.float64).T
    rel = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert 0.01 < rel < 0.2


def test_tolerance_is_positive_and_scales_with_operands():
    rng = np.random.default_rng(5)
    x = O.round_to_bf16(rng.standard_normal((8, 64))).astype(np.float32)
    w = O.round_to_bf16(rng.standard_normal((8, 64))).astype(np.float32)
    gx, gw = O.global_scale(O.tensor_amax(x)), O.global_scale(O.tensor_amax(w))
    xc, xs = O.quantize_nvfp4(x, gx)
    wc, ws = O.quantize_nvfp4(w, gw)
    y = O.gemm_ref(xc, xs, gx, wc, ws, gw)
    tol = O.gemm_tolerance(xc, xs, gx, wc, ws, gw, y)
    assert np.all(tol > 0)
    # the bound is ~2e-3 of |a||b|, far below |a||b| itself
    an = np.linalg.norm(O.dequantize(xc, xs, gx), axis=1)
    assert np.all(tol <= 2e-3 * an[:, None] * an.max() * 100 + 1e-2 * np.abs(y))


@pytest.mark.parametrize("amax", [1.0, 2688.0, 1e-3, 12345.678])
def test_global_scale_is_amax_over_2688(amax):
    g = O.global_scale(amax)
    assert g.dtype == np.float32
    assert g == np.float32(np.float32(amax) / np.float32(2688.0))
    assert abs(float(g) * 2688.0 / amax - 1) < 1e-6


# --------------------------------------------------------------------------
# W4A16: weights dequantized to bf16, regular linear
# --------------------------------------------------------------------------

def test_dequantize_to_bf16_with_power_of_two_scale_is_the_exact_product_rounded():
    # with g a power of two every fp32 step is exact, so the result is the
    # bf16 rounding (torch's) of e2m1(code) * e4m3(scale) * g decoded by ml_dtypes
    rng = np.random.default_rng(60)
    rows, K = 40, 256
    codes = rng.integers(0, 256, (rows, K // 2)).astype(np.uint8)
    sf = rng.integers(0, 127, (rows, K // 16)).astype(np.uint8)
    for g in (1.0, 2.0 ** -7, 2.0 ** 12):
        q = O.unpack_codes(codes)
        exact = (q.view(F4).astype(np.float64) * np.repeat(sf.view(F8).astype(np.float64), 16, axis=1) * g)
        want = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).float().numpy()
        assert np.array_equal(O.dequantize_to_bf16(codes, sf, g), want)


def test_dequantize_to_bf16_rounding_bound():
    rng = np.random.default_rng(61)
    codes = rng.integers(0, 256, (64, 64)).astype(np.uint8)
    sf = rng.integers(1, 127, (64, 8)).astype(np.uint8)
    g = 0.00731
    v = O.dequantize_to_bf16(codes, sf, g)
    exact = O.dequantize(codes, sf, g)   # fp64
    # fp32 then bf16 rounding: within half a bf16 ulp plus half an fp32 ulp
    bound = np.abs(exact) * (2.0 ** -8 + 2.0 ** -24) + 1e-45
    assert np.all(np.abs(v - exact) <= bound)


def test_linear_w4a16_is_the_bf16_linear_of_the_dequantized_weight():
    rng = np.random.default_rng(62)
    x = O.round_to_bf16(rng.standard_normal((5, 64))).astype(np.float32)
    codes = rng.integers(0, 256, (7, 32)).astype(np.uint8)
    sf = rng.integers(40, 60, (7, 4)).astype(np.uint8)
    bias = rng.standard_normal(7)
    y = O.linear_w4a16_ref(x, codes, sf, 0.5, bias)
    w = O.dequantize_to_bf16(codes, sf, 0.5)
    for m in range(5):
        for n in range(7):
            assert y[m, n] == pytest.approx(sum(float(x[m, k]) * float(w[n, k]) for k in range(64)) + bias[n],
                                            rel=1e-12, abs=1e-12)
