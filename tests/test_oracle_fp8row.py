"""Pins for the row-wise FP8 oracle (CPU only).

Row-wise FP8: E4M3 values with one fp32 scale per row ("BFL (fp8r / nvfp4)"
doc, ``fp8r`` bullet).  Checked against ml_dtypes' E4M3, closed forms, the
row maximum landing on the top code, brute-force nearest codes and a
triple-loop GEMM.
"""
import ml_dtypes
import numpy as np
import pytest

from oracle import fp8row_ref as R
from oracle import nvfp4_ref as N

F8 = ml_dtypes.float8_e4m3fn


@pytest.mark.parametrize("k", [-30, -4, 0, 9, 60])
def test_row_scale_closed_form_for_power_of_two_maxima(k):
    # amax = 448 * 2^k (a bf16 value): s = 2^k exactly, and x / s is exact
    rng = np.random.default_rng(k + 40)
    x = N.round_to_bf16(rng.uniform(-1, 1, (16, 96)) * 448.0 * 2.0 ** k).astype(np.float32)
    x[:, 3] = 448.0 * 2.0 ** k
    codes, s = R.quantize_fp8_rowwise(x)
    assert np.all(s == np.float32(2.0 ** k))
    want = np.clip(x / np.float32(2.0 ** k), -448, 448).astype(F8).view(np.uint8)
    assert np.array_equal(codes, want)


def test_row_maximum_lands_on_the_top_code():
    rng = np.random.default_rng(41)
    x = N.round_to_bf16(rng.laplace(size=(64, 300)) * 10.0 ** rng.uniform(-20, 20, (64, 1))).astype(np.float32)
    codes, s = R.quantize_fp8_rowwise(x)
    idx = np.argmax(np.abs(x), axis=1)
    top = codes[np.arange(64), idx]
    assert np.all((top & 0x7F) == 0x7E)
    assert np.all(((top & 0x80) != 0) == (x[np.arange(64), idx] < 0))


def test_codes_are_the_nearest_e4m3_value():
    rng = np.random.default_rng(42)
    x = N.round_to_bf16(rng.standard_normal((12, 200))).astype(np.float32)
    codes, s = R.quantize_fp8_rowwise(x)
    t = (x / s[:, None]).astype(np.float32).astype(np.float64)
    table = N.e4m3_decode(np.arange(256, dtype=np.uint8))
    ok = ~np.isnan(table)
    for r in range(12):
        for c in range(200):
            v = min(max(t[r, c], -448.0), 448.0)
            d = np.abs(table[ok] - v)
            best = np.arange(256)[ok][d == d.min()]
            assert codes[r, c] in set(int(b) for b in best)
    # and ml_dtypes' conversion of the same fp32 quotient agrees on every value
    want = np.clip(t, -448, 448).astype(F8).view(np.uint8)
    assert np.array_equal(codes, want)


def test_zero_row():
    x = np.zeros((2, 64), np.float32)
    x[0, 3] = -0.0
    x[1, 5] = 2.5
    codes, s = R.quantize_fp8_rowwise(x)
    assert s[0] == 0 and codes[0, 3] == 0x80 and not (codes[0] & 0x7F).any()
    assert s[1] == np.float32(2.5) / np.float32(448.0) and codes[1, 5] == 0x7E


def test_gemm_matches_a_triple_loop():
    rng = np.random.default_rng(43)
    M, Nn, K = 3, 5, 40
    a = rng.integers(0, 256, (M, K)).astype(np.uint8)
    b = rng.integers(0, 256, (Nn, K)).astype(np.uint8)
    a[(a & 0x7F) == 0x7F] = 0
    b[(b & 0x7F) == 0x7F] = 0
    sa = rng.uniform(0.1, 2, M).astype(np.float32)
    sb = rng.uniform(0.1, 2, Nn).astype(np.float32)
    bias = rng.standard_normal(Nn)
    y = R.gemm_ref_fp8row(a, sa, b, sb, bias)
    for m in range(M):
        for n in range(Nn):
            acc = sum(float(a[m, k:k + 1].view(F8)[0]) * float(b[n, k:k + 1].view(F8)[0]) for k in range(K))
            assert y[m, n] == pytest.approx(float(sa[m]) * float(sb[n]) * acc + bias[n], rel=1e-12, abs=1e-300)


def test_dequantize_is_the_e4m3_value_times_the_row_scale():
    # every non-NaN byte against ml_dtypes' E4M3, times an fp32 row scale, in
    # exact float64 arithmetic
    codes = np.arange(256, dtype=np.uint8)
    codes = codes[(codes & 0x7F) != 0x7F].reshape(2, 127)
    s = np.array([0.75, 2.0 ** -20], np.float32)
    got = R.dequantize_fp8_rowwise(codes, s)
    want = codes.view(F8).astype(np.float64) * s.astype(np.float64)[:, None]
    assert np.array_equal(got, want)


def test_representable_rows_round_trip():
    # rows of E4M3 values times a power of two, with the top code present:
    # s is that power of two and quantize -> dequantize gives the row back
    rng = np.random.default_rng(44)
    vals = N.e4m3_decode(np.arange(256, dtype=np.uint8))
    vals = vals[~np.isnan(vals)]
    for k in (-12, 0, 7):
        x = (rng.choice(vals, (4, 96)) * 2.0 ** k).astype(np.float32)
        x[:, 0] = 448.0 * 2.0 ** k
        codes, s = R.quantize_fp8_rowwise(x)
        assert np.all(s == np.float32(2.0 ** k))
        assert np.array_equal(R.dequantize_fp8_rowwise(codes, s), x.astype(np.float64))
