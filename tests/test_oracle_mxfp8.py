"""Pins for the MXFP8 oracle (CPU only).

MXFP8: 8-bit E4M3 elements in 32-element blocks sharing one power-of-two
scale, per the Open Compute Project microscaling standard ("NVIDIA FP4 format"
news page, paragraph 1).  The pins check the oracle against ml_dtypes' format
definitions, against blocks that must round-trip, against brute-force nearest
search, and against the special blocks (zeros, saturation), not against a
retyping of its own formulas.
"""
import ml_dtypes
import numpy as np
import pytest

from oracle import mxfp8_ref as X
from oracle import nvfp4_ref as N

F8 = ml_dtypes.float8_e4m3fn
E8 = ml_dtypes.float8_e8m0fnu


def test_e8m0_decode_matches_ml_dtypes_on_every_byte():
    b = np.arange(256, dtype=np.uint8)
    want = b.view(E8).astype(np.float64)
    got = X.e8m0_decode(b)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def test_signed_e4m3_encode_matches_ml_dtypes_after_clamping():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-600, 600, 200000), rng.uniform(-1, 1, 50000) * 2.0 ** -6,
                        np.array([0.0, -0.0, 448.0, -448.0, 464.0, 1e9, -1e9])])
    want = np.clip(v, -448, 448).astype(F8).view(np.uint8)
    got = X.e4m3_encode_signed(v)
    assert np.array_equal(got, want)
    assert X.e4m3_encode_signed(np.array([-0.0]))[0] == 0x80


def _representable_blocks(rng, n, k):
    """Blocks of E4M3 values times 2^k whose largest magnitude is in [256, 448]
    (so floor(log2 amax) = 8 + k): the quantizer must return exactly these
    codes with scale byte k + 127."""
    codes = rng.integers(0, 256, (n, 32)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x01  # no NaN
    top = rng.integers(0x78, 0x7F, n).astype(np.uint8)  # 256 .. 448
    codes[np.arange(n), rng.integers(0, 32, n)] = top | np.where(rng.random(n) < 0.5, 0x80, 0).astype(np.uint8)
    # keep every other element below the top one
    x = codes.view(F8).astype(np.float64) * 2.0 ** k
    return x, codes


@pytest.mark.parametrize("k", [-20, -3, 0, 5, 100, -110])
def test_representable_blocks_round_trip(k):
    rng = np.random.default_rng(k + 200)
    x, codes = _representable_blocks(rng, 300, k)
    got_codes, sf = X.quantize_mxfp8(x.astype(np.float32).reshape(300, 32))
    assert np.all(sf == k + 127)
    # fp32 holds every value exactly here except E4M3 subnormals scaled below fp32's range
    assert np.array_equal(got_codes, codes)


def test_block_maximum_lands_between_256_and_448():
    rng = np.random.default_rng(1)
    x = N.round_to_bf16(rng.laplace(size=(64, 256)) * 10.0 ** rng.uniform(-8, 8, (64, 1))).astype(np.float32)
    codes, sf = X.quantize_mxfp8(x)
    mags = np.abs(N.e4m3_decode(codes)).reshape(64, 8, 32).max(axis=2)
    assert np.all((mags >= 256) & (mags <= 448))


def test_codes_are_the_nearest_e4m3_value_of_the_scaled_input():
    rng = np.random.default_rng(2)
    x = N.round_to_bf16(rng.standard_normal((40, 128)) * 3.0).astype(np.float32)
    codes, sf = X.quantize_mxfp8(x)
    scale = X.e8m0_decode(sf).repeat(32, axis=1)
    t = (x.astype(np.float64) / scale)
    table = N.e4m3_decode(np.arange(256, dtype=np.uint8))
    finite = ~np.isnan(table)
    cand = table[finite]
    cand_bytes = np.arange(256)[finite]
    for r in range(40):
        for c in range(128):
            v = min(max(t[r, c], -448.0), 448.0)
            d = np.abs(cand - v)
            best = cand_bytes[d == d.min()]
            if len(best) > 1:  # tie (or +-0): the even mantissa, matching sign
                best = [b for b in best if (b & 1) == 0 and ((b & 0x80) != 0) == (np.signbit(t[r, c]))] or best
            assert codes[r, c] in set(int(b) for b in best), (r, c, t[r, c], codes[r, c], best)


def test_zero_and_saturating_blocks():
    x = np.zeros((3, 64), np.float32)
    x[0, 5] = -0.0
    x[1, :32] = np.linspace(-1, 1, 32)
    x[1, 7] = 511.0                         # floor(log2) = 8: scale 2^0, 511 saturates to 448
    x[2, 32:] = 2.0 ** -140                 # fp32 subnormal block
    codes, sf = X.quantize_mxfp8(x)
    assert sf[0, 0] == 0 and sf[0, 1] == 0 and not (codes[0] & 0x7F).any()
    assert codes[0, 5] == 0x80
    assert sf[1, 0] == 127 and codes[1, 7] == 0x7E
    assert sf[2, 1] == 0  # floor(log2 2^-140) - 8 = -148 clamps to -127


def test_quantization_error_bound():
    rng = np.random.default_rng(3)
    x = N.round_to_bf16(rng.laplace(size=(128, 256))).astype(np.float32)
    codes, sf = X.quantize_mxfp8(x)
    xhat = X.dequantize_mxfp8(codes, sf)
    scale = X.e8m0_decode(sf).repeat(32, axis=1)
    # 3 mantissa bits: half a step is 2^-4 of the value above 2^-6 (times the
    # scale), and half the subnormal spacing 2^-10 below it; a block maximum
    # in (448, 512) * scale saturates to 448 * scale
    bound = np.maximum(np.maximum(np.abs(x) * 2.0 ** -4, scale * 2.0 ** -10), np.abs(x) - 448.0 * scale)
    assert np.all(np.abs(xhat - x) <= bound * 1.0000001)


def test_swizzle_equals_the_nvfp4_atom_layout_and_is_a_bijection():
    rng = np.random.default_rng(4)
    for rows, k in [(128, 128), (300, 4096), (1, 32), (129, 96)]:
        sf = rng.integers(0, 255, (rows, k // 32)).astype(np.uint8)
        swz = X.swizzle_sf_mxfp8(sf)
        assert swz.size == X.sf_bytes_mxfp8(rows, k)
        # the same 512-byte atoms as NVFP4's scale buffer, one column per 32 elements
        assert np.array_equal(swz, N.swizzle_sf(sf))
        assert np.array_equal(X.unswizzle_sf_mxfp8(swz, rows, k), sf)


def test_gemm_matches_a_brute_force_triple_loop():
    rng = np.random.default_rng(5)
    M, Nn, K = 3, 4, 64
    a_codes = rng.integers(0, 256, (M, K)).astype(np.uint8)
    b_codes = rng.integers(0, 256, (Nn, K)).astype(np.uint8)
    a_codes[(a_codes & 0x7F) == 0x7F] = 0
    b_codes[(b_codes & 0x7F) == 0x7F] = 0
    a_sf = rng.integers(110, 140, (M, K // 32)).astype(np.uint8)
    b_sf = rng.integers(110, 140, (Nn, K // 32)).astype(np.uint8)
    bias = rng.standard_normal(Nn)
    y = X.gemm_ref_mxfp8(a_codes, a_sf, b_codes, b_sf, alpha=0.5, bias=bias)
    for m in range(M):
        for n in range(Nn):
            acc = 0.0
            for k in range(K):
                av = float(a_codes[m, k:k + 1].view(F8)[0]) * 2.0 ** (int(a_sf[m, k // 32]) - 127)
                bv = float(b_codes[n, k:k + 1].view(F8)[0]) * 2.0 ** (int(b_sf[n, k // 32]) - 127)
                acc += av * bv
            assert y[m, n] == pytest.approx(0.5 * acc + bias[n], rel=1e-12, abs=1e-300)


def test_block_exponent_is_floor_log2_in_exact_arithmetic():
    # 2^e <= a < 2^(e+1), checked with exact rationals, on powers of two and
    # their neighbours, random normals, and fp32 subnormals
    from fractions import Fraction
    rng = np.random.default_rng(45)
    a = [np.float32(2.0 ** e) for e in range(-149, 128)]
    a += [np.nextafter(v, np.float32(0)) for v in a[1:]] + [np.nextafter(v, np.float32(np.inf)) for v in a[:-1]]
    a += list(rng.uniform(1, 2, 300).astype(np.float32) * np.float32(2.0) ** rng.integers(-126, 127, 300))
    a += list((rng.integers(1, 1 << 23, 100).astype(np.uint32)).view(np.float32))   # subnormals
    a = np.array(a, np.float32)
    a = a[np.isfinite(a) & (a > 0)]
    e = X.block_exponent(a)
    for v, k in zip(a, e):
        f = Fraction(float(v))
        assert Fraction(2) ** int(k) <= f < Fraction(2) ** (int(k) + 1), (v, k)
