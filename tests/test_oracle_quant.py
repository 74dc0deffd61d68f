"""Pins for the oracle's block quantizer and scale-factor layout (CPU only).

The block quantizer follows the NVFP4 two-level scaling: per-tensor fp32
scale plus one E4M3 scale per 16 elements ("NVIDIA FP4 format" news page,
paragraph 1; "BFL (fp8r / nvfp4)" doc, ``nvfp4`` bullet).  The pins below do
not re-type its formulas: they check it against values that must round-trip
exactly, against brute-force nearest-code search, and against the special
cases (zero blocks, scale saturation, scale underflow).
"""
import ml_dtypes
import numpy as np
import pytest

import oracle as O

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def _representable_blocks(rng, n_blocks, g):
    """Blocks x = code * s * g whose amax is exactly 6 * s * g, so that the
    quantizer must return exactly (codes, s)."""
    s_bytes = rng.integers(1, 127, n_blocks).astype(np.uint8)
    s_val = s_bytes.view(F8).astype(np.float64)
    codes = rng.integers(0, 16, (n_blocks, 16)).astype(np.uint8)
    pin = rng.integers(0, 16, n_blocks)
    codes[np.arange(n_blocks), pin] = np.where(rng.random(n_blocks) < 0.5, 0x7, 0xF)
    x = codes.view(F4).astype(np.float64) * s_val[:, None] * g
    return x, codes, s_bytes


@pytest.mark.parametrize("g", [1.0, 2.0 ** -3, 2.0 ** 5, 2.0 ** -20])
def test_representable_blocks_round_trip_exactly(g):
    rng = np.random.default_rng(1)
    x, codes, s_bytes = _representable_blocks(rng, 4096, g)
    x32 = x.astype(np.float32)
    assert np.array_equal(x32.astype(np.float64), x)  # inputs exact in fp32 (and bf16)
    got_codes, got_s = O.quantize_nvfp4(x32.reshape(256, 256), g)
    assert np.array_equal(got_s.reshape(-1), s_bytes)
    # -0 and +0 both decode to zero; compare values, then signs of non-zeros
    got_q = O.unpack_codes(got_codes).reshape(-1, 16)
    assert np.array_equal(got_q.view(F4).astype(np.float64), codes.view(F4).astype(np.float64))
    assert np.array_equal(O.dequantize(got_codes, got_s, g).reshape(-1, 16), x)


def test_zero_block_gives_zero_bytes():
    x = np.zeros((4, 64), np.float32)
    x[1, 16:32] = 3.0  # one non-zero block among zero blocks
    codes, s = O.quantize_nvfp4(x, O.global_scale(3.0))
    assert s[0].tolist() == [0, 0, 0, 0] and s[1, 0] == 0 and s[1, 2] == 0
    assert s[1, 1] != 0
    q = O.unpack_codes(codes)
    assert np.all(q[0] == 0) and np.all(q[1, :16] == 0) and np.all(q[1, 32:] == 0)


def test_negative_zero_input_in_zero_block_gives_plus_zero_code():
    x = np.zeros((1, 16), np.float32)
    x[0, 3] = -0.0
    codes, s = O.quantize_nvfp4(x, 1.0)
    assert s[0, 0] == 0 and np.all(codes == 0)


def test_scale_underflow_zeroes_the_block():
    # amax/(6g) below half the smallest E4M3 subnormal (2^-10) rounds to 0.
    g = np.float32(1.0)
    x = np.full((1, 16), 6 * 2.0 ** -11, np.float32)
    codes, s = O.quantize_nvfp4(x, g)
    assert s[0, 0] == 0 and np.all(codes == 0)
    x = np.full((1, 16), 6 * 2.0 ** -9, np.float32)  # exactly the smallest scale
    codes, s = O.quantize_nvfp4(x, g)
    assert s[0, 0] == 0x01 and np.all(O.unpack_codes(codes) == 0x7)


def test_scale_saturates_at_448_and_codes_at_6():
    g = np.float32(2.0 ** -4)
    x = np.zeros((1, 32), np.float32)
    x[0, :16] = np.linspace(-100.0, 100.0, 16)       # within 448 * 6 * g = 168
    x[0, 16:] = np.linspace(-1e4, 1e4, 16)           # far beyond it
    codes, s = O.quantize_nvfp4(x, g)
    assert s[0, 1] == 0x7E
    q = O.unpack_codes(codes)[0, 16:]
    assert q[0] == 0xF and q[-1] == 0x7
    # every element of a saturated block is the nearest code under scale 448
    xhat = O.dequantize(codes, s, g)[0, 16:]
    step = 448 * g
    assert np.all(np.abs(xhat) <= 6 * step)


def _brute_force_codes(x, s_byte, g):
    """Nearest E2M1 code to x / (s*g) by scanning all 16 codes (values from
    ml_dtypes), ties to the even code, saturating."""
    vals = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)
    scale = float(np.uint8(s_byte).view(F8)) * g
    out = []
    for v in x:
        d = np.abs(vals * scale - v)
        cand = np.flatnonzero(d == d.min())
        # prefer the even code among equal-distance ones; among +0/-0 follow the sign
        cand_even = [c for c in cand if (c & 1) == 0] or list(cand)
        if len(cand_even) > 1:
            cand_even = [c for c in cand_even if bool(c & 8) == bool(np.signbit(v))] or cand_even
        out.append(cand_even[0])
    return np.array(out, dtype=np.uint8)


def test_codes_equal_brute_force_nearest_with_power_of_two_scales():
    # With s and g powers of two, 1/(s*g) is exact, so the quantizer's scaled
    # value is exactly x/(s*g) and must pick the brute-force nearest code.
    rng = np.random.default_rng(5)
    g = 2.0 ** -2
    pow2_bytes = [b for b in range(1, 127) if (b & 7) == 0 or b < 8 and (b & (b - 1)) == 0]
    checked = 0
    for trial in range(600):
        x = (rng.standard_normal(16) * rng.choice([0.01, 1, 30])).astype(np.float32)
        # round x to bf16 so it is a legal input
        x = O.round_to_bf16(x.astype(np.float64)).astype(np.float32)
        codes, s = O.quantize_nvfp4(x.reshape(1, 16), g)
        if int(s[0, 0]) not in pow2_bytes:
            continue
        want = _brute_force_codes(x.astype(np.float64), s[0, 0], g)
        got = O.unpack_codes(codes)[0]
        assert np.array_equal(got, want), (x, got, want)
        checked += 1
    assert checked >= 20


def test_codes_equal_brute_force_nearest_away_from_ties():
    rng = np.random.default_rng(6)
    x = O.round_to_bf16(rng.laplace(size=(64, 16)) * 3).astype(np.float32)
    g = O.global_scale(np.abs(x).max())
    codes, s = O.quantize_nvfp4(x, g)
    q = O.unpack_codes(codes)
    for b in range(64):
        if s[b, 0] == 0:
            continue
        scale = float(np.uint8(s[b, 0]).view(F8)) * float(g)
        want = _brute_force_codes(x[b].astype(np.float64), s[b, 0], float(g))
        # away from the midpoints between grid values the rounding of 1/(s*g)
        # cannot change the answer
        u = np.abs(x[b].astype(np.float64)) / scale
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
        near_tie = np.min(np.abs(u[:, None] - mids[None, :]), axis=1) < 1e-5
        assert np.array_equal(q[b][~near_tie], want[~near_tie])


def test_block_scale_is_nearest_e4m3_of_amax_over_6g():
    rng = np.random.default_rng(8)
    x = O.round_to_bf16(rng.standard_normal((128, 64)) * 5).astype(np.float32)
    g = np.float32(0.0123)
    _, s = O.quantize_nvfp4(x, g)
    vals = np.array([float(np.uint8(b).view(F8)) for b in range(127)])
    amax = np.abs(x.reshape(128, 4, 16)).max(axis=2).astype(np.float64)
    t = amax / (6 * float(g))
    for i in range(128):
        for j in range(4):
            d = np.abs(vals - min(t[i, j], 448.0))
            # the fp32 rounding of amax/(6g) can only matter right at a tie
            best = np.flatnonzero(d <= d.min() * (1 + 1e-6) + 1e-30)
            assert s[i, j] in best


def test_quantization_error_bound():
    # Each element is within half a code step of its input unless its block
    # saturated: |x_hat - x| <= s*g (largest half-step of the E2M1 grid is 1).
    rng = np.random.default_rng(9)
    x = O.round_to_bf16(rng.laplace(size=(256, 256))).astype(np.float32)
    g = O.global_scale(np.abs(x).max())
    codes, s = O.quantize_nvfp4(x, g)
    xhat = O.dequantize(codes, s, g)
    step = (O.e4m3_decode(s) * float(g)).repeat(16, axis=1)
    assert np.all(np.abs(xhat - x) <= step * 1.0000001 + 1e-45)


# --------------------------------------------------------------------------
# Dynamic (measured) per-tensor scale
# --------------------------------------------------------------------------

@pytest.mark.parametrize("k", [-20, -3, 0, 7, 40])
def test_dynamic_scale_closed_form_for_power_of_two_amax(k):
    # amax = 6 * 448 * 2^k is a bf16 value (21 * 2^(7+k)), so g = 2^k exactly.
    rng = np.random.default_rng(k + 50)
    x = O.round_to_bf16(rng.uniform(-1, 1, (64, 128)) * 2688.0 * 2.0 ** k).astype(np.float32)
    x[17, 33] = -2688.0 * 2.0 ** k
    amax, g = O.dynamic_scale(x)
    assert amax == np.float32(2688.0 * 2.0 ** k)
    assert g == np.float32(2.0 ** k)


def test_dynamic_scale_puts_the_largest_element_on_the_top_code():
    # The tensor's largest element sits at the top of both formats: its block
    # scale is the largest E4M3 value (448, byte 0x7E) and its code is +-6.
    rng = np.random.default_rng(51)
    for trial in range(40):
        x = O.round_to_bf16(rng.laplace(size=(32, 256)) * 10.0 ** rng.uniform(-6, 6)).astype(np.float32)
        codes, sf, amax, g = O.quantize_dynamic(x)
        r, c = np.unravel_index(np.argmax(np.abs(x)), x.shape)
        assert sf[r, c // 16] == 0x7E
        q = O.unpack_codes(codes)[r, c]
        assert q == (0x7 if x[r, c] > 0 else 0xF)


def test_dynamic_scale_of_an_all_zero_tensor_is_zero_and_output_is_zero():
    x = np.zeros((8, 64), np.float32)
    x[3, 5] = -0.0
    codes, sf, amax, g = O.quantize_dynamic(x)
    assert amax == 0 and g == 0
    assert not codes.any() and not sf.any()


def test_dynamic_scale_is_clamped_into_the_accepted_range():
    tiny = np.full((4, 64), 2.0 ** -100, np.float32)   # amax / 2688 < 2^-64
    huge = np.full((4, 64), 2.0 ** 120, np.float32)    # amax / 2688 > 2^64
    assert O.dynamic_scale(tiny)[1] == O.G_MIN
    assert O.dynamic_scale(huge)[1] == O.G_MAX
    mid = np.full((4, 64), 2688.0 * 2.0 ** -64, np.float32)
    assert O.dynamic_scale(mid)[1] == O.G_MIN          # the boundary itself is kept


# --------------------------------------------------------------------------
# Scale-factor swizzle
# --------------------------------------------------------------------------

@pytest.mark.parametrize("rows,k", [(128, 64), (129, 64), (300, 192), (4608, 3072), (1, 16), (5, 48)])
def test_sf_swizzle_is_a_bijection_onto_the_padded_buffer(rows, k):
    rp, cp = O.sf_padded_shape(rows, k)
    r, c = np.meshgrid(np.arange(rp), np.arange(cp), indexing="ij")
    off = O.sf_offset(r, c, cp).reshape(-1)
    assert np.array_equal(np.sort(off), np.arange(rp * cp))


@pytest.mark.parametrize("rows,k", [(128, 64), (256, 512), (384, 3072)])
def test_sf_swizzle_equals_atom_reshape_construction(rows, k):
    # Independent construction: view the padded [R, C] scale matrix as
    # [R/128][4][32][C/4][4] (row = 128*rb + 32*q + l, col = 4*cb + j) and
    # order it [rb][cb][l][q][j]: 512-byte atoms of 32 lines x (4 rows x 4 scales).
    rng = np.random.default_rng(11)
    sf = rng.integers(0, 256, (rows, k // 16)).astype(np.uint8)
    rp, cp = O.sf_padded_shape(rows, k)
    pad = np.zeros((rp, cp), np.uint8)
    pad[:rows, :k // 16] = sf
    want = pad.reshape(rp // 128, 4, 32, cp // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    assert np.array_equal(O.swizzle_sf(sf), want)
    assert np.array_equal(O.unswizzle_sf(want, rows, k), sf)


def test_sf_swizzle_padding_is_zero():
    sf = np.full((130, 5), 0xAB, np.uint8)  # 130 rows, 5 scale columns (K=80)
    out = O.swizzle_sf(sf)
    rp, cp = O.sf_padded_shape(130, 80)
    assert out.size == rp * cp == 256 * 8
    assert int(np.count_nonzero(out)) == 130 * 5
