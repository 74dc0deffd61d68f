"""Pins for the oracle's element and scale formats (CPU only).

E2M1 (4-bit element) and E4M3 (block scale) are the formats the NVFP4 pages
name ("NVIDIA FP4 format" news page, paragraph 1; "BFL (fp8r / nvfp4)" doc,
``nvfp4`` bullet).  The oracle's codecs are checked against an independent
library (ml_dtypes) and against the textbook round-to-nearest-even tie table.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def all_bf16_as_f32():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    return v[~np.isnan(v)]


def test_e2m1_decode_matches_ml_dtypes_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(F4).astype(np.float64)
    got = O.e2m1_decode(codes)
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))
    assert sorted(set(np.abs(got).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_encode_matches_ml_dtypes_every_bf16_value():
    v = all_bf16_as_f32()
    ref = v.astype(F4).view(np.uint8)
    got = O.e2m1_encode(v)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (v[bad[:8]], got[bad[:8]], ref[bad[:8]])


@pytest.mark.parametrize("value,code", [
    (0.25, 0x0), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4), (3.5, 0x6), (5.0, 0x6),
    (0.2499, 0x0), (0.2501, 0x1), (5.0001, 0x7), (6.0, 0x7), (7.0, 0x7), (1e30, 0x7),
    (float("inf"), 0x7), (-0.1, 0x8), (-0.0, 0x8), (-3.5, 0xE), (-100.0, 0xF), (0.0, 0x0),
])
def test_e2m1_tie_table(value, code):
    # Ties between adjacent grid points go to the code with an even mantissa
    # bit; beyond 6 the format saturates; the sign bit follows the input.
    assert int(O.e2m1_encode(np.float32(value))) == code


def test_e2m1_every_code_round_trips():
    codes = np.arange(16, dtype=np.uint8)
    back = O.e2m1_encode(O.e2m1_decode(codes))
    assert np.array_equal(back, codes)


def test_e4m3_decode_matches_ml_dtypes_all_bytes():
    b = np.arange(256, dtype=np.uint8)
    ref = b.view(F8).astype(np.float64)
    got = O.e4m3_decode(b)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert O.e4m3_decode(np.uint8(0x7E)) == 448.0
    assert O.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9


def _e4m3_sweep():
    pos = O.E4M3_POS
    mids = (pos[1:] + pos[:-1]) / 2  # exact ties
    f = np.concatenate([pos, mids]).astype(np.float32)
    up = np.nextafter(f, np.float32(np.inf))
    dn = np.nextafter(f, np.float32(0))
    rng = np.random.default_rng(123)
    logu = np.exp2(rng.uniform(-14, 9.5, 200_000)).astype(np.float32)
    extra = np.array([0, 448, 460, 463.99, 464, 464.01, 479.9, 480, 1e6, np.inf], np.float32)
    return np.concatenate([f, up, dn, logu, extra])


def test_e4m3_encode_matches_ml_dtypes_after_clamp():
    t = _e4m3_sweep()
    # ml_dtypes' cast is round-to-nearest-even but not saturating (>= 464 gives
    # NaN), so clamp to 448 first: saturation is then the only difference.
    ref = np.minimum(t, np.float32(448)).astype(F8).view(np.uint8)
    got = O.e4m3_encode_sat(t)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (t[bad[:8]], got[bad[:8]], ref[bad[:8]])


def test_e4m3_encode_equals_brute_force_nearest():
    # Independent of searchsorted: scan all 127 non-negative finite bytes.
    t = _e4m3_sweep()[::37]
    vals = np.array([float(np.uint8(b).view(F8)) for b in range(127)])
    for x in t:
        xv = min(float(x), 448.0)
        d = np.abs(vals - xv)
        best = np.flatnonzero(d == d.min())
        want = best[0] if best.size == 1 else best[best % 2 == 0][0]
        assert int(O.e4m3_encode_sat(np.float32(x))) == want, x


def test_e4m3_saturates_and_never_emits_nan():
    t = np.array([448.0, 464.0, 480.0, 1e30, np.inf], np.float32)
    assert np.all(O.e4m3_encode_sat(t) == 0x7E)
    assert np.all(O.e4m3_encode_sat(O.E4M3_POS) == np.arange(127))


def test_round_to_bf16_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(7)
    f = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32) * np.float32(1e3),
        np.exp2(rng.uniform(-140, 127, 100_000)).astype(np.float32),
        # exact ties halfway between adjacent bf16 values, both parities
        ((np.arange(1, 4000, dtype=np.uint32) << 15) | 0x3F800000).view(np.float32),
    ])
    f = np.concatenate([f, -f])
    ref = torch.from_numpy(f).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_to_bf16(f.astype(np.float64))
    assert np.array_equal(got, ref)


def test_code_packing_is_a_little_endian_stream_of_4_bit_fields():
    # Two E2M1 codes per byte ("BFL (fp8r / nvfp4)" doc, nvfp4 bullet), the
    # even element in the low nibble: the row's codes laid end to end as
    # 4-bit little-endian fields, element 0 first, and cut into bytes.
    # Built here from numpy's bit packing, not from the oracle's shifts.
    rng = np.random.default_rng(7)
    q = rng.integers(0, 16, (5, 64)).astype(np.uint8)
    bits = ((q[:, :, None] >> np.arange(4, dtype=np.uint8)) & 1).reshape(5, 64 * 4)
    want = np.packbits(bits, axis=1, bitorder="little")
    got = O.pack_codes(q)
    assert got.shape == (5, 32) and np.array_equal(got, want)
    assert np.array_equal(O.unpack_codes(got), q)
    # and every byte is the packing of exactly one code pair
    b = np.arange(256, dtype=np.uint8).reshape(1, 256)
    assert np.array_equal(O.pack_codes(O.unpack_codes(b)), b)
    assert O.pack_codes(np.array([[0x1, 0x2]], np.uint8))[0, 0] == 0x21
