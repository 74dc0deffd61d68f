"""Plain CPU oracle for the NVFP4 W4A4 linear-layer hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
anything in this package.  The library's product path never calls it, and this
package imports nothing from the CUDA library (``nvfp4_block_scaled_12_b200``).
The two sides share only the seeded input generators of ``synth``.

What it computes, and where the definition comes from
------------------------------------------------------
* NVFP4 element = 4-bit float E2M1, grouped in 16-element blocks that share one
  higher-precision scale (microscaling).  -- "NVIDIA FP4 format, diffusion
  1.68x" news page (zubnet, Hindi), paragraph 1.
* A ModelOpt NVFP4 linear layer stores packed E2M1 ``weight`` (two values per
  byte), E4M3 block scales ``weight_scale``, a per-tensor fp32
  ``weight_scale_2`` and a calibrated fp32 activation scale ``input_scale``.
  -- "BFL (fp8r / nvfp4)" diffusers quantization doc (Korean), ``nvfp4`` bullet.
* On Blackwell the layer runs as runtime activation quantization
  (``nvfp4_quantize``) followed by an NVFP4 x NVFP4 GEMM (``mm_fp4``).
  -- same doc, section "Kernels", table row ``nvfp4``.

The formulas the pages leave open are fixed as follows (the plainest reading;
every one is listed with its justification in the design notes):

* per-tensor (global) scale, decode convention: ``g = amax / (6 * 448)``;
* block scale ``s = E4M3(amax_block / (6 * g))``, RNE, saturating at 448;
* element code ``q = E2M1(x / (s * g))``, RNE, saturating at +-6; the division
  is taken as a multiply by the fp32 reciprocal ``r = 1 / (s * g)``;
* dequantized value ``x_hat = e2m1(q) * e4m3(s) * g``;
* GEMM ``y = (g_x * g_w) * sum_k a_hat * b_hat + bias`` (fp64 here).

Floating-point steps of the quantizer are single IEEE fp32 operations
(round-to-nearest-even) in the order written: numpy float32 ufuncs are
correctly rounded and never contract into FMAs, so each line below is exactly
one rounding.  Everything else (decode, dequantization, GEMM, GELU) is fp64.

Pins (the tests that tie each function to something other than itself):
  e2m1_decode / e2m1_encode      tests/test_oracle_formats.py (ml_dtypes
                                 float4_e2m1fn over all bf16 values, tie table)
  e4m3_decode / e4m3_encode_sat  tests/test_oracle_formats.py (ml_dtypes
                                 float8_e4m3fn after clamping, all 256 bytes)
  round_to_bf16                  tests/test_oracle_formats.py (torch fp32->bf16)
  quantize_nvfp4                 tests/test_oracle_quant.py (round trip of
                                 representable blocks, zero blocks, saturation,
                                 brute-force nearest code)
  dynamic_scale / quantize_dynamic
                                 tests/test_oracle_quant.py (power-of-two
                                 closed forms, the tensor's largest element
                                 lands on code +-6 under scale 448, all-zero
                                 tensor, both clamps)
  swizzle_sf / sf_offset         tests/test_oracle_quant.py (bijection, and an
                                 independent reshape/transpose construction)
  gemm_ref / dequantize          tests/test_oracle_gemm.py (closed form,
                                 triple-loop brute force)
  gelu_tanh                      tests/test_oracle_gemm.py (torch gelu 'tanh'
                                 in fp64, odd-part identity)
  dequantize_to_bf16 / linear_w4a16_ref
                                 tests/test_oracle_gemm.py (power-of-two
                                 scales against ml_dtypes decoding, the
                                 rounding bound, torch's bf16 conversion)
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# Element and scale formats
# ----------------------------------------------------------------------------

#: Magnitudes of the eight non-negative E2M1 codes 0..7 (1 sign bit, 2 exponent
#: bits with bias 1, 1 mantissa bit; no inf/NaN).
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0
#: Largest finite E4M3 ("fn" variant: no inf, 0x7F/0xFF are NaN).
E4M3_MAX = 448.0
#: Elements per NVFP4 scale block.
BLOCK = 16
#: 6 * 448: the product of the two format maxima, the denominator of the
#: per-tensor scale.
GLOBAL_DENOM = np.float32(6.0 * 448.0)


def e2m1_decode(codes) -> np.ndarray:
    """Value of each 4-bit code ``[s e1 e0 m]`` (bit 3 = sign), as float64."""
    c = np.asarray(codes, dtype=np.uint8) & 0xF
    mag = E2M1_GRID[c & 0x7]
    return np.where(c & 0x8, -mag, mag)


def e2m1_encode(v) -> np.ndarray:
    """Round each value to the nearest E2M1 code, ties to the even code.

    Magnitudes above 6 saturate to 6 (code 7).  The sign bit is the sign of
    the input, so negative values that round to zero give code 0x8 (-0).
    Input must be finite or +-inf (NaN is outside the contract).
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    hi = np.searchsorted(E2M1_GRID, a, side="left")  # first grid point >= a
    hi = np.minimum(hi, 7)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - E2M1_GRID[lo]
    d_hi = E2M1_GRID[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E2M1_MAX, 7, code)  # saturation (and exactly 6)
    sign = np.signbit(v)
    return (code | np.where(sign, 8, 0)).astype(np.uint8)


def _e4m3_table() -> np.ndarray:
    """Values of the non-negative E4M3 bytes 0x00..0x7E (0x7F is NaN)."""
    out = np.empty(127, dtype=np.float64)
    for b in range(127):
        e, m = b >> 3, b & 7
        if e == 0:
            out[b] = m * 2.0 ** -9  # subnormal: m/8 * 2^(1-7)
        else:
            out[b] = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


E4M3_POS = _e4m3_table()


def e4m3_decode(b) -> np.ndarray:
    """Value of each E4M3 byte as float64 (NaN for 0x7F and 0xFF)."""
    b = np.asarray(b, dtype=np.uint8)
    mag = np.where((b & 0x7F) == 0x7F, np.nan, E4M3_POS[np.minimum(b & 0x7F, 126)])
    return np.where(b & 0x80, -mag, mag)


def e4m3_encode_sat(t) -> np.ndarray:
    """Encode non-negative values as E4M3: nearest value, ties to even byte,
    saturating to 448 (byte 0x7E); never emits NaN.  +inf saturates too."""
    t = np.asarray(t, dtype=np.float64)
    if np.any(t < 0) or np.any(np.isnan(t)):
        raise ValueError("e4m3_encode_sat takes non-negative, non-NaN values")
    hi = np.searchsorted(E4M3_POS, t, side="left")
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo = t - E4M3_POS[lo]
    d_hi = E4M3_POS[hi] - t
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(t >= E4M3_MAX, 126, code)
    return code.astype(np.uint8)


def round_to_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as
    float64.  Finite inputs only; results past the bf16 range become inf."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)  # v = m * 2^e, 0.5 <= |m| < 1
    # bf16 keeps 8 significant bits; below 2^-126 the step is fixed at 2^-133.
    e = np.maximum(e, -125)
    step_exp = e - 8
    q = np.rint(np.ldexp(v, -step_exp))  # exact scaling, then RNE
    out = np.ldexp(q, step_exp)
    return np.where(np.abs(out) > 3.3895313892515355e38, np.copysign(np.inf, v), out)


# ----------------------------------------------------------------------------
# Per-tensor scale (calibration)
# ----------------------------------------------------------------------------

def global_scale(amax) -> np.float32:
    """Per-tensor decode scale ``g = amax / (6 * 448)``, one fp32 division.

    For weights this is ModelOpt's ``weight_scale_2``; for activations it is
    the calibrated ``input_scale``.  (BFL doc, ``nvfp4`` bullet.)
    """
    return np.float32(np.float32(amax) / GLOBAL_DENOM)


def tensor_amax(x) -> np.float32:
    """Largest magnitude of a float tensor (exact)."""
    return np.float32(np.max(np.abs(np.asarray(x, dtype=np.float32))))


#: Range of per-tensor scales the quantizer accepts (the library's contract).
G_MIN = np.float32(2.0 ** -64)
G_MAX = np.float32(2.0 ** 64)


def dynamic_scale(x):
    """Per-tensor scale measured on the activation itself, for a layer that
    has no calibrated ``input_scale`` (the BFL doc's ``nvfp4`` bullet makes the
    calibrated scale the default; measuring it per call is the variant).

    Returns ``(amax, g)``: ``amax = max |x|`` and ``g = amax / (6 * 448)``
    (one fp32 division, as for a calibrated scale), clamped into
    ``[G_MIN, G_MAX]``; ``g = 0`` when the tensor is all zeros.
    """
    amax = tensor_amax(x)
    if amax == 0:
        return amax, np.float32(0.0)
    g = global_scale(amax)
    return amax, np.float32(min(max(g, G_MIN), G_MAX))


def quantize_dynamic(x):
    """``quantize_nvfp4`` with the scale from ``dynamic_scale``; an all-zero
    tensor (``g = 0``) gives all-zero codes and scales.
    Returns ``(codes, sf, amax, g)``."""
    x = np.asarray(x, dtype=np.float32)
    amax, g = dynamic_scale(x)
    if g == 0:
        rows, K = x.shape
        return np.zeros((rows, K // 2), np.uint8), np.zeros((rows, K // BLOCK), np.uint8), amax, g
    codes, sf = quantize_nvfp4(x, g)
    return codes, sf, amax, g


# ----------------------------------------------------------------------------
# Block quantizer (runtime activation quantize; also the offline weight quantize)
# ----------------------------------------------------------------------------

def quantize_nvfp4(x, g):
    """Quantize ``x`` [rows, K] (values exactly representable in fp32, e.g. bf16
    inputs) with per-tensor decode scale ``g``.

    Returns ``(codes, sf)``: ``codes`` uint8 [rows, K/2], element 2j in the low
    nibble of byte j and element 2j+1 in the high nibble; ``sf`` uint8
    [rows, K/16], the E4M3 block scales in plain row-major order (ModelOpt's
    ``weight_scale`` layout).

    Steps for each 16-element block along K (each line one fp32 rounding):
      amax = max |x_i|
      d6   = 6 * g
      s    = E4M3_sat(amax / d6)                 (block scale byte)
      if s decodes to 0 (all-zero block or scale underflow): all codes 0x0
      else r = 1 / (e4m3(s) * g);  q_i = E2M1(x_i * r)
    """
    x = np.asarray(x, dtype=np.float32)
    rows, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    g = np.float32(g)
    blocks = x.reshape(rows, K // BLOCK, BLOCK)
    amax = np.max(np.abs(blocks), axis=2)                  # exact
    d6 = np.float32(6.0) * g                                # fp32 multiply
    t = (amax / d6).astype(np.float32)                      # fp32 divide
    s = e4m3_encode_sat(t.astype(np.float64))
    s_val = e4m3_decode(s).astype(np.float32)               # exact
    sg = (s_val * g).astype(np.float32)                     # fp32 multiply
    zero_block = s == 0
    with np.errstate(divide="ignore"):
        r = (np.float32(1.0) / np.where(zero_block, np.float32(1.0), sg)).astype(np.float32)
    xr = (blocks * r[:, :, None]).astype(np.float32)        # fp32 multiply
    q = e2m1_encode(xr.astype(np.float64))
    q = np.where(zero_block[:, :, None], np.uint8(0), q).reshape(rows, K)
    return pack_codes(q), s


def pack_codes(q) -> np.ndarray:
    """Pack 4-bit codes [rows, K] two per byte: even element in the low nibble."""
    q = np.asarray(q, dtype=np.uint8)
    return (q[:, 0::2] & 0xF) | ((q[:, 1::2] & 0xF) << 4)


def unpack_codes(packed) -> np.ndarray:
    """Inverse of :func:`pack_codes`."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def dequantize(codes, sf, g) -> np.ndarray:
    """``x_hat = e2m1(q) * e4m3(s) * g`` in float64, [rows, K]."""
    q = e2m1_decode(unpack_codes(codes))
    rows, K = q.shape
    s = e4m3_decode(sf).reshape(rows, K // BLOCK, 1)
    return (q.reshape(rows, K // BLOCK, BLOCK) * s).reshape(rows, K) * np.float64(np.float32(g))


# ----------------------------------------------------------------------------
# Tensor-core scale-factor layout
# ----------------------------------------------------------------------------

def sf_padded_shape(rows: int, k: int):
    """(rows, scale columns) of the swizzled buffer: rows padded to 128, scale
    columns (k/16) padded to 4."""
    cols = k // BLOCK
    return (rows + 127) // 128 * 128, (cols + 3) // 4 * 4


def sf_offset(r, c, cols_padded):
    """Byte offset of logical scale (row r, scale column c) in the swizzled
    buffer.  The buffer is a row-major grid of 512-byte atoms, each covering
    128 rows x 4 scale columns; inside an atom, row r sits at 16-byte line
    r % 32, 4-byte slot (r % 128) // 32, byte c % 4."""
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    atom = (r // 128) * (cols_padded // 4) + c // 4
    return atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)


def swizzle_sf(sf_linear) -> np.ndarray:
    """Scatter row-major scales [rows, k/16] into the swizzled, zero-padded
    1-D buffer the block-scaled MMA reads."""
    sf_linear = np.asarray(sf_linear, dtype=np.uint8)
    rows, cols = sf_linear.shape
    rp, cp = sf_padded_shape(rows, cols * BLOCK)
    out = np.zeros(rp * cp, dtype=np.uint8)
    r, c = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    out[sf_offset(r, c, cp)] = sf_linear
    return out


def unswizzle_sf(sf_swz, rows: int, k: int) -> np.ndarray:
    """Gather the logical [rows, k/16] scales back out of a swizzled buffer."""
    cols = k // BLOCK
    _, cp = sf_padded_shape(rows, k)
    r, c = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    return np.asarray(sf_swz, dtype=np.uint8)[sf_offset(r, c, cp)]


# ----------------------------------------------------------------------------
# GEMM with dequant epilogue
# ----------------------------------------------------------------------------

def dequantize_to_bf16(codes, sf, g) -> np.ndarray:
    """Weights dequantized to the bf16 compute dtype, as the W4A16 path does on
    every forward ("BFL (fp8r / nvfp4)" doc, section "Kernels", last
    paragraph): ``v = fl32(fl32(e2m1(q) * e4m3(s)) * g)`` -- the first product
    is exact in fp32 -- then rounded to bf16 (RNE).  Returns float32 values
    that are exactly bf16, shape [rows, K]."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows = codes.shape[0]
    q = e2m1_decode(unpack_codes(codes)).astype(np.float32)            # exact
    s = e4m3_decode(np.asarray(sf, np.uint8)).astype(np.float32)       # exact
    prod = (q.reshape(rows, -1, BLOCK) * s[:, :, None]).astype(np.float32)   # exact (<= 3 x 4 significant bits)
    v = (prod * np.float32(g)).astype(np.float32).reshape(rows, -1)    # one fp32 rounding
    return round_to_bf16(v.astype(np.float64)).astype(np.float32)


def linear_w4a16_ref(x_bf16, w_codes, w_sf, g_w, bias=None) -> np.ndarray:
    """``y = x @ w_bf16^T + bias`` in float64 with ``w_bf16 =
    dequantize_to_bf16(w)``: the regular linear the W4A16 path runs (the
    activations stay bf16)."""
    w = dequantize_to_bf16(w_codes, w_sf, g_w).astype(np.float64)
    y = np.asarray(x_bf16, dtype=np.float64) @ w.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def gemm_ref(a_codes, a_sf, g_a, b_codes, b_sf, g_b, bias=None) -> np.ndarray:
    """``y[m, n] = (g_a * g_b) * sum_k a_hat[m, k] * b_hat[n, k] + bias[n]`` in
    float64, where ``a_hat = e2m1 * e4m3`` (no global scale).  A is [M, K]
    (activations), B is [N, K] (weight in PyTorch ``[out, in]`` order)."""
    a_hat = dequantize(a_codes, a_sf, 1.0)
    b_hat = dequantize(b_codes, b_sf, 1.0)
    alpha = np.float64(np.float32(g_a)) * np.float64(np.float32(g_b))
    y = alpha * (a_hat @ b_hat.T)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def gemm_tolerance(a_codes, a_sf, g_a, b_codes, b_sf, g_b, y_ref) -> np.ndarray:
    """Elementwise bound ``2e-3 * |a_m|_2 * |b_n|_2 + 1e-2 * |y_ref|`` where
    a_m, b_n are the dequantized (globally scaled) operand rows."""
    a_n = np.linalg.norm(dequantize(a_codes, a_sf, g_a), axis=1)
    b_n = np.linalg.norm(dequantize(b_codes, b_sf, g_b), axis=1)
    return 2e-3 * a_n[:, None] * b_n[None, :] + 1e-2 * np.abs(y_ref)


# ----------------------------------------------------------------------------
# Fused epilogue: optional GELU-tanh, then the next layer's quantize
# ----------------------------------------------------------------------------

def gelu_tanh(v) -> np.ndarray:
    """GELU, tanh form: 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), fp64."""
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (v + 0.044715 * v ** 3)))


ACT_NONE = 0
ACT_GELU_TANH = 1


def epilogue_ref(y, ranges):
    """Apply the fused epilogue to an fp64 GEMM result ``y`` [M, N].

    ``ranges`` is a list of ``(begin, end, act)``: columns [begin, end) are
    rounded to bf16, passed through ``act`` (computed in fp64 on the bf16
    value) and rounded to bf16 again.  Returns the bf16-valued float64 array
    of the concatenated ranges, in the order given.
    """
    parts = []
    for begin, end, act in ranges:
        v = round_to_bf16(y[:, begin:end])
        if act == ACT_GELU_TANH:
            v = round_to_bf16(gelu_tanh(v))
        parts.append(v)
    return np.concatenate(parts, axis=1)
