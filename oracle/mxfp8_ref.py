"""Plain CPU oracle for the MXFP8 variant of the linear-layer hot path.

TEST INFRASTRUCTURE ONLY (same rules as ``oracle/nvfp4_ref.py``): only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use it,
and it imports nothing from the CUDA library.

What it computes, and where the definition comes from
------------------------------------------------------
* MXFP8 = 8-bit E4M3 (or E5M2) elements grouped in 32-element blocks that
  share one scale, following the Open Compute Project microscaling standard;
  NVFP4's sibling for the same Blackwell kernels.  -- "NVIDIA FP4 format,
  diffusion 1.68x" news page (zubnet, Hindi), paragraph 1 (and its 1.26x
  figure for MXFP8).
* The OCP microscaling standard fixes the shared scale as a power of two
  stored as E8M0 (an 8-bit biased exponent, bias 127, 0xFF = NaN) and the
  conversion as: ``X = 2^(floor(log2(max_i |V_i|)) - emax)`` with ``emax``
  the exponent of the element format's largest normal (8 for E4M3: 448 =
  1.75 * 2^8), then ``P_i = V_i / X`` rounded to the element format with
  normal values above its largest normal clamped to it.  This is the plainest
  reading of "MXFP8 follows the OCP standard"; the pages print no formula.

Choices the standard leaves to the implementation (listed in the design
notes with the reasons):
* an all-zero block gets scale byte 0 (2^-127) and all-zero elements (their
  sign kept, as the element conversion keeps it);
* the shared exponent is clamped into E8M0's range [-127, 127];
* ``V_i / X`` is the fp32 product ``V_i * 2^-s`` (exact unless it falls
  below fp32's normal range), and the E4M3 rounding is to nearest, ties to
  even, saturating at +-448;
* the E4M3 element variant (the pages name E4M3/E5M2; E4M3 is the one the
  activations and weights use here).

Pins: tests/test_oracle_mxfp8.py (E8M0 decode vs ml_dtypes float8_e8m0fnu on
all bytes; element encode vs ml_dtypes float8_e4m3fn after clamping; blocks
of representable values round-trip; the block maximum lands in [256, 448];
brute-force nearest element; zero and saturating blocks; brute-force GEMM).
"""
from __future__ import annotations

import numpy as np

from .nvfp4_ref import E4M3_MAX, e4m3_decode, e4m3_encode_sat, sf_offset, sf_padded_shape

#: Elements per MXFP8 scale block.
MX_BLOCK = 32
#: Exponent of E4M3's largest normal value (448 = 1.75 * 2^8).
E4M3_EMAX = 8


def e8m0_decode(b) -> np.ndarray:
    """Value of each E8M0 byte, 2^(b - 127), as float64 (NaN for 0xFF)."""
    b = np.asarray(b, dtype=np.int64)
    return np.where(b == 255, np.nan, np.ldexp(1.0, b - 127))


def e4m3_encode_signed(v) -> np.ndarray:
    """E4M3 byte of each value: sign bit from the value's sign (-0 included),
    magnitude rounded to nearest, ties to even, saturating at 448."""
    v = np.asarray(v, dtype=np.float64)
    mag = e4m3_encode_sat(np.abs(v))
    neg = np.signbit(v)
    return (mag | np.where(neg, 0x80, 0)).astype(np.uint8)


def block_exponent(amax) -> np.ndarray:
    """floor(log2(a)) of positive finite floats, exact (frexp: a = m * 2^e with
    m in [0.5, 1), so floor(log2 a) = e - 1), subnormals included."""
    _, e = np.frexp(np.asarray(amax, dtype=np.float64))
    return e.astype(np.int64) - 1


def quantize_mxfp8(x):
    """Quantize ``x`` [rows, K] (fp32-exact values, e.g. bf16 inputs) to MXFP8.

    Returns ``(codes, sf)``: ``codes`` uint8 [rows, K], one E4M3 byte per
    element; ``sf`` uint8 [rows, K/32], the E8M0 block scales row-major.

    For each 32-element block along K:
      amax = max |x_i|
      amax == 0:  scale byte 0, codes = E4M3(x_i) (zeros, sign kept)
      else        s = clamp(floor(log2 amax) - 8, -127, 127);  scale byte s + 127
                  code_i = E4M3_sat(fl(x_i * 2^-s))
    """
    x = np.asarray(x, dtype=np.float32)
    rows, K = x.shape
    if K % MX_BLOCK:
        raise ValueError("K must be a multiple of 32")
    blocks = x.reshape(rows, K // MX_BLOCK, MX_BLOCK)
    amax = np.max(np.abs(blocks), axis=2).astype(np.float64)
    e = np.where(amax > 0, block_exponent(np.where(amax > 0, amax, 1.0)), 0)
    s = np.clip(e - E4M3_EMAX, -127, 127)
    s = np.where(amax > 0, s, -127)
    inv = np.ldexp(np.float32(1.0), -s).astype(np.float32)          # 2^-s, exact in fp32
    scaled = (blocks * inv[:, :, None]).astype(np.float32)           # one fp32 multiply
    codes = e4m3_encode_signed(scaled.astype(np.float64)).reshape(rows, K)
    return codes, (s + 127).astype(np.uint8)


def dequantize_mxfp8(codes, sf) -> np.ndarray:
    """x_hat = e4m3(code) * 2^(scale - 127), float64 [rows, K]."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows, K = codes.shape
    vals = e4m3_decode(codes).reshape(rows, K // MX_BLOCK, MX_BLOCK)
    return (vals * e8m0_decode(sf)[:, :, None]).reshape(rows, K)


def sf_bytes_mxfp8(rows: int, k: int) -> int:
    """Size of the swizzled MXFP8 scale buffer: the NVFP4 atom layout with one
    scale column per 32 elements (rows padded to 128, columns to 4)."""
    rp = (rows + 127) // 128 * 128
    cp = (k // MX_BLOCK + 3) // 4 * 4
    return rp * cp


def swizzle_sf_mxfp8(sf_linear) -> np.ndarray:
    """Scatter row-major E8M0 scales [rows, K/32] into the swizzled,
    zero-padded buffer (512-byte atoms of 128 rows x 4 scale columns, the
    layout the block-scaled MMA reads)."""
    sf_linear = np.asarray(sf_linear, dtype=np.uint8)
    rows, cols = sf_linear.shape
    out = np.zeros(sf_bytes_mxfp8(rows, cols * MX_BLOCK), dtype=np.uint8)
    cp = (cols + 3) // 4 * 4
    r, c = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    out[sf_offset(r, c, cp)] = sf_linear
    return out


def unswizzle_sf_mxfp8(sf_swz, rows: int, k: int) -> np.ndarray:
    """Gather the logical [rows, K/32] scales back out of a swizzled buffer."""
    cols = k // MX_BLOCK
    cp = (cols + 3) // 4 * 4
    r, c = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    return np.asarray(sf_swz, dtype=np.uint8)[sf_offset(r, c, cp)]


def gemm_ref_mxfp8(a_codes, a_sf, b_codes, b_sf, alpha=1.0, bias=None) -> np.ndarray:
    """``y = alpha * a_hat @ b_hat^T + bias`` in float64 (A [M,K] activations,
    B [N,K] weights in PyTorch ``[out, in]`` order)."""
    y = np.float64(np.float32(alpha)) * (dequantize_mxfp8(a_codes, a_sf) @ dequantize_mxfp8(b_codes, b_sf).T)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def gemm_tolerance_mxfp8(a_codes, a_sf, b_codes, b_sf, y_ref, alpha=1.0) -> np.ndarray:
    """Elementwise bound 2e-3 * |alpha| * ||a_hat_m|| * ||b_hat_n|| + 1e-2 * |y_ref|
    (the NVFP4 GEMM's tolerance: fp32 accumulation error plus bf16 output
    rounding)."""
    na = np.linalg.norm(dequantize_mxfp8(a_codes, a_sf), axis=1)
    nb = np.linalg.norm(dequantize_mxfp8(b_codes, b_sf), axis=1)
    return 2e-3 * abs(float(np.float32(alpha))) * np.outer(na, nb) + 1e-2 * np.abs(y_ref)


__all__ = ["MX_BLOCK", "E4M3_EMAX", "e8m0_decode", "e4m3_encode_signed", "block_exponent", "quantize_mxfp8",
           "dequantize_mxfp8", "sf_bytes_mxfp8", "swizzle_sf_mxfp8", "unswizzle_sf_mxfp8", "gemm_ref_mxfp8",
           "gemm_tolerance_mxfp8", "sf_padded_shape", "E4M3_MAX"]
