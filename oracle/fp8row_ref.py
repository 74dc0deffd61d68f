"""Plain CPU oracle for the row-wise FP8 (W8A8) variant.

TEST INFRASTRUCTURE ONLY (same rules as ``oracle/nvfp4_ref.py``).

What it computes, and where the definition comes from
------------------------------------------------------
* ``fp8r`` = row-wise FP8: each quantized linear layer stores an E4M3
  ``weight`` and a per-row fp32 ``weight_scale``; activations are quantized
  to E4M3 row by row at run time; the GEMM applies the row scales
  (``torch._scaled_mm`` with row-wise scales).  -- "BFL (fp8r / nvfp4)"
  diffusers doc (Korean), ``fp8r`` bullet and section "Kernels", row ``fp8r``.

The page gives no formula for the row scale.  Plainest reading (listed in
the design notes): absmax scaling onto E4M3's largest value,
* ``s = fl(amax_row / 448)`` (one fp32 division), ``q = E4M3_sat(fl(x / s))``
  (one fp32 division, round to nearest even, saturating at +-448);
* a row of zeros gets ``s = 0`` and zero codes (sign kept);
* ``y[m, n] = s_x[m] * s_w[n] * sum_k e4m3(q_x[m,k]) e4m3(q_w[n,k]) + bias[n]``.

Pins: tests/test_oracle_fp8row.py (closed forms, the row maximum lands on
code +-448, zero rows, brute-force nearest code, ml_dtypes encoding,
triple-loop GEMM).
"""
from __future__ import annotations

import numpy as np

from .mxfp8_ref import e4m3_encode_signed
from .nvfp4_ref import e4m3_decode

#: Largest finite E4M3 value, the target of a row's maximum.
FP8_MAX = np.float32(448.0)


def quantize_fp8_rowwise(x):
    """``x`` [rows, K] (fp32-exact values) -> ``(codes uint8 [rows, K],
    scale float32 [rows])`` with the steps in the module docstring."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1)
    s = (amax / FP8_MAX).astype(np.float32)                    # fp32 divide
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (x / np.where(s > 0, s, np.float32(1.0))[:, None]).astype(np.float32)  # fp32 divide
    t = np.where((s > 0)[:, None], t, x)                       # zero row: codes of +-0
    return e4m3_encode_signed(t.astype(np.float64)), s


def dequantize_fp8_rowwise(codes, scale) -> np.ndarray:
    """x_hat = e4m3(code) * s_row, float64."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, None]


def gemm_ref_fp8row(a_codes, a_scale, b_codes, b_scale, bias=None) -> np.ndarray:
    """``y = s_a[m] s_b[n] sum_k a_q[m,k] b_q[n,k] + bias[n]`` in float64 (B is
    the weight [N, K] in PyTorch ``[out, in]`` order)."""
    acc = e4m3_decode(a_codes) @ e4m3_decode(b_codes).T
    y = np.asarray(a_scale, np.float64)[:, None] * np.asarray(b_scale, np.float64)[None, :] * acc
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def gemm_tolerance_fp8row(a_codes, a_scale, b_codes, b_scale, y_ref) -> np.ndarray:
    """``2e-3 * |a_hat_m| * |b_hat_n| + 1e-2 * |y_ref|`` (as for NVFP4)."""
    na = np.linalg.norm(dequantize_fp8_rowwise(a_codes, a_scale), axis=1)
    nb = np.linalg.norm(dequantize_fp8_rowwise(b_codes, b_scale), axis=1)
    return 2e-3 * np.outer(na, nb) + 1e-2 * np.abs(y_ref)


__all__ = ["FP8_MAX", "quantize_fp8_rowwise", "dequantize_fp8_rowwise", "gemm_ref_fp8row", "gemm_tolerance_fp8row"]
