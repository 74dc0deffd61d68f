"""GPU parity of the W4A16 path: NVFP4 weights dequantized to bf16 by this
library (bit-exact against the oracle), then a regular bf16 linear on the
unquantized activations ("BFL (fp8r / nvfp4)" doc, section "Kernels", last
paragraph).  The linear is a library GEMM; its result is checked within the
GEMM tolerance of the oracle's fp64 linear of the same bf16 operands.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from tests.gpu_helpers import assert_bytes_equal, assert_within_tol, f32, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    require_gpu()
    import nvfp4_block_scaled_12_b200 as F
    return F


def _bf16_bytes(t):
    return t.contiguous().view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("rows,k,g", [(1, 64, 1.0), (7, 192, 0.0123), (300, 4160, 3.7e-4), (128, 256, 2.0 ** 20)])
def test_dequantize_bit_exact(F, rows, k, g):
    rng = np.random.default_rng(rows + k)
    codes = rng.integers(0, 256, (rows, k // 2)).astype(np.uint8)
    sf = rng.integers(0, 127, (rows, k // 16)).astype(np.uint8)
    t = F.NVFP4Tensor(torch.from_numpy(codes).cuda(), torch.from_numpy(O.swizzle_sf(sf)).cuda(), g, rows, k)
    got = F.dequantize(t)
    torch.cuda.synchronize()
    want = torch.from_numpy(O.dequantize_to_bf16(codes, sf, g)).to(torch.bfloat16)
    assert_bytes_equal(_bf16_bytes(got), _bf16_bytes(want), f"dequantize {rows}x{k}")


def test_dequantize_the_weights_the_quantizer_wrote(F):
    wl = synth.MLP_UP
    w = wl.weight()[:512]
    g = float(O.global_scale(O.tensor_amax(f32(w))))
    wq = F.quantize(w.cuda(), g)
    got = F.dequantize(wq)
    codes, sf = O.quantize_nvfp4(f32(w), g)
    want = torch.from_numpy(O.dequantize_to_bf16(codes, sf, g)).to(torch.bfloat16)
    assert_bytes_equal(_bf16_bytes(got), _bf16_bytes(want), "weights")


@pytest.mark.parametrize("m", [1, 100, 512])
def test_w4a16_linear_matches_the_oracle(F, m):
    wl = synth.LinearWorkload(f"w4a16_m{m}", m, 3072, 768, seed=70 + m)
    x, w, bias = wl.activations(), wl.weight(), wl.bias_vec()
    g = float(O.global_scale(O.tensor_amax(f32(w))))
    wq = F.quantize(w.cuda(), g)
    y = F.linear_w4a16(x.cuda(), wq, bias.cuda()).float().cpu().numpy()
    codes, sf = O.quantize_nvfp4(f32(w), g)
    y_ref = O.linear_w4a16_ref(f32(x), codes, sf, g, f32(bias))
    wb = O.dequantize_to_bf16(codes, sf, g).astype(np.float64)
    tol = 2e-3 * np.outer(np.linalg.norm(f32(x).astype(np.float64), axis=1), np.linalg.norm(wb, axis=1)) \
        + 1e-2 * np.abs(y_ref)
    assert_within_tol(y, y_ref, tol, wl.name)


def test_no_kernel_reported_a_fault(F):
    F.nvfp4_check_fault()
