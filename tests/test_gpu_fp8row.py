"""GPU parity of the row-wise FP8 (W8A8) variant against the oracle: the
quantizer bit-exact (codes and fp32 row scales), the GEMM within the NVFP4
GEMM's tolerance and bit-exact where fp32 accumulation is exact.

Row-wise FP8: E4M3 weights with one fp32 scale per row, activations
quantized to E4M3 row by row at run time ("BFL (fp8r / nvfp4)" doc, ``fp8r``
bullet and section "Kernels").
"""
import numpy as np
import pytest
import torch

import synth
from oracle import fp8row_ref as R
from oracle import nvfp4_ref as N
from tests.gpu_helpers import assert_bytes_equal, assert_within_tol, f32, gpu_bytes, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    require_gpu()
    import nvfp4_block_scaled_12_b200 as F
    return F


def _check_quant(F, x_bf16, what, rows=None):
    q = F.quantize_fp8row(x_bf16.cuda())
    torch.cuda.synchronize()
    x = f32(x_bf16)
    sel = np.arange(x.shape[0]) if rows is None else rows
    codes, s = R.quantize_fp8_rowwise(x[sel])
    assert_bytes_equal(gpu_bytes(q.codes)[sel], codes, what + " codes")
    assert np.array_equal(q.scale.cpu().numpy()[sel], s), what + " scales"
    return q


def test_tiny(F):
    _check_quant(F, synth.TINY.activations(), "tiny")


@pytest.mark.parametrize("m,k", [(1, 64), (7, 192), (9, 320), (300, 4160), (33, 15360),
                                 (1, 1024), (9, 1024), (300, 2048), (17, 3072), (129, 4096), (5, 5120)])
def test_ragged_shapes(F, m, k):
    # K = 1024/2048/3072/4096 take the register-resident kernel, the rest the
    # two-pass one
    _check_quant(F, synth.activations_with_outlier_channels(m, k, seed=m + k), f"ragged {m}x{k}")


def test_special_rows(F):
    x = np.zeros((6, 256), np.float32)
    x[0, 7] = -0.0                                 # zero row
    x[1, :] = np.linspace(-1e30, 1e30, 256)
    x[2, :] = np.linspace(-1e-30, 1e-30, 256)      # tiny values
    x[3, :] = -np.logspace(-20, 20, 256)
    x[4, 5] = 3.0                                  # a single non-zero element
    x[5, :] = 2.0 ** -130                          # bf16 subnormals
    _check_quant(F, torch.from_numpy(x).to(torch.bfloat16), "special")


@pytest.mark.parametrize("k", [1024, 3072, 1088])
def test_special_rows_register_path(F, k):
    # row scales inside and outside the range of the kernels' branch-free
    # division, signed zeros in zero and non-zero rows, quotients far below
    # the smallest E4M3 subnormal
    x = np.zeros((8, k), np.float32)
    x[0, 7] = -0.0
    x[1, :] = np.linspace(-1e30, 1e30, k)
    x[2, :] = np.linspace(-1e-30, 1e-30, k)
    x[3, :] = -np.logspace(-20, 20, k)
    x[4, k - 1] = 3.0                              # the row's last element
    x[5, :] = 2.0 ** -130
    r = np.random.default_rng(k).laplace(size=k).astype(np.float32)
    r[::7] = -0.0
    r[3::11] = -(2.0 ** -133)
    x[6, :] = r
    x[7, :] = r * np.float32(2.0 ** 110)           # row scale above 2^100
    _check_quant(F, torch.from_numpy(x).to(torch.bfloat16), f"special K={k}")


def test_mlp_up_activations_sampled_rows(F):
    x = synth.MLP_UP.activations()
    rows = np.sort(np.random.default_rng(12).choice(x.shape[0], 96, replace=False))
    _check_quant(F, x, "mlp-up", rows=rows)


def _linear(F, wl, rows=None, cols=None):
    x, w, bias = wl.activations(), wl.weight(), wl.bias_vec()
    xq, wq = F.quantize_fp8row(x.cuda()), F.quantize_fp8row(w.cuda())
    y = F.gemm_fp8row(xq, wq, bias=bias.cuda() if bias is not None else None)
    torch.cuda.synchronize()
    ac, as_ = R.quantize_fp8_rowwise(f32(x))
    bc, bs = R.quantize_fp8_rowwise(f32(w))
    r = np.arange(wl.m) if rows is None else rows
    c = np.arange(wl.n) if cols is None else cols
    b_np = None if bias is None else f32(bias)[c]
    y_ref = R.gemm_ref_fp8row(ac[r], as_[r], bc[c], bs[c], b_np)
    tol = R.gemm_tolerance_fp8row(ac[r], as_[r], bc[c], bs[c], y_ref)
    assert_within_tol(y.float().cpu().numpy()[np.ix_(r, c)], y_ref, tol, wl.name)


def test_gemm_tiny(F):
    _linear(F, synth.TINY)


@pytest.mark.parametrize("m,n,k", [(1, 8, 64), (100, 200, 192), (130, 264, 320), (257, 392, 4160), (512, 768, 3072)])
def test_gemm_ragged(F, m, n, k):
    _linear(F, synth.LinearWorkload(f"r8_{m}x{n}x{k}", m, k, n, seed=m * 3 + n + k))


@pytest.mark.parametrize("m,n,k", [(2341, 2056, 3136), (4608, 3072, 1088)])
def test_gemm_wide_tiles_ragged_sampled(F, m, n, k):
    # shapes that take the 256 x 256 tiles: sampled rows and columns, the last
    # ones and those at 128-row / 128-column boundaries included
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert F.nvfp4_gemm_tile_shape(m, n, sms) == (2, 256, 1)
    rng = np.random.default_rng(m + n)
    rows = np.unique(np.r_[rng.choice(m, 40, replace=False), m - 1, 127, 128, 255, 256])
    cols = np.unique(np.r_[rng.choice(n, 64, replace=False), n - 1, 127, 128, 255, 256])
    _linear(F, synth.LinearWorkload(f"r8_wide_{m}x{n}x{k}", m, k, n, seed=m * 3 + n + k), rows=rows, cols=cols)


def test_gemm_mlp_up_sampled(F):
    wl = synth.MLP_UP
    rng = np.random.default_rng(13)
    _linear(F, wl, rows=np.sort(rng.choice(wl.m, 48, replace=False)), cols=np.sort(rng.choice(wl.n, 96, replace=False)))


def test_gemm_bit_exact_when_accumulation_is_exact(F):
    rng = np.random.default_rng(14)
    M, Nn, K = 130, 264, 320
    choices = np.array([0x00, 0x38, 0xB8, 0x40, 0xC0, 0x30, 0xB0], np.uint8)  # 0, +-1, +-2, +-0.5
    a = rng.choice(choices, (M, K))
    b = rng.choice(choices, (Nn, K))
    sa = rng.choice(np.array([0.5, 1.0, 2.0], np.float32), M)
    sb = rng.choice(np.array([0.25, 1.0, 4.0], np.float32), Nn)
    at = F.FP8RowTensor(torch.from_numpy(a).cuda(), torch.from_numpy(sa).cuda(), M, K)
    bt = F.FP8RowTensor(torch.from_numpy(b).cuda(), torch.from_numpy(sb).cuda(), Nn, K)
    y = F.gemm_fp8row(at, bt).float().cpu().numpy()
    assert np.array_equal(y, N.round_to_bf16(R.gemm_ref_fp8row(a, sa, b, sb)))


def test_no_kernel_reported_a_fault(F):
    F.nvfp4_check_fault()
