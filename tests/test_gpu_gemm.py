"""GPU parity of the block-scaled NVFP4 GEMM against the oracle.

The GEMM is the `mm_fp4` NVFP4 x NVFP4 product of an NVFP4 linear layer
("BFL (fp8r / nvfp4)" diffusers doc, section "Kernels"), with
y = bf16(alpha * acc + bias) and alpha = input_scale * weight_scale_2.
Results must lie within |y - y_ref| <= 2e-3 |a_m| |b_n| + 1e-2 |y_ref| of the
oracle's fp64 dequantize-then-matmul; cases whose fp32 accumulation is exact
must match bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from tests.gpu_helpers import assert_within_tol, f32, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    require_gpu()
    import nvfp4_block_scaled_12_b200 as F
    return F


def _gpu_layer(F, x_bf16, w_bf16):
    """The CUDA path: calibrate and quantize both operands on the GPU."""
    x = x_bf16.cuda()
    w = w_bf16.cuda()
    xq = F.quantize(x, F.global_scale(x))
    wq = F.quantize(w, F.global_scale(w))
    return xq, wq


def _oracle_layer(x_bf16, w_bf16):
    x = f32(x_bf16)
    w = f32(w_bf16)
    gx = O.global_scale(O.tensor_amax(x))
    gw = O.global_scale(O.tensor_amax(w))
    xc, xs = O.quantize_nvfp4(x, gx)
    wc, ws = O.quantize_nvfp4(w, gw)
    return (xc, xs, gx), (wc, ws, gw)


def _check_linear(F, wl: synth.LinearWorkload, rows=None, cols=None):
    x, w, b = wl.activations(), wl.weight(), wl.bias_vec()
    xq, wq = _gpu_layer(F, x, w)
    y = F.gemm(xq, wq, bias=None if b is None else b.cuda())
    torch.cuda.synchronize()
    y = y.float().cpu().numpy()
    (xc, xs, gx), (wc, ws, gw) = _oracle_layer(x, w)
    assert np.float32(xq.g) == gx and np.float32(wq.g) == gw
    bias = None if b is None else b.float().numpy()
    rows = np.arange(wl.m) if rows is None else rows
    cols = np.arange(wl.n) if cols is None else cols
    y_ref = O.gemm_ref(xc[rows], xs[rows], gx, wc[cols], ws[cols], gw, None if bias is None else bias[cols])
    tol = O.gemm_tolerance(xc[rows], xs[rows], gx, wc[cols], ws[cols], gw, y_ref)
    assert_within_tol(y[np.ix_(rows, cols)], y_ref, tol, wl.name)
    return y


def test_tiny_workload(F):
    _check_linear(F, synth.TINY)


@pytest.mark.parametrize("m,n,k", [(1, 8, 64), (100, 200, 192), (129, 392, 320), (300, 64, 1024),
                                   (128, 192, 256), (256, 384, 512), (77, 1000, 4096), (1000, 3000, 1088),
                                   (300, 520, 15360), (97, 136, 15424)])
def test_ragged_shapes(F, m, n, k):
    _check_linear(F, synth.LinearWorkload(f"ragged_{m}x{n}x{k}", m, k, n, seed=m + n + k))


@pytest.mark.parametrize("idx", [0, 1])
def test_sweep_small_token_counts_full(F, idx):
    _check_linear(F, synth.SWEEP[idx])


@pytest.mark.parametrize("idx", [2, 3, 4])
def test_sweep_large_token_counts_sampled(F, idx):
    # The token sweep's larger points (M = 4608, 9216, 16896; K = N = 3072):
    # all columns of sampled rows (the last ones included) and all rows of
    # sampled columns.
    wl = synth.SWEEP[idx]
    rng = np.random.default_rng(wl.seed)
    rows = np.unique(np.r_[rng.choice(wl.m, 64, replace=False), wl.m - 1, wl.m - 129, 255, 256])
    y = _check_linear(F, wl, rows=rows)
    x, w, b = wl.activations(), wl.weight(), wl.bias_vec()
    (xc, xs, gx), (wc, ws, gw) = _oracle_layer(x, w)
    cols = np.unique(np.r_[rng.choice(wl.n, 48, replace=False), wl.n - 1, 255, 256])
    y_ref = O.gemm_ref(xc, xs, gx, wc[cols], ws[cols], gw, b.float().numpy()[cols])
    tol = O.gemm_tolerance(xc, xs, gx, wc[cols], ws[cols], gw, y_ref)
    assert_within_tol(y[:, cols], y_ref, tol, wl.name + " columns")


def test_mlp_up_full_size_sampled(F):
    # The benchmarked shape M=4608, K=3072, N=12288 with bias: all columns of
    # a seeded sample of rows, and all rows of a sample of columns.
    wl = synth.MLP_UP
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(wl.m, 96, replace=False))
    y = _check_linear(F, wl, rows=rows)
    x, w, b = wl.activations(), wl.weight(), wl.bias_vec()
    (xc, xs, gx), (wc, ws, gw) = _oracle_layer(x, w)
    cols = np.sort(rng.choice(wl.n, 96, replace=False))
    y_ref = O.gemm_ref(xc, xs, gx, wc[cols], ws[cols], gw, b.float().numpy()[cols])
    tol = O.gemm_tolerance(xc, xs, gx, wc[cols], ws[cols], gw, y_ref)
    assert_within_tol(y[:, cols], y_ref, tol, wl.name + " columns")


def _uniform_operand(rows, k, code=0x22, scale=0x38):
    return np.full((rows, k // 2), code, np.uint8), np.full((rows, k // 16), scale, np.uint8)


def _run_raw(F, a_codes, a_sf, b_codes, b_sf, alpha=1.0, bias=None):
    M, N, K = a_codes.shape[0], b_codes.shape[0], a_codes.shape[1] * 2
    a = F.NVFP4Tensor(torch.from_numpy(a_codes).cuda(), torch.from_numpy(O.swizzle_sf(a_sf)).cuda(), 1.0, M, K)
    b = F.NVFP4Tensor(torch.from_numpy(b_codes).cuda(), torch.from_numpy(O.swizzle_sf(b_sf)).cuda(), 1.0, N, K)
    y = F.gemm(a, b, bias=None if bias is None else torch.from_numpy(bias).to(torch.bfloat16).cuda(), alpha=alpha)
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


@pytest.mark.parametrize("side", ["a", "b"])
@pytest.mark.parametrize("row,kblk", [(0, 0), (37, 3), (127, 5), (128, 0), (200, 17), (255, 9), (300, 31)])
def test_scale_layout_probe(F, side, row, kblk):
    # All elements 1.0 and all scales 1.0, except one scale 2.0 at (row, kblk)
    # of one operand: exactly one output row (or column) grows by 16.
    M = N = 384
    K = 512
    ac, asf = _uniform_operand(M, K)
    bc, bsf = _uniform_operand(N, K)
    (asf if side == "a" else bsf)[row, kblk] = 0x40  # 2.0
    y = _run_raw(F, ac, asf, bc, bsf)
    want = np.full((M, N), float(K))
    if side == "a":
        want[row, :] += 16
    else:
        want[:, row] += 16
    bad = np.argwhere(y != want)
    assert bad.size == 0, f"{bad.shape[0]} wrong, first {bad[:4].tolist()} got {y[tuple(bad[0])]}"


def test_exact_accumulation_is_bit_exact(F):
    # Codes and power-of-two scales small enough that every fp32 partial sum
    # is exact: the GPU's bf16 output must equal the rounded exact result.
    rng = np.random.default_rng(12)
    M, N, K = 256, 384, 256
    a_codes = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    b_codes = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    pow2 = np.array([0x30, 0x38, 0x40], np.uint8)  # 0.5, 1, 2: |partial sums| < 2^16, step 2^-4
    a_sf = rng.choice(pow2, (M, K // 16))
    b_sf = rng.choice(pow2, (N, K // 16))
    bias = O.round_to_bf16(rng.integers(-64, 64, N) * 0.5)
    y = _run_raw(F, a_codes, a_sf, b_codes, b_sf, alpha=0.5, bias=bias.astype(np.float32))
    y_ref = O.gemm_ref(a_codes, a_sf, 1.0, b_codes, b_sf, 1.0, None) * 0.5 + bias
    want = O.round_to_bf16(y_ref)
    bad = np.argwhere(y != want)
    assert bad.size == 0, f"{bad.shape[0]} differ, first {bad[:4].tolist()}: {y[tuple(bad[0])]} vs {want[tuple(bad[0])]}"


def test_closed_form_constant_operands(F):
    M, N, K = 130, 200, 3072
    ac, asf = _uniform_operand(M, K, code=0x55, scale=0x30)  # 3.0 * 0.5
    bc, bsf = _uniform_operand(N, K, code=0xBB, scale=0x38)  # -1.5 * 1.0
    y = _run_raw(F, ac, asf, bc, bsf, alpha=2.0 ** -4)
    assert np.all(y == K * (1.5 * -1.5) * 2.0 ** -4)


def test_gemm_is_deterministic(F):
    wl = synth.LinearWorkload("det", 512, 1024, 768, seed=9)
    xq, wq = _gpu_layer(F, wl.activations(), wl.weight())
    b = wl.bias_vec().cuda()
    y1 = F.gemm(xq, wq, bias=b)
    y2 = F.gemm(xq, wq, bias=b)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def _wide(M, N):
    """True when the library takes its 256 x 256 CTA-pair tiles for this
    GEMM on this device."""
    import nvfp4_block_scaled_12_b200 as F
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return F.nvfp4_gemm_tile_shape(M, N, sms) == (2, 256, 1)


@pytest.mark.parametrize("m,n,k", [(2341, 2056, 3136), (4608, 3072, 3072), (2305, 8200, 1088),
                                   (2341, 2056, 15360)])
def test_wide_tiles_ragged_sampled(F, m, n, k):
    # Shapes that take the 256 x 256 tiles, ragged in M, N and K (a last
    # k-tile with one or two MMA k-blocks): all columns of sampled rows (the
    # last rows included) and all rows of sampled columns (the last included).
    assert _wide(m, n)
    wl = synth.LinearWorkload(f"wide_{m}x{n}x{k}", m, k, n, seed=m + 3 * n + k)
    rng = np.random.default_rng(m + n)
    rows = np.unique(np.r_[rng.choice(m, 64, replace=False), m - 1, m - 2, 255, 256])
    y = _check_linear(F, wl, rows=rows)
    x, w, b = wl.activations(), wl.weight(), wl.bias_vec()
    (xc, xs, gx), (wc, ws, gw) = _oracle_layer(x, w)
    cols = np.unique(np.r_[rng.choice(n, 64, replace=False), n - 1, n - 8, 127, 128, 255, 256])
    y_ref = O.gemm_ref(xc, xs, gx, wc[cols], ws[cols], gw, b.float().numpy()[cols])
    tol = O.gemm_tolerance(xc, xs, gx, wc[cols], ws[cols], gw, y_ref)
    assert_within_tol(y[:, cols], y_ref, tol, wl.name + " columns")


@pytest.mark.parametrize("side", ["a", "b"])
@pytest.mark.parametrize("row,kblk", [(0, 0), (131, 3), (255, 17), (256, 6), (700, 31), (2303, 9)])
def test_wide_tiles_scale_layout_probe(F, side, row, kblk):
    # As test_scale_layout_probe, on a shape that takes the 256 x 256 tiles:
    # the probed row lands in either 128-row half of an A tile and in either
    # 128-column half of a B tile.
    M = N = 2304
    K = 512
    assert _wide(M, N)
    ac, asf = _uniform_operand(M, K)
    bc, bsf = _uniform_operand(N, K)
    (asf if side == "a" else bsf)[row, kblk] = 0x40  # 2.0
    y = _run_raw(F, ac, asf, bc, bsf)
    want = np.full((M, N), float(K))
    if side == "a":
        want[row, :] += 16
    else:
        want[:, row] += 16
    bad = np.argwhere(y != want)
    assert bad.size == 0, f"{bad.shape[0]} wrong, first {bad[:4].tolist()} got {y[tuple(bad[0])]}"


def test_wide_tiles_exact_accumulation_is_bit_exact(F):
    rng = np.random.default_rng(21)
    M, N, K = 2304, 2304, 256
    assert _wide(M, N)
    a_codes = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    b_codes = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    pow2 = np.array([0x30, 0x38, 0x40], np.uint8)
    a_sf = rng.choice(pow2, (M, K // 16))
    b_sf = rng.choice(pow2, (N, K // 16))
    bias = O.round_to_bf16(rng.integers(-64, 64, N) * 0.5)
    y = _run_raw(F, a_codes, a_sf, b_codes, b_sf, alpha=0.5, bias=bias.astype(np.float32))
    want = O.round_to_bf16(O.gemm_ref(a_codes, a_sf, 1.0, b_codes, b_sf, 1.0, None) * 0.5 + bias)
    bad = np.argwhere(y != want)
    assert bad.size == 0, f"{bad.shape[0]} differ, first {bad[:4].tolist()}: {y[tuple(bad[0])]} vs {want[tuple(bad[0])]}"


def test_wide_tiles_are_deterministic(F):
    wl = synth.LinearWorkload("det_wide", 4608, 1024, 4096, seed=10)
    assert _wide(wl.m, wl.n)
    xq, wq = _gpu_layer(F, wl.activations(), wl.weight())
    b = wl.bias_vec().cuda()
    y1 = F.gemm(xq, wq, bias=b)
    y2 = F.gemm(xq, wq, bias=b)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def _plan(F, m, n, k, w16=0):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return F.nvfp4_gemm_plan(m, n, k, sms, w16)


@pytest.mark.parametrize("m,n,k,ks", [(100, 3072, 3072, 4), (77, 1000, 4160, 4), (16, 3072, 15360, 4),
                                      (1, 8, 4096, 4), (300, 520, 15360, 2), (129, 392, 4096, 2)])
def test_split_k_matches_the_oracle(F, m, n, k, ks):
    # A few hundred tokens or fewer: CTAs of one cluster share each output
    # tile over disjoint k-tile ranges and sum their partial tiles through
    # distributed shared memory; ragged M, N and a last k-tile of one k-block.
    assert _plan(F, m, n, k)[3] == ks
    _check_linear(F, synth.LinearWorkload(f"split_{m}x{n}x{k}", m, k, n, seed=m + 7 * n + k))


def test_split_k_exact_accumulation_is_bit_exact(F):
    # every partial sum and their sum are exact in fp32, so the split result
    # equals the rounded exact result bit for bit
    rng = np.random.default_rng(33)
    M, N, K = 100, 384, 4096  # |partial sums| < 2^20, a step of 2^-4: exact in fp32
    assert _plan(F, M, N, K)[3] == 4
    a_codes = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    b_codes = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    pow2 = np.array([0x30, 0x38, 0x40], np.uint8)
    a_sf, b_sf = rng.choice(pow2, (M, K // 16)), rng.choice(pow2, (N, K // 16))
    bias = O.round_to_bf16(rng.integers(-64, 64, N) * 0.5)
    y = _run_raw(F, a_codes, a_sf, b_codes, b_sf, alpha=0.5, bias=bias.astype(np.float32))
    want = O.round_to_bf16(O.gemm_ref(a_codes, a_sf, 1.0, b_codes, b_sf, 1.0, None) * 0.5 + bias)
    bad = np.argwhere(y != want)
    assert bad.size == 0, f"{bad.shape[0]} differ, first {bad[:4].tolist()}"


def test_split_k_is_deterministic(F):
    wl = synth.LinearWorkload("det_split", 300, 15360, 520, seed=11)
    assert _plan(F, wl.m, wl.n, wl.k)[3] == 2
    xq, wq = _gpu_layer(F, wl.activations(), wl.weight())
    b = wl.bias_vec().cuda()
    ys = [F.gemm(xq, wq, bias=b) for _ in range(3)]
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])


def test_long_k(F):
    # K = 65536: 256 k-tiles, split over CTA pairs, offsets far past the
    # sizes of the other tests
    wl = synth.LinearWorkload("long_k", 300, 65536, 256, seed=99)
    assert _plan(F, wl.m, wl.n, wl.k)[3] > 1
    _check_linear(F, wl)


def test_no_kernel_reported_a_fault(F):
    F.nvfp4_check_fault()
