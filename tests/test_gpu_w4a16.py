"""GPU parity of the W4A16 path ("BFL (fp8r / nvfp4)" doc, section "Kernels",
last paragraph: NVFP4 weights dequantized to the bf16 compute dtype, the
activations left in bf16, a regular linear).

Two entry points: the dequantization alone (nvfp4_dequantize, bit-exact
against the oracle) and the whole layer in one tcgen05 GEMM
(nvfp4_w4a16_gemm), which dequantizes each weight tile in shared memory and
multiplies bf16 x bf16 on the tensor cores.  Its result is checked within the
GEMM tolerance of the oracle's fp64 linear of the same bf16 operands, bit for
bit where the fp32 accumulation is exact, and with a scale-layout probe on
every tile shape.
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


def _plan(F, m, n, k):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return F.nvfp4_gemm_plan(m, n, k, sms, 1)


def _w4a16_check(F, wl, rows=None, cols=None, shape=None):
    x, w, bias = wl.activations(), wl.weight(), wl.bias_vec()
    if shape is not None:
        assert _plan(F, wl.m, wl.n, wl.k) == shape
    g = float(O.global_scale(O.tensor_amax(f32(w))))
    wq = F.quantize(w.cuda(), g)
    y = F.linear_w4a16(x.cuda(), wq, None if bias is None else bias.cuda())
    torch.cuda.synchronize()
    y = y.float().cpu().numpy()
    codes, sf = O.quantize_nvfp4(f32(w), g)
    assert_bytes_equal(gpu_bytes_of(wq.codes), codes, "weight codes")
    rows = np.arange(wl.m) if rows is None else rows
    cols = np.arange(wl.n) if cols is None else cols
    b = None if bias is None else f32(bias)[cols]
    y_ref = O.linear_w4a16_ref(f32(x)[rows], codes[cols], sf[cols], g, b)
    wb = O.dequantize_to_bf16(codes[cols], sf[cols], g).astype(np.float64)
    tol = 2e-3 * np.outer(np.linalg.norm(f32(x)[rows].astype(np.float64), axis=1), np.linalg.norm(wb, axis=1)) \
        + 1e-2 * np.abs(y_ref)
    assert_within_tol(y[np.ix_(rows, cols)], y_ref, tol, wl.name)
    return y


def gpu_bytes_of(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("m", [1, 100, 512])
def test_w4a16_linear_matches_the_oracle(F, m):
    _w4a16_check(F, synth.LinearWorkload(f"w4a16_m{m}", m, 3072, 768, seed=70 + m))


@pytest.mark.parametrize("m,n,k,shape", [(1, 8, 64, (1, 192, 2, 1)), (77, 1000, 4160, (1, 192, 2, 4)),
                                         (300, 520, 1088, (2, 128, 2, 2)), (1000, 2880, 3136, (2, 192, 2, 1)),
                                         (2341, 2056, 1024, (2, 256, 1, 1)), (512, 3072, 3072, (2, 192, 2, 2))])
def test_w4a16_every_tile_shape_ragged(F, m, n, k, shape):
    wl = synth.LinearWorkload(f"w4a16_{m}x{n}x{k}", m, k, n, seed=m + n + k)
    rng = np.random.default_rng(m + n)
    rows = None if m <= 300 else np.unique(np.r_[rng.choice(m, 64, replace=False), m - 1, 255, 256])
    _w4a16_check(F, wl, rows=rows, shape=shape)


def test_w4a16_mlp_up_sampled(F):
    # the MLP-up shape, M = 4608 (wide tiles): all columns of sampled rows
    wl = synth.MLP_UP
    rows = np.sort(np.random.default_rng(5).choice(wl.m, 48, replace=False))
    _w4a16_check(F, wl, rows=rows, shape=(2, 256, 1, 1))


@pytest.mark.parametrize("m,n", [(100, 384), (512, 768), (1000, 2880), (2304, 2304)])
def test_w4a16_exact_accumulation_is_bit_exact(F, m, n):
    # Activations that are small integers, power-of-two weight scales and g:
    # every product and partial sum is exact in fp32, so the bf16 output is
    # the rounded exact result.
    rng = np.random.default_rng(m)
    K = 256
    x = rng.integers(-4, 5, (m, K)).astype(np.float32)
    codes = rng.integers(0, 256, (n, K // 2)).astype(np.uint8)
    sf = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (n, K // 16))   # 0.5, 1, 2
    g = 0.25
    bias = O.round_to_bf16(rng.integers(-64, 64, n) * 0.5).astype(np.float32)
    w = F.NVFP4Tensor(torch.from_numpy(codes).cuda(), torch.from_numpy(O.swizzle_sf(sf)).cuda(), g, n, K)
    y = F.linear_w4a16(torch.from_numpy(x).to(torch.bfloat16).cuda(), w,
                       torch.from_numpy(bias).to(torch.bfloat16).cuda())
    torch.cuda.synchronize()
    want = O.round_to_bf16(O.linear_w4a16_ref(x, codes, sf, g, bias))
    got = y.float().cpu().numpy()
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{bad.shape[0]} differ, first {bad[:4].tolist()}"


def test_w4a16_split_k_is_deterministic(F):
    wl = synth.LinearWorkload("w4a16_det_split", 100, 3072, 3072, seed=12)
    assert _plan(F, wl.m, wl.n, wl.k)[3] == 4
    x, w = wl.activations().cuda(), wl.weight().cuda()
    wq = F.quantize(w, F.global_scale(w))
    ys = [F.linear_w4a16(x, wq) for _ in range(3)]
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])


@pytest.mark.parametrize("m,n,row,kblk", [(100, 384, 37, 3), (100, 384, 200, 15), (512, 768, 130, 9),
                                          (512, 768, 767, 0), (1000, 2880, 2000, 7), (1000, 2880, 95, 12),
                                          (2304, 2304, 131, 5), (2304, 2304, 2303, 15)])
def test_w4a16_weight_scale_layout_probe(F, m, n, row, kblk):
    # Every weight element 1.0 with unit scales except one block scale 2.0:
    # exactly output column `row` grows, by 16 (x = 1).
    K = 256
    codes = np.full((n, K // 2), 0x22, np.uint8)
    sf = np.full((n, K // 16), 0x38, np.uint8)
    sf[row, kblk] = 0x40
    w = F.NVFP4Tensor(torch.from_numpy(codes).cuda(), torch.from_numpy(O.swizzle_sf(sf)).cuda(), 1.0, n, K)
    y = F.linear_w4a16(torch.ones(m, K, dtype=torch.bfloat16, device="cuda"), w)
    torch.cuda.synchronize()
    want = np.full((m, n), float(K))
    want[:, row] += 16
    got = y.float().cpu().numpy()
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{bad.shape[0]} wrong, first {bad[:4].tolist()} got {got[tuple(bad[0])]}"


def test_no_kernel_reported_a_fault(F):
    F.nvfp4_check_fault()
