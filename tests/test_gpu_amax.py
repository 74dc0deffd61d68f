"""GPU parity of the one-pass dynamic scale: the GEMM epilogue that measures
max|Y| of its own output (nvfp4_gemm_amax) and the quantizer that derives
the per-tensor scale from a given amax on the device
(nvfp4_quantize_from_amax).

This is the one-pass alternative to the two-pass dynamic quantize: the amax
of a layer's input is emitted by the previous layer's epilogue ("BFL (fp8r /
nvfp4)" doc, ``nvfp4`` bullet: the measured scale is the variant of the
calibrated ``input_scale``).  The amax must equal
the largest magnitude of the bf16 values the GEMM wrote, bit for bit, and the
GEMM's Y must not change; the one-pass quantize must give the oracle's codes,
scales, amax and g bit for bit, i.e. the same bytes as the two-pass dynamic
quantize of the same tensor.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from tests.gpu_helpers import assert_bytes_equal, f32, gpu_bytes, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    require_gpu()
    import nvfp4_block_scaled_12_b200 as F
    return F


def _layer(F, wl):
    x, w = wl.activations().cuda(), wl.weight().cuda()
    b = wl.bias_vec()
    return F.quantize(x, F.global_scale(x)), F.quantize(w, F.global_scale(w)), None if b is None else b.cuda()


def _plan(F, m, n, k):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return F.nvfp4_gemm_plan(m, n, k, sms, 0)


@pytest.mark.parametrize("m,n,k,ks", [(128, 256, 256, None), (300, 520, 1024, None), (77, 1000, 4160, 4),
                                      (100, 3072, 3072, 4), (2341, 2056, 3136, None), (4608, 3072, 3072, None)])
def test_gemm_amax_is_the_largest_output_magnitude(F, m, n, k, ks):
    # ragged M and N (rows past M and columns past N must not count), every
    # epilogue (wide, standard, and the K split's reduction)
    if ks is not None:
        assert _plan(F, m, n, k)[3] == ks
    xq, wq, b = _layer(F, synth.LinearWorkload(f"amax_{m}x{n}x{k}", m, k, n, seed=m + n + k))
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    y = F.gemm(xq, wq, bias=b, amax_out=amax)
    y_plain = F.gemm(xq, wq, bias=b)
    torch.cuda.synchronize()
    assert torch.equal(y, y_plain), "the amax epilogue changed Y"
    want = np.float32(np.max(np.abs(y.float().cpu().numpy())))
    assert amax.item() == want, (amax.item(), want)


def test_gemm_amax_folds_into_the_given_maximum(F):
    xq, wq, b = _layer(F, synth.LinearWorkload("amax_fold", 300, 1024, 520, seed=5))
    y = F.gemm(xq, wq, bias=b)
    torch.cuda.synchronize()
    ymax = float(y.float().abs().max())
    big = torch.full((1,), 4.0 * ymax, dtype=torch.float32, device="cuda")
    small = torch.full((1,), 0.25 * ymax, dtype=torch.float32, device="cuda")
    F.gemm(xq, wq, bias=b, amax_out=big)
    F.gemm(xq, wq, bias=b, amax_out=small)
    torch.cuda.synchronize()
    assert big.item() == np.float32(4.0 * ymax) and small.item() == np.float32(ymax)


def test_gemm_amax_with_the_activation_scale_on_the_device(F):
    # a layer whose input was quantized with a measured scale: alpha read on
    # the device, Y identical to the dynamic GEMM's
    wl = synth.LinearWorkload("amax_dyn", 512, 3072, 768, seed=9)
    x, w = wl.activations().cuda(), wl.weight().cuda()
    xq = F.quantize_dynamic(x)
    wq = F.quantize(w, F.global_scale(w))
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    y = F.gemm(xq, wq, bias=wl.bias_vec().cuda(), amax_out=amax)
    y_dyn = F.gemm(xq, wq, bias=wl.bias_vec().cuda())
    torch.cuda.synchronize()
    assert torch.equal(y, y_dyn)
    assert amax.item() == np.float32(np.max(np.abs(y.float().cpu().numpy())))


def _check_from_amax(F, x_bf16, amax_value, what):
    x = x_bf16.cuda()
    amax = torch.full((1,), float(amax_value), dtype=torch.float32, device="cuda")
    q = F.quantize_from_amax(x, amax)
    torch.cuda.synchronize()
    # the oracle's rule for this amax: dynamic_scale of a tensor whose largest
    # magnitude is amax_value
    a_ref, g = O.dynamic_scale(np.array([[np.float32(amax_value)]], np.float32))
    got = q.scale.cpu().numpy()
    assert got[0] == a_ref and got[1] == g, (what, got, a_ref, g)
    M, K = x_bf16.shape
    if g == 0:
        codes, sf = np.zeros((M, K // 2), np.uint8), np.zeros((M, K // 16), np.uint8)
    else:
        codes, sf = O.quantize_nvfp4(f32(x_bf16), g)
    assert_bytes_equal(gpu_bytes(q.codes), codes, what + " codes")
    assert_bytes_equal(gpu_bytes(q.sf), O.swizzle_sf(sf), what + " scale buffer")
    return q


@pytest.mark.parametrize("m,k", [(1, 64), (7, 192), (300, 4160), (1000, 3072)])
def test_quantize_from_amax_matches_the_oracle(F, m, k):
    x = synth.activations_with_outlier_channels(m, k, seed=2 * m + k)
    _check_from_amax(F, x, O.tensor_amax(f32(x)), f"from_amax {m}x{k}")


def test_quantize_from_amax_with_another_amax_and_the_clamps(F):
    # the amax need not be the tensor's own: a larger one (as after a
    # max over several outputs), the smallest and largest g, and g = 0
    x = synth.activations_with_outlier_channels(128, 256, seed=4)
    a = O.tensor_amax(f32(x))
    _check_from_amax(F, x, 3.0 * a, "larger amax")
    _check_from_amax(F, torch.zeros(128, 256, dtype=torch.bfloat16), 0.0, "zero amax")
    tiny = (x.float() * 2.0 ** -100).to(torch.bfloat16)
    _check_from_amax(F, tiny, O.tensor_amax(f32(tiny)), "g clamped to 2^-64")
    huge = (x.float() * 2.0 ** 90).to(torch.bfloat16)
    _check_from_amax(F, huge, O.tensor_amax(f32(huge)), "g clamped to 2^64")


def test_two_layers_with_the_amax_from_the_epilogue(F):
    # layer 1 writes Y1 and its amax; layer 2's input is quantized in one pass
    # from that amax: the same bytes as the oracle's dynamic quantize of the
    # kernel's own Y1, and as the two-pass dynamic quantize
    xq, wq, b = _layer(F, synth.LinearWorkload("chain1", 1000, 3072, 3072, seed=21))
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    y1 = F.gemm(xq, wq, bias=b, amax_out=amax)
    q1 = F.quantize_from_amax(y1, amax)
    q2 = F.quantize_dynamic(y1)
    torch.cuda.synchronize()
    codes, sf, a_ref, g = O.quantize_dynamic(f32(y1.cpu()))
    got = q1.scale.cpu().numpy()
    assert got[0] == a_ref and got[1] == g
    assert_bytes_equal(gpu_bytes(q1.codes), codes, "chain codes")
    assert_bytes_equal(gpu_bytes(q1.sf), O.swizzle_sf(sf), "chain scales")
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.sf, q2.sf) and torch.equal(q1.scale, q2.scale)


def test_no_kernel_reported_a_fault(F):
    F.nvfp4_check_fault()
