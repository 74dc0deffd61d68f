"""GPU parity of the dynamic-scale path: the quantizer that measures the
per-tensor activation scale in the same launch, and the GEMM that reads
that scale from device memory.

A measured scale is the variant of the calibrated ``input_scale`` ("BFL
(fp8r / nvfp4)" diffusers doc, ``nvfp4`` bullet).  Codes, scales, amax and g
must equal the oracle's bit for bit; the GEMM must equal the static-scale
GEMM bit for bit when that is given the same alpha.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from tests.gpu_helpers import assert_bytes_equal, assert_within_tol, f32, gpu_bytes, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    require_gpu()
    import nvfp4_block_scaled_12_b200 as F
    return F


def _check_dynamic(F, x_bf16: torch.Tensor, what: str, rows=None):
    xq = F.quantize_dynamic(x_bf16.cuda())
    torch.cuda.synchronize()
    x = f32(x_bf16)
    amax, g = O.dynamic_scale(x)
    got = xq.scale.cpu().numpy()
    assert got[0] == amax, (what, got[0], amax)
    assert got[1] == g, (what, got[1], g)
    M, K = x.shape
    sel = np.arange(M) if rows is None else rows
    if g == 0:
        codes = np.zeros((len(sel), K // 2), np.uint8)
        sf = np.zeros((len(sel), K // 16), np.uint8)
    else:
        codes, sf = O.quantize_nvfp4(x[sel], g)
    assert_bytes_equal(gpu_bytes(xq.codes)[sel], codes, what + " codes")
    sf_lin = O.unswizzle_sf(gpu_bytes(xq.sf), M, K)
    assert_bytes_equal(sf_lin[sel], sf, what + " scales")
    if rows is None:  # the padding rows of the scale buffer are zero too
        assert_bytes_equal(gpu_bytes(xq.sf), O.swizzle_sf(sf_lin), what + " scale buffer")
    return xq


def test_tiny_workload(F):
    _check_dynamic(F, synth.TINY.activations(), "tiny")


@pytest.mark.parametrize("m,k", [(1, 64), (7, 192), (127, 320), (300, 4160), (1000, 3072)])
def test_ragged_shapes(F, m, k):
    _check_dynamic(F, synth.activations_with_outlier_channels(m, k, seed=m + 3 * k), f"ragged {m}x{k}")


def test_mlp_up_activations_sampled_rows(F):
    # more tiles than SMs: every CTA folds several tiles into the maximum
    x = synth.MLP_UP.activations()
    rows = np.sort(np.random.default_rng(3).choice(x.shape[0], 64, replace=False))
    _check_dynamic(F, x, "mlp-up", rows=rows)


def test_laplace_workload_sampled_rows(F):
    x = synth.quantize_input()
    rows = np.sort(np.random.default_rng(4).choice(x.shape[0], 48, replace=False))
    _check_dynamic(F, x, "laplace 4608x12288", rows=rows)


def test_all_zero_tensor_gives_zero_scale_and_output(F):
    x = torch.zeros(300, 256, dtype=torch.bfloat16)
    x[5, 7] = -0.0
    xq = _check_dynamic(F, x, "zeros")
    assert not xq.codes.any() and not xq.sf.any()


@pytest.mark.parametrize("value", [2.0 ** -100, 2.0 ** 120, -3.0e-20])
def test_scale_is_clamped_like_the_oracle(F, value):
    rng = np.random.default_rng(8)
    x = (rng.uniform(0.25, 1.0, (130, 128)) * value).astype(np.float32)
    _check_dynamic(F, torch.from_numpy(x).to(torch.bfloat16), f"clamp {value}")


def test_repeated_calls_reuse_the_workspace(F):
    x = synth.laplace_activations(640, 3072, seed=91).cuda()
    ws = torch.full((F.NVFP4_DYNAMIC_WORKSPACE_BYTES,), 0xAB, dtype=torch.uint8, device="cuda")  # stale contents
    a = F.quantize_dynamic(x, workspace=ws)
    b = F.quantize_dynamic(x * 2, workspace=ws)   # different scale, same workspace
    c = F.quantize_dynamic(x, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, c.codes) and torch.equal(a.sf, c.sf) and torch.equal(a.scale, c.scale)
    assert b.scale[0].item() == 2 * a.scale[0].item()


def test_dynamic_gemm_equals_the_static_gemm_with_the_same_alpha(F):
    wl = synth.TINY
    x, w = wl.activations(), wl.weight()
    wq = F.quantize(w.cuda(), float(O.global_scale(O.tensor_amax(f32(w)))))
    xq = F.quantize_dynamic(x.cuda())
    y_dyn = F.gemm(xq, wq)
    g_a = float(xq.scale[1].item())
    alpha = float(np.float32(g_a) * np.float32(wq.g))
    y_static = F.gemm(xq, wq, alpha=alpha)
    torch.cuda.synchronize()
    assert torch.equal(y_dyn, y_static)


def test_dynamic_linear_layer_matches_the_oracle(F):
    # x -> quantize with a measured scale -> GEMM with the device-side scale,
    # on a few tiles of the MLP-up shape with bias.
    wl = synth.LinearWorkload("dynamic_m512_k3072_n768", 512, 3072, 768, seed=17)
    x, w, bias = wl.activations(), wl.weight(), wl.bias_vec()
    g_w = float(O.global_scale(O.tensor_amax(f32(w))))
    wq = F.quantize(w.cuda(), g_w)
    xq = F.quantize_dynamic(x.cuda())
    y = F.gemm(xq, wq, bias=bias.cuda()).float().cpu().numpy()
    a_codes, a_sf, _, g_a = O.quantize_dynamic(f32(x))
    b_codes, b_sf = O.quantize_nvfp4(f32(w), g_w)
    y_ref = O.gemm_ref(a_codes, a_sf, g_a, b_codes, b_sf, g_w, f32(bias))
    tol = O.gemm_tolerance(a_codes, a_sf, g_a, b_codes, b_sf, g_w, y_ref)
    assert_within_tol(y, y_ref, tol, "dynamic linear")


def test_no_kernel_reported_a_fault(F):
    F.nvfp4_check_fault()
