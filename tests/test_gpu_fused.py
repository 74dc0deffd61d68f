"""GPU parity of the fused epilogue: GEMM -> (GELU-tanh) -> the next layer's
NVFP4 activations, plus bf16 column ranges.

Several byte results are correct here (the GEMM itself is only defined to a
tolerance), so the checks are: the bf16 ranges are within the GEMM
tolerance of the oracle; the fused NVFP4 bytes equal the GPU's own
standalone quantizer applied to the GPU's own bf16 values of those columns
(bit-exact); the dequantized fused values are within tolerance of the
oracle's epilogue; and in an exactly-accumulated case the identity range
matches the oracle's bytes bit for bit.
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


def _layer(F, wl):
    x, w, b = wl.activations(), wl.weight(), wl.bias_vec()
    xd, wd = x.cuda(), w.cuda()
    xq = F.quantize(xd, F.global_scale(xd))
    wq = F.quantize(wd, F.global_scale(wd))
    return x, w, b, xq, wq


def _empty_nvfp4(F, m, k):
    return F.NVFP4Tensor(torch.zeros(m, k // 2, dtype=torch.uint8, device="cuda"),
                         torch.full((F.nvfp4_sf_bytes(m, k),), 0xAA, dtype=torch.uint8, device="cuda"), 1.0, m, k)


def _fused_vs_references(F, wl, q_rng, bf_rng, act_rng, g_next, rows=None):
    """Run ranges: q_rng -> NVFP4 identity at dst 0; bf_rng -> bf16; act_rng
    -> GELU -> NVFP4 after q.  Returns everything needed to compare."""
    x, w, b, xq, wq = _layer(F, wl)
    bias = b.cuda() if b is not None else None
    q_w = q_rng[1] - q_rng[0]
    a_w = act_rng[1] - act_rng[0]
    k_next = q_w + a_w
    nxt = _empty_nvfp4(F, wl.m, k_next)
    ybf = torch.zeros(wl.m, bf_rng[1] - bf_rng[0], dtype=torch.bfloat16, device="cuda")
    ranges = [(q_rng[0], q_rng[1], F.ACT_NONE, F.DST_NVFP4, 0),
              (bf_rng[0], bf_rng[1], F.ACT_NONE, F.DST_BF16, 0),
              (act_rng[0], act_rng[1], F.ACT_GELU_TANH, F.DST_NVFP4, q_w)]
    F.gemm_quant(xq, wq, ranges, bias=bias, y_bf16=ybf, g_next=g_next, next_out=nxt)
    # the same kernel with every range sent to bf16: the GPU's own values
    all_bf = torch.zeros(wl.m, k_next, dtype=torch.bfloat16, device="cuda")
    F.gemm_quant(xq, wq, [(q_rng[0], q_rng[1], F.ACT_NONE, F.DST_BF16, 0),
                          (act_rng[0], act_rng[1], F.ACT_GELU_TANH, F.DST_BF16, q_w)],
                 bias=bias, y_bf16=all_bf)
    requant = F.quantize(all_bf, g_next)
    torch.cuda.synchronize()
    return x, w, b, xq, wq, nxt, ybf, all_bf, requant, k_next


def _check_fused(F, wl, q_rng, bf_rng, act_rng, rows):
    g_next = 0.01
    x, w, b, xq, wq, nxt, ybf, all_bf, requant, k_next = _fused_vs_references(F, wl, q_rng, bf_rng, act_rng,
                                                                               g_next)
    # (1) fused bytes == GPU quantize of the GPU's own bf16 values
    assert_bytes_equal(gpu_bytes(nxt.codes), gpu_bytes(requant.codes), "fused codes vs requantized")
    assert_bytes_equal(gpu_bytes(nxt.sf), gpu_bytes(requant.sf), "fused scales vs requantized")

    # (2) bf16 outputs within the GEMM tolerance of the oracle
    xf, wf = f32(x), f32(w)
    gx, gw = O.global_scale(O.tensor_amax(xf)), O.global_scale(O.tensor_amax(wf))
    xc, xs = O.quantize_nvfp4(xf[rows], gx)
    wc, ws = O.quantize_nvfp4(wf, gw)
    bias = b.float().numpy() if b is not None else None
    y_ref = O.gemm_ref(xc, xs, gx, wc, ws, gw, bias)
    tol = O.gemm_tolerance(xc, xs, gx, wc, ws, gw, y_ref)
    ybf_np = ybf.float().cpu().numpy()[rows]
    sl = slice(*bf_rng)
    assert_within_tol(ybf_np, O.round_to_bf16(y_ref[:, sl]), tol[:, sl] + np.abs(y_ref[:, sl]) * 2.0 ** -8,
                      "bf16 range")
    # (3) the GPU's pre-quantization values (identity and GELU) vs the oracle epilogue
    ep_ref = O.epilogue_ref(y_ref, [(q_rng[0], q_rng[1], O.ACT_NONE), (act_rng[0], act_rng[1], O.ACT_GELU_TANH)])
    ep_tol = np.concatenate([tol[:, slice(*q_rng)], 1.2 * tol[:, slice(*act_rng)]], axis=1)
    ep_tol = ep_tol + np.abs(ep_ref) * 2.0 ** -7 + 1e-6
    all_np = all_bf.float().cpu().numpy()[rows]
    assert_within_tol(all_np, ep_ref, ep_tol, "epilogue values")
    # (4) dequantized fused NVFP4 output vs the oracle epilogue, within the
    # tolerance plus one quantization step of the block
    codes = gpu_bytes(nxt.codes)[rows]
    sf_lin = O.unswizzle_sf(gpu_bytes(nxt.sf), wl.m, k_next)[rows]
    deq = O.dequantize(codes, sf_lin, g_next)
    step = (O.e4m3_decode(sf_lin) * g_next).repeat(16, axis=1)
    assert_within_tol(deq, ep_ref, ep_tol + 1.01 * step, "dequantized fused output")
    # (5) scale padding rows are zero
    m = wl.m
    sf_all = gpu_bytes(nxt.sf)
    mp = (m + 127) // 128 * 128
    if mp > m:
        r, c = np.meshgrid(np.arange(m, mp), np.arange(k_next // 16), indexing="ij")
        assert np.all(sf_all[O.sf_offset(r, c, k_next // 16)] == 0)


def test_fused_small(F):
    wl = synth.LinearWorkload("fused_small", 200, 256, 640, seed=21)
    _check_fused(F, wl, (0, 128), (128, 384), (384, 640), rows=np.arange(200))


def test_fused_single_stream_block_shape_sampled(F):
    # FLUX single-stream fused QKV+MLP-in GEMM: Q -> NVFP4, K/V -> bf16,
    # MLP -> GELU-tanh -> NVFP4, together the output projection's input.
    wl = synth.SINGLE_IN
    rows = np.sort(np.random.default_rng(3).choice(wl.m, 48, replace=False))
    _check_fused(F, wl, synth.SINGLE_Q, synth.SINGLE_KV, synth.SINGLE_MLP, rows=rows)


def test_fused_256x192_tiles_sampled(F):
    # about a thousand tokens: 256 x 192 tiles (too few for the wide ones, too
    # many 256 x 128 ones for a single wave)
    wl = synth.LinearWorkload("fused_mid", 1000, 1088, 2880, seed=24)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert F.nvfp4_gemm_tile_shape(wl.m, wl.n, sms) == (2, 192, 2)
    rows = np.unique(np.r_[np.random.default_rng(24).choice(wl.m, 40, replace=False), wl.m - 1, 255, 256])
    _check_fused(F, wl, (0, 768), (768, 1408), (1408, 2880), rows=rows)


def test_fused_wide_tiles_ragged_sampled(F):
    # A shape that takes the 256 x 256 tiles (at least one per CTA pair), ragged
    # in M and with range boundaries inside tiles and inside 128-column halves.
    wl = synth.LinearWorkload("fused_wide", 2341, 1088, 8288, seed=23)  # columns 8256.. in no range
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert F.nvfp4_gemm_tile_shape(wl.m, wl.n, sms) == (2, 256, 1)
    rows = np.unique(np.r_[np.random.default_rng(23).choice(wl.m, 40, replace=False), wl.m - 1, 255, 256])
    _check_fused(F, wl, (0, 1600), (1600, 4160), (4160, 8256), rows=rows)


def test_fused_identity_range_bit_exact_when_accumulation_is_exact(F):
    rng = np.random.default_rng(22)
    M, N, K = 130, 256, 256
    pow2 = np.array([0x30, 0x38, 0x40], np.uint8)
    a_codes = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    b_codes = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    a_sf, b_sf = rng.choice(pow2, (M, K // 16)), rng.choice(pow2, (N, K // 16))
    a = F.NVFP4Tensor(torch.from_numpy(a_codes).cuda(), torch.from_numpy(O.swizzle_sf(a_sf)).cuda(), 1.0, M, K)
    b = F.NVFP4Tensor(torch.from_numpy(b_codes).cuda(), torch.from_numpy(O.swizzle_sf(b_sf)).cuda(), 1.0, N, K)
    nxt = _empty_nvfp4(F, M, N)
    g_next = 0.037
    F.gemm_quant(a, b, [(0, N, F.ACT_NONE, F.DST_NVFP4, 0)], alpha=0.25, g_next=g_next, next_out=nxt)
    torch.cuda.synchronize()
    y_ref = O.gemm_ref(a_codes, a_sf, 1.0, b_codes, b_sf, 1.0) * 0.25   # exact in fp32
    v = O.round_to_bf16(y_ref).astype(np.float32)
    codes, sf = O.quantize_nvfp4(v, g_next)
    assert_bytes_equal(gpu_bytes(nxt.codes), codes, "codes")
    assert_bytes_equal(gpu_bytes(nxt.sf), O.swizzle_sf(sf), "scales")


def test_fused_rejects_bad_ranges(F):
    wl = synth.LinearWorkload("bad", 128, 256, 256, seed=1)
    _, _, _, xq, wq = _layer(F, wl)
    nxt = _empty_nvfp4(F, 128, 256)
    for bad in ([(0, 100, 0, 1, 0)], [(0, 128, 0, 1, 0), (64, 192, 0, 1, 128)], [(0, 128, 5, 1, 0)],
                [(0, 320, 0, 1, 0)], [(0, 256, 0, 1, 64)]):
        with pytest.raises(F.NVFP4Error) as e:
            F.gemm_quant(xq, wq, bad, g_next=0.1, next_out=nxt)
        assert e.value.status == F.NVFP4_EINVAL


def test_no_kernel_reported_a_fault(F):
    F.nvfp4_check_fault()
