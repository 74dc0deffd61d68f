"""GPU parity of the fused epilogue: GEMM -> (GELU-tanh) -> the next layer's
NVFP4 activations, plus bf16 column ranges, and the FLUX single-stream block
pair that chains it into the output projection (K = 15360).

The GEMM itself is only defined to a tolerance, so several bf16 results are
correct and the fused NVFP4 bytes are checked against what is unique given
them: the oracle's quantizer (steps 4-7 of the method) applied to the kernel's
own bf16 epilogue values, read back from a debug run of the same kernel with
every range sent to bf16 -- bit for bit.  The rest is checked for validity
against the oracle: the bf16 ranges and the pre-quantization values lie within
the GEMM tolerance of the oracle's fp64 epilogue, the dequantized fused output
within that tolerance plus one quantization step, and in an
exactly-accumulated case the identity range matches the oracle's bytes bit for
bit with no GPU value involved.  The output projection of the pair is checked
against the oracle's GEMM of those (oracle-checked) fused bytes with the
oracle-quantized weight.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from tests.gpu_helpers import (assert_bytes_equal, assert_within_tol, f32, gpu_bytes, require_gpu,
                               single_stream_scales)

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


def _fused_vs_references(F, wl, q_rng, bf_rng, act_rng, g_next):
    """Run ranges: q_rng -> NVFP4 identity at dst 0; bf_rng -> bf16; act_rng
    -> GELU -> NVFP4 after q; then the same kernel with every NVFP4 range sent
    to bf16 (the kernel's own pre-quantization values).  Returns everything
    needed to compare, the device tensors still on the GPU."""
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
    # debug run: the same kernel with every range sent to bf16
    all_bf = torch.zeros(wl.m, k_next, dtype=torch.bfloat16, device="cuda")
    F.gemm_quant(xq, wq, [(q_rng[0], q_rng[1], F.ACT_NONE, F.DST_BF16, 0),
                          (act_rng[0], act_rng[1], F.ACT_GELU_TANH, F.DST_BF16, q_w)],
                 bias=bias, y_bf16=all_bf)
    torch.cuda.synchronize()
    return dict(x=x, w=w, b=b, xq=xq, wq=wq, nxt=nxt, ybf=ybf, all_bf=all_bf, k_next=k_next)


def _check_fused_bytes_against_oracle(nxt, all_bf_rows, g_next, rows, m, k_next):
    """The fused NVFP4 codes and scales of ``rows`` equal the oracle's quantizer
    applied to the kernel's own bf16 values of those rows (bit for bit)."""
    codes_ref, sf_ref = O.quantize_nvfp4(all_bf_rows, np.float32(g_next))
    assert_bytes_equal(gpu_bytes(nxt.codes)[rows], codes_ref, "fused codes vs oracle")
    sf_gpu = O.unswizzle_sf(gpu_bytes(nxt.sf), m, k_next)[rows]
    assert_bytes_equal(sf_gpu, sf_ref, "fused scales vs oracle")
    return codes_ref, sf_ref


def _check_fused(F, wl, q_rng, bf_rng, act_rng, rows, g_next=0.01, run=None):
    r = run if run is not None else _fused_vs_references(F, wl, q_rng, bf_rng, act_rng, g_next)
    x, w, b, nxt, ybf, all_bf, k_next = r["x"], r["w"], r["b"], r["nxt"], r["ybf"], r["all_bf"], r["k_next"]
    m = wl.m
    all_np = all_bf.float().cpu().numpy()
    # (1) fused bytes == the oracle's quantizer on the kernel's own bf16 values
    _check_fused_bytes_against_oracle(nxt, all_np[rows], g_next, rows, m, k_next)
    if len(rows) == m:  # every row: the whole swizzled buffer, padding included
        _, sf_all = O.quantize_nvfp4(all_np, np.float32(g_next))
        assert_bytes_equal(gpu_bytes(nxt.sf), O.swizzle_sf(sf_all), "fused swizzled scale buffer vs oracle")

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
    assert_within_tol(all_np[rows], ep_ref, ep_tol, "epilogue values")
    # (4) dequantized fused NVFP4 output vs the oracle epilogue, within the
    # tolerance plus one quantization step of the block
    codes = gpu_bytes(nxt.codes)[rows]
    sf_lin = O.unswizzle_sf(gpu_bytes(nxt.sf), m, k_next)[rows]
    deq = O.dequantize(codes, sf_lin, g_next)
    step = (O.e4m3_decode(sf_lin) * g_next).repeat(16, axis=1)
    assert_within_tol(deq, ep_ref, ep_tol + 1.01 * step, "dequantized fused output")
    # (5) scale padding rows are zero
    sf_all = gpu_bytes(nxt.sf)
    mp = (m + 127) // 128 * 128
    if mp > m:
        rr, cc = np.meshgrid(np.arange(m, mp), np.arange(k_next // 16), indexing="ij")
        assert np.all(sf_all[O.sf_offset(rr, cc, k_next // 16)] == 0)


def test_fused_small(F):
    wl = synth.LinearWorkload("fused_small", 200, 256, 640, seed=21)
    _check_fused(F, wl, (0, 128), (128, 384), (384, 640), rows=np.arange(200))


@pytest.fixture(scope="module")
def single_stream(F):
    """The FLUX single-stream block pair on the GPU, run once: GEMM1 (fused
    QKV+MLP-in: Q -> NVFP4, K/V -> bf16, MLP -> GELU-tanh -> NVFP4) writing the
    output projection's NVFP4 input with its calibrated scale, the debug run of
    GEMM1 with every range in bf16, and GEMM2 (the output projection, K =
    15360) on the fused output."""
    wl, w2l = synth.SINGLE_IN, synth.SINGLE_OUT
    g_next = single_stream_scales()["g_next"]
    r = _fused_vs_references(F, wl, synth.SINGLE_Q, synth.SINGLE_KV, synth.SINGLE_MLP, g_next)
    w2 = w2l.weight()
    w2d = w2.cuda()
    w2q = F.quantize(w2d, F.global_scale(w2d))
    b2 = w2l.bias_vec()
    y2 = F.gemm(r["nxt"], w2q, bias=b2.cuda())
    torch.cuda.synchronize()
    r.update(w2=w2, w2q=w2q, b2=b2, y2=y2.float().cpu().numpy(), g_next=g_next)
    return r


def test_fused_single_stream_block_shape_sampled(F, single_stream):
    # FLUX single-stream fused QKV+MLP-in GEMM: Q -> NVFP4, K/V -> bf16,
    # MLP -> GELU-tanh -> NVFP4, together the output projection's input, with
    # that projection's calibrated input scale.
    wl = synth.SINGLE_IN
    rows = np.sort(np.random.default_rng(3).choice(wl.m, 48, replace=False))
    rows = np.unique(np.r_[rows, wl.m - 1])
    _check_fused(F, wl, synth.SINGLE_Q, synth.SINGLE_KV, synth.SINGLE_MLP, rows=rows,
                 g_next=single_stream["g_next"], run=single_stream)


def test_single_stream_pair_output_projection_sampled(F, single_stream):
    # GEMM2 of the pair, [4608, 15360] x [3072, 15360]^T + bias: its A is the
    # fused output of GEMM1 (the oracle's quantizer of the kernel's own bf16
    # values, checked bit for bit here), its B the weight the GPU quantized
    # (checked bit for bit against the oracle's weight preparation).
    r = single_stream
    w2l = synth.SINGLE_OUT
    m, k2, g_next = w2l.m, w2l.k, r["g_next"]
    w2f = f32(r["w2"])
    gw2 = O.global_scale(O.tensor_amax(w2f))
    assert np.float32(r["w2q"].g) == gw2 == np.float32(single_stream_scales()["g_w2"])
    w2c, w2s = O.quantize_nvfp4(w2f, gw2)
    assert_bytes_equal(gpu_bytes(r["w2q"].codes), w2c, "W2 codes")
    assert_bytes_equal(gpu_bytes(r["w2q"].sf), O.swizzle_sf(w2s), "W2 scales")
    all_np = r["all_bf"].float().cpu().numpy()
    b2 = r["b2"].float().numpy()
    rng = np.random.default_rng(33)
    rows = np.unique(np.r_[rng.choice(m, 48, replace=False), m - 1, 255, 256])
    a2c, a2s = _check_fused_bytes_against_oracle(r["nxt"], all_np[rows], g_next, rows, m, k2)
    y_ref = O.gemm_ref(a2c, a2s, g_next, w2c, w2s, gw2, b2)
    tol = O.gemm_tolerance(a2c, a2s, g_next, w2c, w2s, gw2, y_ref)
    assert_within_tol(r["y2"][rows], y_ref, tol, "output projection rows")
    # every row of sampled columns (the last ones and the 128 / 256 edges)
    cols = np.unique(np.r_[rng.choice(w2l.n, 40, replace=False), w2l.n - 1, 127, 128, 255, 256])
    a2c_all, a2s_all = O.quantize_nvfp4(all_np, np.float32(g_next))
    assert_bytes_equal(gpu_bytes(r["nxt"].codes), a2c_all, "fused codes (all rows) vs oracle")
    y_ref = O.gemm_ref(a2c_all, a2s_all, g_next, w2c[cols], w2s[cols], gw2, b2[cols])
    tol = O.gemm_tolerance(a2c_all, a2s_all, g_next, w2c[cols], w2s[cols], gw2, y_ref)
    assert_within_tol(r["y2"][:, cols], y_ref, tol, "output projection columns")


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
