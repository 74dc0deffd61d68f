"""GPU parity of the activation quantizer, the scale swizzle and the
calibration against the oracle: bit-exact on every byte.

The quantizer is NVFP4's runtime activation quantization ("BFL (fp8r /
nvfp4)" diffusers doc, section "Kernels": `nvfp4_quantize`).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from tests.gpu_helpers import assert_bytes_equal, f32, gpu_bytes, oracle_quant, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    require_gpu()
    import nvfp4_block_scaled_12_b200 as F
    return F


def _check_quant(F, x_bf16: torch.Tensor, g: float, what: str):
    xq = F.quantize(x_bf16.cuda(), g)
    torch.cuda.synchronize()
    codes, sf_swz, _ = oracle_quant(x_bf16, g)
    assert_bytes_equal(gpu_bytes(xq.codes), codes, what + " codes")
    assert_bytes_equal(gpu_bytes(xq.sf), sf_swz, what + " scales")


def test_every_bf16_value_in_range_with_unit_scale(F):
    # Blocks [6, v1..v15] with g = 1: the block scale is exactly 1.0, so every
    # element is encoded as E2M1(v) -- all bf16 values in [-6, 6].
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= 6.0)]
    n_blk = (v.size + 14) // 15
    vals = np.zeros(n_blk * 15, np.float32)
    vals[:v.size] = v
    blocks = np.concatenate([np.full((n_blk, 1), 6.0, np.float32), vals.reshape(n_blk, 15)], axis=1)
    rows = (n_blk + 3) // 4
    x = np.zeros((rows * 4, 16), np.float32)
    x[:n_blk] = blocks
    x = torch.from_numpy(x.reshape(rows, 64)).to(torch.bfloat16)
    _check_quant(F, x, 1.0, "all-bf16 unit-scale")


@pytest.mark.parametrize("g", [2.0 ** -3, 0.0123, 1e-5, 37.0])
def test_every_bf16_amax_gives_the_oracle_scale(F, g):
    # One block per positive finite bf16 value used as the block amax.
    bits = (np.arange(1, 0x7F80, dtype=np.uint32) << 16)
    amax = bits.view(np.float32)
    rng = np.random.default_rng(int(g * 1e6) % 1000)
    frac = rng.uniform(-1, 1, (amax.size, 16)).astype(np.float32)
    blocks = O.round_to_bf16((frac * amax[:, None]).astype(np.float64)).astype(np.float32)
    blocks[np.arange(amax.size), rng.integers(0, 16, amax.size)] = amax
    pad = (-amax.size) % 4
    blocks = np.concatenate([blocks, np.zeros((pad, 16), np.float32)])
    x = torch.from_numpy(blocks.reshape(-1, 64)).to(torch.bfloat16)
    _check_quant(F, x, g, f"all-amax g={g}")


def test_tiny_workload(F):
    x = synth.TINY.activations()
    g = float(O.global_scale(O.tensor_amax(f32(x))))
    _check_quant(F, x, g, "tiny")


@pytest.mark.parametrize("m,k", [(1, 64), (7, 192), (127, 320), (129, 64), (300, 4160), (256, 128)])
def test_ragged_shapes_including_scale_padding(F, m, k):
    x = synth.activations_with_outlier_channels(m, k, seed=m * 31 + k)
    g = float(O.global_scale(O.tensor_amax(f32(x))))
    _check_quant(F, x, g, f"ragged {m}x{k}")


def test_laplace_quantize_workload_medium(F):
    x = synth.laplace_activations(512, synth.QUANT_K, seed=synth.QUANT_SEED)
    g = float(O.global_scale(O.tensor_amax(f32(x))))
    _check_quant(F, x, g, "laplace 512x12288")


def test_laplace_quantize_workload_full_size_sampled_rows(F):
    # The benchmarked quantize shape [4608, 12288]; the oracle checks a seeded
    # sample of 128-row blocks (rows are independent) and all scale padding.
    x = synth.quantize_input()
    M, K = x.shape
    g = float(O.global_scale(O.tensor_amax(f32(x))))
    xq = F.quantize(x.cuda(), g)
    torch.cuda.synchronize()
    codes_gpu = gpu_bytes(xq.codes)
    sf_gpu = gpu_bytes(xq.sf)
    rng = np.random.default_rng(0)
    blocks = sorted(set([0, M // 128 - 1] + rng.choice(M // 128, 4, replace=False).tolist()))
    katoms = K // 64
    for b in blocks:
        rows = slice(b * 128, (b + 1) * 128)
        codes, sf_swz, _ = oracle_quant(x[rows], g)
        assert_bytes_equal(codes_gpu[rows], codes, f"block {b} codes")
        assert_bytes_equal(sf_gpu[b * katoms * 512:(b + 1) * katoms * 512], sf_swz, f"block {b} scales")


def test_special_blocks(F):
    x = np.zeros((4, 128), np.float32)
    x[0, 0:16] = 0.0                       # zero block
    x[0, 16:32] = -0.0                     # negative zeros only
    x[0, 32:48] = np.linspace(-3, 3, 16)
    x[0, 33] = -0.0                        # -0 inside a live block -> code 0x8
    x[1, :16] = 1e30                       # saturating scale
    x[1, 16:32] = 1e-30                    # scale underflow
    x[2, :] = np.linspace(-1e4, 1e4, 128)
    x[3, :] = -np.logspace(-8, 4, 128)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    for g in (1.0, 2.0 ** -64, 2.0 ** 64, 3.7e-3):
        _check_quant(F, xb, g, f"special g={g}")


@pytest.mark.parametrize("m,k", [(4700, 12288), (4609, 15360), (4608, 12352)])
def test_large_ragged_quantize_stays_inside_its_buffers(F, m, k):
    # Shapes that take the 256-row tiles with M not a multiple of 256 (nor,
    # for two of them, of 128): the last tile reaches past the scale buffer's
    # padded rows, and must write neither codes nor scales there.  Both outputs
    # sit inside larger buffers whose tails must stay untouched; sampled rows
    # (the last ones included) are bit-exact and the padding rows are zero.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert F.nvfp4_quantize_tile_rows(m, k, sms) == 256
    rng = np.random.default_rng(m + k)
    x = synth.normal_bf16((m, k), 1.0, synth._gen(m + k))
    g = float(O.global_scale(O.tensor_amax(f32(x))))
    guard = 1 << 16
    sf_bytes = F.nvfp4_sf_bytes(m, k)
    codes_buf = torch.full((m * k // 2 + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    sf_buf = torch.full((sf_bytes + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    xd = x.cuda()
    F.nvfp4_quantize(xd.data_ptr(), m, k, g, codes_buf.data_ptr(), sf_buf.data_ptr(),
                     torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    F.nvfp4_check_fault()
    assert torch.all(codes_buf[m * k // 2:] == 0xA5), "codes written past the buffer"
    assert torch.all(sf_buf[sf_bytes:] == 0xA5), "scales written past the buffer"
    rows = np.unique(np.r_[rng.choice(m, 48, replace=False), m - 1, m - 2, 4607, 4608])
    rows = rows[rows < m]
    xf = f32(x)[rows]
    codes, sf = O.quantize_nvfp4(xf, np.float32(g))
    got_codes = codes_buf[: m * k // 2].view(m, k // 2).cpu().numpy()[rows]
    assert_bytes_equal(got_codes, codes, "codes")
    sf_all = sf_buf[:sf_bytes].cpu().numpy()
    r, c = np.meshgrid(rows, np.arange(k // 16), indexing="ij")
    assert_bytes_equal(sf_all[O.sf_offset(r, c, k // 16)], sf, "scales")
    mp = (m + 127) // 128 * 128
    if mp > m:
        r, c = np.meshgrid(np.arange(m, mp), np.arange(k // 16), indexing="ij")
        assert np.all(sf_all[O.sf_offset(r, c, k // 16)] == 0), "scale padding rows"


def test_quantize_is_deterministic(F):
    x = synth.laplace_activations(384, 3072, seed=77).cuda()
    a = F.quantize(x, 0.01)
    b = F.quantize(x, 0.01)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes) and torch.equal(a.sf, b.sf)


def test_quantize_is_deterministic_when_every_stage_is_reused(F):
    # [4608, 15360] is 8640 tiles of 128 x 64: every CTA cycles its stage
    # ring several times, so a shared-memory read that raced the refill of
    # its stage would show up as run-to-run differences.  Sampled rows are
    # also checked against the oracle.
    x = synth.laplace_activations(4608, 15360, seed=78).cuda()
    g = 0.0137
    first = F.quantize(x, g)
    for _ in range(12):
        again = F.quantize(x, g)
        torch.cuda.synchronize()
        assert torch.equal(first.codes, again.codes) and torch.equal(first.sf, again.sf)
    rows = np.sort(np.random.default_rng(5).choice(4608, 48, replace=False))
    codes, _, sf_ref = oracle_quant(x[torch.from_numpy(rows).cuda()].cpu(), g)
    got_codes = gpu_bytes(first.codes).reshape(4608, -1)[rows]
    assert_bytes_equal(got_codes, codes, "stage-reuse codes")
    sf_lin = O.unswizzle_sf(gpu_bytes(first.sf), 4608, 15360)
    assert_bytes_equal(sf_lin[rows], sf_ref, "stage-reuse scales")


@pytest.mark.parametrize("rows,k", [(1, 64), (128, 256), (300, 3072), (4608, 3072)])
def test_swizzle_sf_matches_oracle(F, rows, k):
    rng = np.random.default_rng(rows + k)
    sf = rng.integers(0, 127, (rows, k // 16)).astype(np.uint8)
    got = F.swizzle_sf(torch.from_numpy(sf).cuda(), rows, k)
    torch.cuda.synchronize()
    assert_bytes_equal(gpu_bytes(got), O.swizzle_sf(sf), f"swizzle {rows}x{k}")


@pytest.mark.parametrize("shape", [(128, 256), (4608, 3072), (3, 8)])
def test_calibrate_matches_oracle_global_scale(F, shape):
    x = synth.activations_with_outlier_channels(*shape, seed=5)
    out = F.calibrate(x.cuda()).cpu().numpy()
    amax = O.tensor_amax(f32(x))
    assert out[0] == amax
    assert out[1] == O.global_scale(amax)


def test_no_kernel_reported_a_fault(F):
    F.nvfp4_check_fault()
