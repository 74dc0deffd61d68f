"""The no-allocation dynamic quantize, nvfp4_quantize_dynamic_noalloc, against
the workspace entry point nvfp4_quantize_dynamic and against the oracle, all
called through the C ABI with raw device pointers.  Two calls in a row (on
tensors with different scales, so the shared scratch must be re-zeroed by each
call) must give the same codes, scales, amax and g as the workspace path, and
both must equal the oracle's dynamic quantize bit for bit.  This file sorts
last so that it also runs after every other GPU test in one session; it passes
alone as well.
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


def _buffers(F, M, K):
    codes = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sf = torch.empty(F.nvfp4_sf_bytes(M, K), dtype=torch.uint8, device="cuda")
    scale = torch.empty(2, dtype=torch.float32, device="cuda")
    return codes, sf, scale


def _with_workspace(F, x):
    M, K = x.shape
    codes, sf, scale = _buffers(F, M, K)
    ws = torch.empty(F.NVFP4_DYNAMIC_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    F.nvfp4_quantize_dynamic(x.data_ptr(), M, K, codes.data_ptr(), sf.data_ptr(), scale.data_ptr(),
                             ws.data_ptr(), ws.numel(), stream)
    return codes, sf, scale


def _no_alloc(F, x):
    M, K = x.shape
    codes, sf, scale = _buffers(F, M, K)
    stream = torch.cuda.current_stream().cuda_stream
    F.nvfp4_quantize_dynamic_noalloc(x.data_ptr(), M, K, codes.data_ptr(), sf.data_ptr(), scale.data_ptr(), stream)
    return codes, sf, scale


def test_no_alloc_matches_the_workspace_entry_point_twice_in_a_row(F):
    x1 = synth.laplace_activations(1000, 3072, seed=61).cuda()      # more tiles than SMs
    x2 = (synth.activations_with_outlier_channels(300, 4160, seed=62) * 7).cuda()
    for x in (x1, x2):
        want = _with_workspace(F, x)
        got = _no_alloc(F, x)
        torch.cuda.synchronize()
        # quantized bytes are exact; amax and g are exact floats
        assert_bytes_equal(gpu_bytes(got[0]), gpu_bytes(want[0]), "no-alloc codes")
        assert_bytes_equal(gpu_bytes(got[1]), gpu_bytes(want[1]), "no-alloc scales")
        assert np.array_equal(got[2].cpu().numpy(), want[2].cpu().numpy())
        # and the oracle's dynamic quantize of the same bf16 values
        codes, sf, amax, g = O.quantize_dynamic(f32(x.cpu()))
        assert_bytes_equal(gpu_bytes(got[0]), codes, "no-alloc codes vs oracle")
        assert_bytes_equal(gpu_bytes(got[1]), O.swizzle_sf(sf), "no-alloc scales vs oracle")
        assert np.array_equal(got[2].cpu().numpy(), np.array([amax, g], np.float32))
    F.nvfp4_check_fault()


def test_no_alloc_rejects_bad_arguments_before_touching_the_device(F):
    P = 1 << 20
    with pytest.raises(F.NVFP4Error) as e:
        F.nvfp4_quantize_dynamic_noalloc(P, 4, 96, P, P, P, 0)
    assert e.value.status == F.NVFP4_EINVAL
    with pytest.raises(F.NVFP4Error) as e:
        F.nvfp4_quantize_dynamic_noalloc(P, 4, 64, P, P, 0, 0)
    assert e.value.status == F.NVFP4_EINVAL
