"""The failure path on the GPU, made to happen without a fault: the dynamic
quantize's grid-wide wait is given a short limit and one arrival that never
comes, so every CTA gives up.  The kernel must return, write none of its
outputs, and leave NVFP4_ETIMEOUT in the device fault word; the context stays
usable and the next call with the normal settings is bit-exact against the
oracle.  (No barrier is removed and nothing faults: the wait is the library's
own bounded wait, run out on purpose.)
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from tests.gpu_helpers import assert_bytes_equal, f32, gpu_bytes, require_gpu

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture(scope="module")
def F():
    require_gpu()
    import nvfp4_block_scaled_12_b200 as F
    return F


def _outputs(M, K, F):
    codes = torch.full((M, K // 2), 0x5A, dtype=torch.uint8, device="cuda")
    sf = torch.full((F.nvfp4_sf_bytes(M, K),), 0xA5, dtype=torch.uint8, device="cuda")
    scale = torch.full((2,), -7.0, dtype=torch.float32, device="cuda")
    return codes, sf, scale


def _call(F, which, x, codes, sf, scale, ws):
    M, K = x.shape
    stream = torch.cuda.current_stream().cuda_stream
    if which == "workspace":
        F.nvfp4_quantize_dynamic(x.data_ptr(), M, K, codes.data_ptr(), sf.data_ptr(), scale.data_ptr(),
                                 ws.data_ptr(), ws.numel(), stream)
    else:
        F.nvfp4_quantize_dynamic_noalloc(x.data_ptr(), M, K, codes.data_ptr(), sf.data_ptr(), scale.data_ptr(),
                                         stream)


@pytest.mark.parametrize("which", ["workspace", "noalloc"])
def test_grid_wait_times_out_then_the_next_call_is_exact(F, which):
    x = synth.laplace_activations(1000, 3072, seed=71).cuda()
    M, K = x.shape
    ws = torch.empty(F.NVFP4_DYNAMIC_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    F.nvfp4_check_fault()  # nothing pending from earlier work
    codes, sf, scale = _outputs(M, K, F)
    F.nvfp4_testing_set_grid_wait(LIMIT_NS, 1)
    try:
        _call(F, which, x, codes, sf, scale, ws)
    finally:
        F.nvfp4_testing_set_grid_wait(0, 0)
    with pytest.raises(F.NVFP4Error) as e:
        F.nvfp4_check_fault()  # synchronizes: the kernel returned
    assert e.value.status == F.NVFP4_ETIMEOUT
    F.nvfp4_check_fault()  # read and cleared
    # nothing was written
    assert torch.all(codes == 0x5A) and torch.all(sf == 0xA5) and torch.all(scale == -7.0)
    # the next call, with the normal settings, is exact
    _call(F, which, x, codes, sf, scale, ws)
    torch.cuda.synchronize()
    F.nvfp4_check_fault()
    c_ref, s_ref, amax, g = O.quantize_dynamic(f32(x.cpu()))
    assert_bytes_equal(gpu_bytes(codes), c_ref, "codes after the time-out")
    assert_bytes_equal(gpu_bytes(sf), O.swizzle_sf(s_ref), "scales after the time-out")
    assert np.array_equal(scale.cpu().numpy(), np.array([amax, g], np.float32))


def test_other_entry_points_still_work_after_a_time_out(F):
    # a static quantize and a GEMM on the same context, exact vs the oracle
    wl = synth.TINY
    x = wl.activations()
    g = O.global_scale(O.tensor_amax(f32(x)))
    xq = F.quantize(x.cuda(), float(g))
    torch.cuda.synchronize()
    c_ref, s_ref = O.quantize_nvfp4(f32(x), g)
    assert_bytes_equal(gpu_bytes(xq.codes), c_ref, "codes")
    assert_bytes_equal(gpu_bytes(xq.sf), O.swizzle_sf(s_ref), "scales")
    F.nvfp4_check_fault()
