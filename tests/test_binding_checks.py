"""The torch helpers of the binding check every caller-supplied tensor before
its raw pointer reaches the library: dtype, contiguity, the current device,
and enough elements for what the kernel reads or writes.  Run on the CPU
with stand-in CUDA tensors and the C entry points replaced by recorders, so
no kernel is launched: well-formed buffers (the shapes the helpers allocate
themselves) go through, malformed ones raise before the call."""
import pytest
import torch

import nvfp4_block_scaled_12_b200 as F


class _FakeCuda(torch.Tensor):
    """A CPU tensor that reports itself as living on cuda:<_dev>."""
    _dev = 0

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return torch.device("cuda", self._dev)


def cu(t, dev=0):
    f = t.as_subclass(_FakeCuda)
    f._dev = dev
    return f


def empty(*shape, dtype=torch.uint8, dev=0):
    return cu(torch.zeros(*shape, dtype=dtype), dev)


@pytest.fixture
def calls(monkeypatch):
    rec = []
    for name in ("nvfp4_quantize", "nvfp4_quantize_dynamic", "nvfp4_gemm", "nvfp4_gemm_dynamic",
                 "nvfp4_gemm_scaled", "nvfp4_gemm_quant_scaled", "nvfp4_gemm_quant", "nvfp4_mxfp8_quantize", "nvfp4_mxfp8_gemm", "nvfp4_fp8row_quantize",
                 "nvfp4_fp8row_gemm", "nvfp4_dequantize", "nvfp4_gemm_amax", "nvfp4_quantize_from_amax"):
        monkeypatch.setattr(F, name, lambda *a, _n=name: rec.append(_n))
    monkeypatch.setattr(F, "_stream", lambda stream: 0)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    return rec


def nvfp4(rows, k, g=1.0, dev=0):
    return F.NVFP4Tensor(empty(rows, k // 2, dev=dev), empty(F.nvfp4_sf_bytes(rows, k), dev=dev), g, rows, k)


def test_well_formed_buffers_reach_the_library(calls):
    M, N, K = 130, 192, 256
    x = empty(M, K, dtype=torch.bfloat16)
    a, b = nvfp4(M, K), nvfp4(N, K)
    F.quantize(x, 0.5, out=a)
    y = empty(M, N, dtype=torch.bfloat16)
    F.gemm(a, b, bias=empty(N, dtype=torch.bfloat16), y=y)
    d = F.NVFP4Tensor(empty(M, K // 2), empty(F.nvfp4_sf_bytes(M, K)), None, M, K, empty(2, dtype=torch.float32))
    F.quantize_dynamic(x, out=d, workspace=empty(F.NVFP4_DYNAMIC_WORKSPACE_BYTES))
    F.gemm(d, b, y=y)                                   # the device-scale path
    nxt = nvfp4(M, 128)
    F.gemm_quant(a, b, [(0, 128, F.ACT_NONE, F.DST_NVFP4, 0), (128, 192, F.ACT_NONE, F.DST_BF16, 0)],
                 y_bf16=empty(M, 64, dtype=torch.bfloat16), g_next=0.1, next_out=nxt)
    F.dequantize(b, out=empty(N, K, dtype=torch.bfloat16))
    m8 = F.MXFP8Tensor(empty(M, K), empty(F.nvfp4_mxfp8_sf_bytes(M, K)), M, K)
    w8 = F.MXFP8Tensor(empty(N, K), empty(F.nvfp4_mxfp8_sf_bytes(N, K)), N, K)
    F.quantize_mxfp8(x, out=m8)
    F.gemm_mxfp8(m8, w8, y=y)
    r8 = F.FP8RowTensor(empty(M, K), empty(M, dtype=torch.float32), M, K)
    rw = F.FP8RowTensor(empty(N, K), empty(N, dtype=torch.float32), N, K)
    F.quantize_fp8row(x, out=r8)
    F.gemm_fp8row(r8, rw, y=y)
    assert calls == ["nvfp4_quantize", "nvfp4_gemm_scaled", "nvfp4_quantize_dynamic", "nvfp4_gemm_dynamic",
                     "nvfp4_gemm_quant_scaled", "nvfp4_dequantize", "nvfp4_mxfp8_quantize", "nvfp4_mxfp8_gemm",
                     "nvfp4_fp8row_quantize", "nvfp4_fp8row_gemm"]


def test_malformed_outputs_are_rejected_before_the_call(calls):
    M, N, K = 130, 192, 256
    x = empty(M, K, dtype=torch.bfloat16)
    a, b = nvfp4(M, K), nvfp4(N, K)
    short = F.NVFP4Tensor(empty(M, K // 2 - 1), a.sf, 1.0, M, K)
    with pytest.raises(ValueError):
        F.quantize(x, 0.5, out=short)                     # codes one byte short per row
    with pytest.raises(ValueError):
        F.quantize(x, 0.5, out=nvfp4(M - 1, K))           # another shape
    with pytest.raises(TypeError):
        F.quantize(x, 0.5, out=F.NVFP4Tensor(a.codes, empty(a.sf.numel(), dtype=torch.int8), 1.0, M, K))
    strided = cu(torch.zeros(M, K, dtype=torch.uint8)[:, ::2])
    with pytest.raises(ValueError):
        F.quantize(x, 0.5, out=F.NVFP4Tensor(strided, a.sf, 1.0, M, K))   # not contiguous
    with pytest.raises(ValueError):
        F.quantize(x, 0.5, out=nvfp4(M, K, dev=1))        # not on the current device
    with pytest.raises(ValueError):
        F.gemm(a, b, y=empty(N, M, dtype=torch.bfloat16))  # transposed output
    with pytest.raises(ValueError):
        F.gemm(a, F.NVFP4Tensor(b.codes, empty(10), 1.0, N, K))   # B scales too short
    with pytest.raises(ValueError):
        F.gemm(a, nvfp4(N, K, g=None))                    # no host scale for the weight
    with pytest.raises(ValueError):
        F.gemm_quant(a, b, [(0, 128, F.ACT_NONE, F.DST_NVFP4, 0)], g_next=0.1, next_out=nvfp4(M - 2, 128))
    with pytest.raises(ValueError):
        F.gemm_quant(a, b, [(0, 64, F.ACT_NONE, F.DST_BF16, 0)], y_bf16=empty(M - 1, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        F.dequantize(b, out=empty(N, K - 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        F.quantize_mxfp8(x, out=F.MXFP8Tensor(empty(M, K // 2), empty(F.nvfp4_mxfp8_sf_bytes(M, K)), M, K))
    with pytest.raises(ValueError):
        F.quantize_fp8row(x, out=F.FP8RowTensor(empty(M, K), empty(M - 1, dtype=torch.float32), M, K))
    with pytest.raises(ValueError):
        F.gemm_fp8row(F.FP8RowTensor(empty(M, K), empty(M, dtype=torch.float32), M, K),
                      F.FP8RowTensor(empty(N, K), empty(N, dtype=torch.float32), N, K),
                      y=empty(M, N - 8, dtype=torch.bfloat16))
    assert calls == []


def test_amax_helpers_check_their_buffers(calls):
    M, N, K = 130, 192, 256
    x = empty(M, K, dtype=torch.bfloat16)
    a, b = nvfp4(M, K), nvfp4(N, K)
    amax = empty(1, dtype=torch.float32)
    y = empty(M, N, dtype=torch.bfloat16)
    d = F.NVFP4Tensor(empty(M, K // 2), empty(F.nvfp4_sf_bytes(M, K)), None, M, K, empty(2, dtype=torch.float32))
    F.gemm(a, b, y=y, amax_out=amax)
    F.gemm(a, b, alpha=0.5, y=y, amax_out=amax)
    F.quantize_from_amax(x, amax, out=d)
    assert calls == ["nvfp4_gemm_amax", "nvfp4_gemm_amax", "nvfp4_quantize_from_amax"]
    with pytest.raises((TypeError, ValueError)):
        F.gemm(a, b, y=y, amax_out=empty(1, dtype=torch.float16))
    with pytest.raises((TypeError, ValueError)):
        F.quantize_from_amax(x, empty(1, dtype=torch.int32), out=d)
    with pytest.raises((TypeError, ValueError)):
        F.quantize_from_amax(x, amax, out=F.NVFP4Tensor(empty(M, K // 2), empty(F.nvfp4_sf_bytes(M, K)), None,
                                                        M, K, empty(1, dtype=torch.float32)))
