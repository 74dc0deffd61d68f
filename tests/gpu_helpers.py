"""Shared helpers of the GPU parity tests: move synthetic inputs to the GPU,
run the oracle on the same inputs, compare."""
import numpy as np
import torch

import oracle as O


def require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device (B200, sm_100a)"
    major, minor = torch.cuda.get_device_capability()
    assert (major, minor) == (10, 0), f"need compute capability 10.0, got {major}.{minor}"


def f32(x_bf16: torch.Tensor) -> np.ndarray:
    """bf16 CPU tensor -> exact float32 numpy array."""
    return x_bf16.float().numpy()


def oracle_quant(x_bf16: torch.Tensor, g: float):
    """Oracle codes [M, K/2] and swizzled scales for bf16 x."""
    codes, sf = O.quantize_nvfp4(f32(x_bf16), np.float32(g))
    return codes, O.swizzle_sf(sf), sf


def gpu_bytes(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def assert_bytes_equal(got: np.ndarray, want: np.ndarray, what: str):
    got = np.asarray(got).reshape(-1)
    want = np.asarray(want).reshape(-1)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{what}: {bad.size} bytes differ, first at {bad[:8]}: got {got[bad[:8]]} want {want[bad[:8]]}"


def assert_within_tol(y_gpu: np.ndarray, y_ref: np.ndarray, tol: np.ndarray, what: str):
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, (f"{what}: {len(bad)} of {err.size} outside tolerance; first {bad[:5].tolist()}: "
                           f"got {y_gpu[tuple(bad[0])]} want {y_ref[tuple(bad[0])]} tol {tol[tuple(bad[0])]}")


def single_stream_scales() -> dict:
    """Per-tensor scales of the FLUX single-stream block pair, written by
    tests/golden/make_golden.py from the oracle alone: the output
    projection's calibrated input scale is ``g_next``."""
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "single_stream_pair.json")
    with open(path) as f:
        return json.load(f)
