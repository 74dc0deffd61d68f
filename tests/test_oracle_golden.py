"""The oracle against the stated format facts and its own regression fixture."""
import hashlib
import json
import os

import numpy as np

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _facts():
    out = {}
    with open(os.path.join(GOLDEN, "nvfp4_format_facts.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            kv, _cite = line.split("|", 1)
            k, v = kv.split("=")
            out[k.strip()] = v.strip()
    return out


def test_oracle_constants_follow_the_stated_format():
    facts = _facts()
    assert O.BLOCK == int(facts["block_elements"])
    # two 4-bit values per byte
    codes, sf = O.quantize_nvfp4(np.ones((1, 32), np.float32), 1.0)
    assert codes.shape == (1, 32 // int(facts["values_per_byte"]))
    assert sf.shape == (1, 32 // int(facts["block_elements"]))
    assert facts["element_format"] == "E2M1" and O.E2M1_GRID.max() == 6.0
    assert facts["block_scale_format"] == "E4M3" and O.E4M3_MAX == 448.0


def test_tiny_workload_regression_fixture():
    with open(os.path.join(GOLDEN, "tiny_quant.json")) as f:
        want = json.load(f)
    w = synth.TINY
    x = w.activations().float().numpy()
    wt = w.weight().float().numpy()
    gx = O.global_scale(O.tensor_amax(x))
    gw = O.global_scale(O.tensor_amax(wt))
    xc, xs = O.quantize_nvfp4(x, gx)
    wc, ws = O.quantize_nvfp4(wt, gw)
    h = lambda a: hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()  # noqa: E731
    assert float(gx) == want["g_x"] and float(gw) == want["g_w"]
    assert h(xc) == want["x_codes_sha256"] and h(O.swizzle_sf(xs)) == want["x_sf_swizzled_sha256"]
    assert h(wc) == want["w_codes_sha256"] and h(O.swizzle_sf(ws)) == want["w_sf_swizzled_sha256"]
    y = O.gemm_ref(xc, xs, gx, wc, ws, gw)
    assert abs(y[0, 0] - want["y_00"]) < 1e-12 and abs(y[-1, -1] - want["y_last"]) < 1e-12
    assert abs(y.sum() - want["y_sum"]) < 1e-9


def test_single_stream_pair_fixture_matches_the_oracle():
    # The stored scales of the single-stream pair (written by make_golden.py,
    # which calls only the oracle and the input generators): recomputed here,
    # including the output projection's calibrated input scale from the
    # oracle's full GEMM1 and fused epilogue.
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(GOLDEN, "make_golden.py"))
    MG = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(MG)
    with open(os.path.join(GOLDEN, "single_stream_pair.json")) as f:
        fx = json.load(f)
    got = MG.single_stream_pair()
    for key in ("g_x", "g_w1", "g_w2", "amax_next", "g_next"):
        assert np.float32(got[key]) == np.float32(fx[key]), key
    assert np.float32(fx["g_next"]) == O.global_scale(np.float32(fx["amax_next"]))
