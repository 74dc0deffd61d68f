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
