"""Write the oracle fixtures ``tiny_quant.json`` and ``single_stream_pair.json``.

Calls only ``oracle`` and ``synth``.  ``tiny_quant.json`` holds digests of the
oracle's own output for the tiny workload, so a later change to the oracle's
arithmetic shows up as a mismatch that must be justified.
``single_stream_pair.json`` holds the per-tensor scales of the FLUX
single-stream block pair (seed 3): the input's and both weights' scales, and
the output projection's calibrated input scale, i.e. amax of the oracle's
fused-epilogue values (Q columns as they are, MLP columns after GELU-tanh,
both rounded to bf16) divided by 6 * 448, the calibration the BFL doc's
``nvfp4`` bullet describes applied to the tensor the output projection reads.
Run from the repo root: ``python tests/golden/make_golden.py`` (about a minute:
the single-stream fixture needs the oracle's full 4608 x 3072 x 21504 GEMM).
"""
import hashlib
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402
import synth  # noqa: E402


def digest(a) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def main():
    w = synth.TINY
    x = w.activations().float().numpy()
    wt = w.weight().float().numpy()
    gx = O.global_scale(O.tensor_amax(x))
    gw = O.global_scale(O.tensor_amax(wt))
    xc, xs = O.quantize_nvfp4(x, gx)
    wc, ws = O.quantize_nvfp4(wt, gw)
    y = O.gemm_ref(xc, xs, gx, wc, ws, gw)
    out = {
        "workload": w.name,
        "g_x": float(gx), "g_w": float(gw),
        "x_codes_sha256": digest(xc), "x_sf_swizzled_sha256": digest(O.swizzle_sf(xs)),
        "w_codes_sha256": digest(wc), "w_sf_swizzled_sha256": digest(O.swizzle_sf(ws)),
        "y_00": float(y[0, 0]), "y_last": float(y[-1, -1]), "y_sum": float(y.sum()),
    }
    with open(os.path.join(HERE, "tiny_quant.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    with open(os.path.join(HERE, "single_stream_pair.json"), "w") as f:
        json.dump(single_stream_pair(), f, indent=1)
        f.write("\n")


def single_stream_next_scale(x, w1, b1):
    """The output projection's calibrated input scale: the oracle's GEMM1 with
    bias, its fused epilogue on the Q and MLP column ranges, amax / 2688."""
    gx = O.global_scale(O.tensor_amax(x))
    gw1 = O.global_scale(O.tensor_amax(w1))
    xc, xs = O.quantize_nvfp4(x, gx)
    wc, ws = O.quantize_nvfp4(w1, gw1)
    y = O.gemm_ref(xc, xs, gx, wc, ws, gw1, b1)
    ep = O.epilogue_ref(y, [(*synth.SINGLE_Q, O.ACT_NONE), (*synth.SINGLE_MLP, O.ACT_GELU_TANH)])
    return gx, gw1, O.tensor_amax(ep), O.global_scale(O.tensor_amax(ep))


def single_stream_pair():
    w1l, w2l = synth.SINGLE_IN, synth.SINGLE_OUT
    x = w1l.activations().float().numpy()
    w1 = w1l.weight().float().numpy()
    b1 = w1l.bias_vec().float().numpy()
    w2 = w2l.weight().float().numpy()
    gx, gw1, amax_next, g_next = single_stream_next_scale(x, w1, b1)
    return {
        "workload": [w1l.name, w2l.name],
        "g_x": float(gx), "g_w1": float(gw1), "g_w2": float(O.global_scale(O.tensor_amax(w2))),
        "amax_next": float(amax_next), "g_next": float(g_next),
    }


if __name__ == "__main__":
    main()
