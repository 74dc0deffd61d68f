"""Write the oracle regression fixture ``tiny_quant.json``.

Calls only ``oracle`` and ``synth``: the stored digests are the oracle's own
output for the tiny workload, so a later change to the oracle's arithmetic
shows up as a mismatch that must be justified.  Run from the repo root:
``python tests/golden/make_golden.py``.
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


if __name__ == "__main__":
    main()
