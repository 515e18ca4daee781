"""Writes the fixtures of this directory from the oracle and the seeded generator only.

    python tests/golden/make_golden.py

The pages print no worked example (no codes, scales or outputs of any layer), so nothing
here is a value from the pages.  These fixtures are regression guards of the oracle: a
change to its arithmetic changes them, and the commit that regenerates them must name the
passage or the reading that justifies the change.  They are not pins of the oracle (the pins
are the tests against code tables, closed forms, brute force and exact arithmetic).
"""

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import awq, nvfp4, svdq  # noqa: E402
import synth  # noqa: E402


def _hex(a):
    return [float(v).hex() for v in np.asarray(a, dtype=np.float64).ravel()]


def svdq_tiny():
    """The seeded SVDQ layer at M = 4, K = 64, N = 128: activation codes and scales, the
    weight per-tensor scale and the float64 output."""
    w = synth.svdq_workload(4, 64, 128, seed=3)
    cx, sx = svdq.quantize_activations(w.X, w.smooth_inv, w.g_a)
    cw, sw, g_w = svdq.quantize_weights(w.R)
    y = svdq.forward(w.X, w.smooth_inv, w.R, w.L1, w.L2, w.bias, w.g_a)
    return {"what": "svdq forward, synth.svdq_workload(4, 64, 128, seed=3)",
            "g_a": float(w.g_a).hex(), "g_w": float(g_w).hex(),
            "act_codes_packed_hex": nvfp4.pack_nibbles(cx).tobytes().hex(),
            "act_scales_hex": np.asarray(sx, dtype=np.uint8).tobytes().hex(),
            "weight_scales_hex": np.asarray(sw, dtype=np.uint8).tobytes().hex(),
            "y_shape": list(y.shape), "y_hex": _hex(y)}


def awq_tiny():
    """The seeded AWQ layer at M = 3, K = 128, N = 64: the float64 output."""
    a = synth.awq_workload(3, 128, 64, seed=4)
    y = awq.forward(a.X, a.q, a.scales, a.zeros)
    return {"what": "awq forward, synth.awq_workload(3, 128, 64, seed=4)", "y_shape": list(y.shape), "y_hex": _hex(y)}


FIXTURES = {"svdq_tiny_4x64x128.json": svdq_tiny, "awq_tiny_3x128x64.json": awq_tiny}

if __name__ == "__main__":
    for name, fn in FIXTURES.items():
        with open(os.path.join(HERE, name), "w") as f:
            json.dump(fn(), f, indent=1)
            f.write("\n")
        print("wrote", name)
