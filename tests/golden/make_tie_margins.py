"""Write tie_margins.json: how far the synthetic full-size weights sit from
the ternarisation's rounding tie.

A weight's code is rint(W * s) clipped to [-1, 1] with s = 1/mean|W| per
tensor ("VibeVoice-ASR-BitNet-ONNX" model page, "Quantization" table, row
"LM projections (196 mats)"), so the only decision that a rounding
difference could flip is |W| * s against 0.5 (1.5 and above clip to 1
either way).  For each of the 196 seeded matrices of the Qwen2.5-1.5B-shaped
stack this records mean|W| from the oracle and the smallest distance
| |W| * s - 0.5 | over the matrix, in fp64.  A product of fp64 values is off
by at most 2^-53 relative, so a margin well above 1e-15 means no code of
these inputs depends on how the product is rounded.

Calls only the oracle and the seeded input generator.  Run from the
repository root:  python tests/golden/make_tie_margins.py  (about two
minutes on one core).
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import oracle as orc  # noqa: E402
from ternary_weight_decoder_b200 import synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tie_margins.json")


def tie_margin(W, mean):
    """Smallest | |W| * (1/mean) - 0.5 | over W, in fp64, and its position."""
    s = 1.0 / mean
    d = np.abs(np.abs(W.astype(np.float64)) * s - 0.5)
    i = int(np.argmin(d))
    return float(d.flat[i]), i


def record(layer, proj, name, N, K):
    W = synth.weights(layer, proj, N, K)
    _, mean = orc.ternarize(W)
    margin, i = tie_margin(W, mean)
    return {"layer": layer, "proj": proj, "name": name, "N": N, "K": K,
            "mean_abs": mean, "min_margin": margin, "at": [i // K, i % K]}


def main():
    rows = [record(*s) for s in synth.sweep_shapes()]
    worst = min(rows, key=lambda r: r["min_margin"])
    out = {
        "about": "Per matrix of the synthetic 196-matrix sweep: mean|W| from the oracle and the "
                 "smallest | |W| * (1/mean) - 0.5 | in fp64, the distance of its weights from "
                 "the one rounding tie that decides a ternary code. Written by "
                 "make_tie_margins.py beside this file.",
        "weights": "synth.weights(layer, proj, N, K), N(0, 0.02^2), every matrix of the "
                   "28-layer sweep",
        "min_margin": worst["min_margin"],
        "min_at": {k: worst[k] for k in ("layer", "proj", "name", "at")},
        "matrices": rows,
    }
    with open(OUT, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print(f"{len(rows)} matrices; smallest margin {worst['min_margin']:.3e} "
          f"({worst['name']} of layer {worst['layer']})")


if __name__ == "__main__":
    main()
