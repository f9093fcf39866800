"""No code of the synthetic full-size weights sits on a rounding tie.

The ternary code of a weight is decided by |W| * s against 0.5 (s = 1/mean|W|
per tensor: "VibeVoice-ASR-BitNet-ONNX" model page, "Quantization" table,
row "LM projections (196 mats)").  Both the oracle and the GPU compute that
product in fp64, whose rounding error is at most 2^-53 relative; the record
``golden/tie_margins.json`` (written by ``golden/make_tie_margins.py`` from
the oracle and the seeded generator) gives, for each of the 196 matrices,
the smallest distance of |W| * s from 0.5.  These tests check the record and
recompute a layer of it.
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle as orc
from ternary_weight_decoder_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module")
def rec():
    with open(os.path.join(GOLDEN, "tie_margins.json")) as f:
        return json.load(f)


def test_record_covers_the_sweep(rec):
    shapes = synth.sweep_shapes()
    assert len(rec["matrices"]) == len(shapes) == 196
    for r, (l, p, name, N, K) in zip(rec["matrices"], shapes):
        assert (r["layer"], r["proj"], r["name"], r["N"], r["K"]) == (l, p, name, N, K)
        assert 0.0 < r["min_margin"] < 0.5
        assert 0.014 < r["mean_abs"] < 0.018   # E|W| = 0.02 * sqrt(2/pi) = 0.01596
    assert rec["min_margin"] == min(r["min_margin"] for r in rec["matrices"])


def test_no_code_depends_on_product_rounding(rec):
    # |W| * s is near 0.5, so one fp64 rounding moves it by at most
    # 0.5 * 2^-53 ~ 5.6e-17: margins many orders above that cannot flip.
    assert rec["min_margin"] > 1e-13


@pytest.mark.parametrize("proj", range(7))
def test_layer0_recomputed(rec, proj):
    r = rec["matrices"][proj]
    W = synth.weights(r["layer"], r["proj"], r["N"], r["K"])
    codes, mean = orc.ternarize(W)
    assert mean == r["mean_abs"]
    d = np.abs(np.abs(W.astype(np.float64)) * (1.0 / mean) - 0.5)
    assert float(d.min()) == r["min_margin"]
    n, k = r["at"]
    assert d[n, k] == r["min_margin"]
    # the weight nearest the tie gets the code the comparison says
    assert abs(int(codes[n, k])) == (1 if abs(float(W[n, k])) * (1.0 / mean) > 0.5 else 0)
