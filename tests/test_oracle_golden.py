"""The oracle reproduces its stored outputs (tests/golden/tiny_layer.json and
tests/golden/tiny_layer_formats.json)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_golden  # noqa: E402


def test_tiny_layer_golden(orc):
    with open(os.path.join(HERE, "golden", "tiny_layer.json")) as f:
        gold = json.load(f)
    wl, wg, wu, wd, wr, x = make_golden.tiny_case()
    assert make_golden.digest(wg, wu, wd, wr, x) == gold["inputs_sha256"], \
        "the seeded input generator changed"
    layer = orc.Layer.from_float(wl.hidden, wl.ffn, wl.n_experts, wl.top_k, wg, wu, wd)
    assert make_golden.digest(layer.gate[0], layer.gate[1], layer.up[0], layer.up[1],
                              layer.down[0], layer.down[1]) == gold["packed_sha256"]
    y, idx, wts, dbg = orc.moe_forward(layer, wr, x, debug=True)
    assert make_golden.digest(dbg["xq"], dbg["xd"]) == gold["xq_sha256"]
    assert make_golden.digest(dbg["aq"], dbg["ad"]) == gold["aq_sha256"]
    assert idx.tolist() == gold["idx"]
    assert np.array_equal(wts, np.array(gold["wts"]))
    assert np.array_equal(y, np.array(gold["y"]))


def test_tiny_layer_formats_golden(orc):
    with open(os.path.join(HERE, "golden", "tiny_layer_formats.json")) as f:
        gold = json.load(f)
    got = make_golden.formats_case()
    for key in ("sign", "e16", "shared"):
        assert got[key]["packed_sha256"] == gold[key]["packed_sha256"], key
        assert np.array_equal(np.array(got[key]["y"]), np.array(gold[key]["y"])), key
    for key in ("sign", "e16"):
        assert got[key]["idx"] == gold[key]["idx"]
