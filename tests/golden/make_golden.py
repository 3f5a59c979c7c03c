"""Write the stored expected values under tests/golden/ from the oracle alone.

No page prints a worked example of this method, so the stored values are the
oracle's own outputs on small seeded synthetic inputs.  They guard the oracle
against unnoticed changes: a commit that changes any of them must name the
passage (or the reading of it) that justifies the change.

Run:  python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synthetic  # noqa: E402


def digest(*arrays):
    h = hashlib.sha256()
    for a in arrays:
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def tiny_case():
    wl = synthetic.WORKLOADS["tiny"]
    wg, wu, wd = (t.numpy() for t in synthetic.layer_float(wl, 0, "cpu"))
    wr = synthetic.router(wl, 0, "cpu").numpy()
    x = synthetic.activations(wl, 0, ntok=3, device="cpu").numpy()
    return wl, wg, wu, wd, wr, x


def main():
    wl, wg, wu, wd, wr, x = tiny_case()
    layer = oracle.Layer.from_float(wl.hidden, wl.ffn, wl.n_experts, wl.top_k, wg, wu, wd)
    y, idx, wts, dbg = oracle.moe_forward(layer, wr, x, debug=True)
    out = {
        "what": "oracle outputs for the tiny layer (hidden 256, ffn 512, 8 experts, top-2), "
                "3 tokens of x ~ N(0,1), weights N(0, 0.02), router N(0, 0.02)",
        "inputs_sha256": digest(wg, wu, wd, wr, x),
        "packed_sha256": digest(layer.gate[0], layer.gate[1], layer.up[0], layer.up[1],
                                layer.down[0], layer.down[1]),
        "xq_sha256": digest(dbg["xq"], dbg["xd"]),
        "aq_sha256": digest(dbg["aq"], dbg["ad"]),
        "idx": idx.tolist(),
        "wts": [[float(v) for v in row] for row in wts],
        "y": [[float(v) for v in row] for row in y],
    }
    path = os.path.join(HERE, "tiny_layer.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)

    path = os.path.join(HERE, "tiny_layer_formats.json")
    with open(path, "w") as f:
        json.dump(formats_case(), f, indent=1)
    print("wrote", path)


def shared_expert(wl):
    """A seeded shared expert of the tiny layer's width (ffn 256)."""
    rng = np.random.default_rng(99)
    fs = 256
    return oracle.SharedExpert(wl.hidden, fs,
                               (rng.standard_normal((fs, wl.hidden)) * 0.02).astype(np.float32),
                               (rng.standard_normal((fs, wl.hidden)) * 0.02).astype(np.float32),
                               (rng.standard_normal((wl.hidden, fs)) * 0.02).astype(np.float32))


def formats_case():
    """The tiny layer in the sign-code and E16 formats, and the ternary layer
    with a shared expert: packed digests and outputs."""
    wl, wg, wu, wd, wr, x = tiny_case()
    out = {"what": "oracle outputs of the tiny layer of tiny_layer.json in the 1-bit sign-code and "
                   "two-level (E16) formats, and of the ternary layer with a seeded 8-bit shared "
                   "expert (ffn 256, weights N(0, 0.02) from numpy's default_rng(99))"}
    for fmt in ("sign", "e16"):
        layer = oracle.Layer.from_float(wl.hidden, wl.ffn, wl.n_experts, wl.top_k, wg, wu, wd, fmt=fmt)
        y, idx, _ = oracle.moe_forward(layer, wr, x)
        out[fmt] = {"packed_sha256": digest(*layer.gate, *layer.up, *layer.down),
                    "idx": idx.tolist(), "y": [[float(v) for v in row] for row in y]}
    layer = oracle.Layer.from_float(wl.hidden, wl.ffn, wl.n_experts, wl.top_k, wg, wu, wd)
    sh = shared_expert(wl)
    y, idx, _ = oracle.moe_forward(layer, wr, x, shared=sh)
    out["shared"] = {"packed_sha256": digest(*sh.gate, *sh.up, *sh.down),
                     "y": [[float(v) for v in row] for row in y]}
    return out


if __name__ == "__main__":
    main()
