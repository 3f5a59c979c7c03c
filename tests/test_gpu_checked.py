"""The bounds-checked build (-DMOE_CHECKED, libbitmoe_checked.so) on the
parity cases: every guarded index of the kernels (pair ids from the grouping
tables, items, groups of the prefill layout, tokens of the combine) stays in
its buffer -- no MOE_ERR_BOUNDS -- and the checked build gives the normal
build's outputs bit for bit.  This stands in for a memory checker, which is
not available on this machine's GPUs; the guard-canary tests cover writes past
the ends of the outputs."""
import numpy as np
import pytest

import synthetic
from gpu_helpers import bm, gpu_layer

pytestmark = pytest.mark.gpu

MOE_ERR_BOUNDS = -9


@pytest.fixture(scope="module")
def checked():
    B = bm()
    from bit_moe_b200 import build
    build.build_checked()
    return B.load_library(B.CHECKED_LIB_PATH)


def _with_lib(B, L, fn):
    saved = B._lib
    B._lib = L
    try:
        return fn()
    finally:
        B._lib = saved


@pytest.mark.parametrize("name,ntok", [("tiny", 1), ("tiny", 3), ("tiny", 70), ("30b-b16", 16),
                                       ("30b", 1), ("tiny", 300)])
def test_checked_build_matches_and_stays_in_bounds(checked, name, ntok):
    B = bm()
    wl = synthetic.WORKLOADS[name]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 97, ntok=ntok, device="cuda")
    ws = B.Workspace.for_layer(layer, ntok)
    ref = B.moe_forward(layer, wr, x, ws).cpu().numpy()
    assert B.moe_check_status(ws) == 0

    def run():
        wsc = B.Workspace.for_layer(layer, ntok)
        y = B.moe_forward(layer, wr, x, wsc).cpu().numpy()
        return y, B.moe_check_status(wsc)

    y, status = _with_lib(B, checked, run)
    assert status != MOE_ERR_BOUNDS, "an index left its buffer"
    assert status == 0
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("ntok,prefill", [(3, False), (17, False), (70, True), (130, True)])
def test_checked_build_tensor_core_hook(checked, ntok, prefill):
    """The tensor-core decode mat-vecs and the prefill GEMM (through the block
    sum hook, which runs them for any batch) under the bounds checks."""
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 98, ntok=ntok, device="cuda")
    xq, xd = B.moe_quant_act_q8(x)
    idx, wts = B.moe_route_topk(x, wr, wl.top_k)
    ws = B.Workspace.for_layer(layer, ntok, prefill=prefill)
    ref = [t.cpu().numpy() for t in B.moe_debug_ffn_blocksums(layer, xq, xd, idx, wts, ws, prefill=prefill)]

    def run():
        wsc = B.Workspace.for_layer(layer, ntok, prefill=prefill)
        out = [t.cpu().numpy() for t in B.moe_debug_ffn_blocksums(layer, xq, xd, idx, wts, wsc, prefill=prefill)]
        return out, B.moe_check_status(wsc)

    out, status = _with_lib(B, checked, run)
    assert status == 0
    for a, b in zip(out, ref):
        assert np.array_equal(a, b)
