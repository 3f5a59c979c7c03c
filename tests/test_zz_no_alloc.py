"""moe_expert_ffn_decode_static -- the decode FFN for callers that cannot
allocate device memory -- gives the same outputs as moe_expert_ffn_decode
with a caller workspace, call after call.

Both entry points run the same kernels on the same inputs, so the outputs must
agree bit for bit; a difference would mean that the shared array kept
something (a counter, a status word, a stale table) from an earlier call.

Kept in a file of its own that is collected last: the entry point shares one
static scratch array per process, and this test must pass both alone in a
fresh process and after every other test has used the library."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, gpu_layer

pytestmark = pytest.mark.gpu


def _call_pair(B, wl, layer, wr, ntok, seed):
    """(static-scratch output, workspace-path output) for one seeded batch."""
    x = synthetic.activations(wl, seed, ntok=ntok, device="cuda")
    xq, xd = B.moe_quant_act_q8(x)
    idx, wts = B.moe_route_topk(x, wr, wl.top_k)
    ws = B.Workspace.for_layer(layer, ntok, prefill=False)
    ref = B.moe_expert_ffn_decode(layer, xq, xd, idx, wts, ws).cpu().numpy()
    assert B.moe_check_status(ws) == 0
    y = B.moe_expert_ffn_decode_static(layer, xq, xd, idx, wts).cpu().numpy()
    return y, ref


@pytest.mark.parametrize("name,ntok", [("tiny", 1), ("30b", 1), ("30b", 4), ("30b-b16", 16)])
def test_static_scratch_matches_workspace_path(name, ntok):
    B = bm()
    wl = synthetic.WORKLOADS[name]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    for call in range(2):  # two calls in a row, different inputs
        y, ref = _call_pair(B, wl, layer, wr, ntok, 40 + call)
        assert np.isfinite(y).all()
        assert np.array_equal(y, ref), "static-scratch output differs from the workspace path"


def test_static_scratch_large_then_small_call():
    """A 16-token call leaves more of the array dirty than a 1-token call
    clears; the 1-token call that follows must still match bit for bit."""
    B = bm()
    wl = synthetic.WORKLOADS["30b-b16"]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    for ntok, seed in ((16, 50), (1, 51), (16, 52), (2, 53)):
        y, ref = _call_pair(B, wl, layer, wr, ntok, seed)
        assert np.array_equal(y, ref), "%d-token call after a larger one differs" % ntok


def test_static_scratch_rejects_oversize_calls():
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, _ = gpu_layer(wl)
    # 64 tokens need about 4.6 MB of scratch (aq, per-slot outputs, ...)
    assert layer.workspace_bytes(64) > 4 << 20
    xq = torch.zeros((64, wl.hidden), dtype=torch.int8, device="cuda")
    xd = torch.zeros((64, wl.hidden // 32), dtype=torch.float32, device="cuda")
    idx = torch.zeros((64, wl.top_k), dtype=torch.int32, device="cuda")
    wts = torch.zeros((64, wl.top_k), dtype=torch.float32, device="cuda")
    with pytest.raises(B.MoEError) as ei:
        B.moe_expert_ffn_decode_static(layer, xq, xd, idx, wts)
    assert ei.value.code == -4
