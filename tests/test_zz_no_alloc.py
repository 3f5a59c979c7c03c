"""moe_expert_ffn_decode_static -- the decode FFN for callers that cannot
allocate device memory -- gives the same outputs as moe_expert_ffn_decode
with a caller workspace, call after call.

Kept in a file of its own that is collected last: the entry point shares one
static scratch array per process, and this test must pass both alone in a
fresh process and after every other test has used the library."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, gpu_layer, rel_err_rms

pytestmark = pytest.mark.gpu

LAYER_TOL = 2e-3  # the full-layer tolerance of the parity tests


@pytest.mark.parametrize("name,ntok", [("tiny", 1), ("30b", 1), ("30b", 4), ("30b-b16", 16)])
def test_static_scratch_matches_workspace_path(name, ntok):
    B = bm()
    wl = synthetic.WORKLOADS[name]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    for call in range(2):  # two calls in a row, different inputs
        x = synthetic.activations(wl, 40 + call, ntok=ntok, device="cuda")
        xq, xd = B.moe_quant_act_q8(x)
        idx, wts = B.moe_route_topk(x, wr, wl.top_k)
        ws = B.Workspace.for_layer(layer, ntok, prefill=False)
        ref = B.moe_expert_ffn_decode(layer, xq, xd, idx, wts, ws).cpu().numpy()
        assert B.moe_check_status(ws) == 0
        y = B.moe_expert_ffn_decode_static(layer, xq, xd, idx, wts).cpu().numpy()
        assert rel_err_rms(y, ref) <= LAYER_TOL
        assert np.isfinite(y).all()


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
