"""Which kernels each entry point launches, read through the library's launch
trace: the test of a path also checks that the path's kernels are the ones
that ran (no silent fallback to another path)."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, gpu_layer

pytestmark = pytest.mark.gpu


def _names(B, fn):
    tr = B.KernelTrace(capacity=64)
    with tr:
        fn()
    torch.cuda.synchronize()
    return [B.lib().moe_kernel_name(i).decode() for i in tr.ids]


@pytest.mark.parametrize("fmt,ntok,expect", [
    ("ternary", 1, ["step1"]),
    ("ternary", 16, ["route_group", "gateup", "down"]),
    ("sign", 1, ["step1"]),
    ("sign", 3, ["route_group", "gateup", "down"]),
    ("e16", 1, ["step1"]),
    ("e16", 3, ["route_group", "gateup", "down"]),
])
def test_forward_kernels(fmt, ntok, expect):
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, _ = gpu_layer(wl, fmt=fmt)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 81, ntok=ntok, device="cuda")
    ws = B.Workspace.for_layer(layer, ntok)
    assert _names(B, lambda: B.moe_forward(layer, wr, x, ws)) == expect


def test_routing_in_one_launch_and_in_two():
    """A decode batch routes in one launch (k_route_group) where a one-wave
    shape holds the router rows and tokens in shared memory, and in two
    (router with quantization, then top-k with grouping) where none does:
    64 tokens of hidden 4096 over 128 experts.  Both give the same outputs,
    bit for bit (each token's result does not depend on its batch)."""
    B = bm()
    wl = synthetic.WORKLOADS["tiny"].with_(hidden=4096, ffn=256, n_experts=128, top_k=2, seed=85)
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 86, ntok=64, device="cuda")
    ws = B.Workspace.for_layer(layer, 64)
    y64 = torch.empty((64, wl.hidden), device="cuda")
    assert _names(B, lambda: B.moe_forward(layer, wr, x, ws, y=y64)) == [
        "router_quant", "topk_group", "gateup", "down"]
    assert B.moe_check_status(ws) == 0
    ws8 = B.Workspace.for_layer(layer, 8)
    for c in range(8):
        xc = x[8 * c:8 * (c + 1)].contiguous()
        y8 = torch.empty((8, wl.hidden), device="cuda")
        names = _names(B, lambda: B.moe_forward(layer, wr, xc, ws8, y=y8))
        assert names == ["route_group", "gateup", "down"]
        assert torch.equal(y8, y64[8 * c:8 * (c + 1)])
    assert B.moe_check_status(ws8) == 0


def test_forward_prefill_kernels():
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 82, ntok=65, device="cuda")
    ws = B.Workspace.for_layer(layer, 65)
    assert _names(B, lambda: B.moe_forward(layer, wr, x, ws)) == [
        "quant_act_q8", "router_logits", "topk_softmax", "group", "prefill_gather", "prefill_gateup",
        "prefill_down", "combine"]


def test_forward_outside_fused_step_and_decode_kernels():
    B = bm()
    wl = synthetic.WORKLOADS["tiny"].with_(n_experts=300, seed=83)
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 84, ntok=4, device="cuda")
    ws = B.Workspace.for_layer(layer, 4)
    assert _names(B, lambda: B.moe_forward(layer, wr, x[:1].contiguous(), ws)) == ["route", "gateup", "down"]
    xq, xd = B.moe_quant_act_q8(x)
    idx, wts = B.moe_route_topk(x, wr, wl.top_k)
    assert _names(B, lambda: B.moe_expert_ffn_decode(layer, xq[:1].contiguous(), xd[:1].contiguous(),
                                                     idx[:1].contiguous(), wts[:1].contiguous(), ws)) == ["gateup", "down"]
    assert _names(B, lambda: B.moe_expert_ffn_decode(layer, xq, xd, idx, wts, ws)) == ["group", "gateup", "down"]


def test_blocksum_hook_kernels():
    """The block-sum test hook runs the tensor-core kernels (decode: grouping
    then the two mat-vecs; prefill: the grouped GEMM chain)."""
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    for ntok, prefill, expect in ((3, False, ["group", "tc_gateup", "tc_down"]),
                                  (70, True, ["group", "prefill_gather", "prefill_gateup", "prefill_down",
                                              "combine"])):
        x = synthetic.activations(wl, 86, ntok=ntok, device="cuda")
        xq, xd = B.moe_quant_act_q8(x)
        idx, wts = B.moe_route_topk(x, wr, wl.top_k)
        ws = B.Workspace.for_layer(layer, ntok, prefill=prefill)
        assert _names(B, lambda: B.moe_debug_ffn_blocksums(layer, xq, xd, idx, wts, ws, prefill=prefill)) == expect


def test_forward_host_kernels():
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    xh = synthetic.activations(wl, 85, ntok=1, device="cpu").pin_memory()
    yh = torch.empty((1, wl.hidden), dtype=torch.float32).pin_memory()
    ws = B.Workspace.for_layer(layer, 1)
    assert _names(B, lambda: B.moe_forward_host(layer, wr, xh, yh, ws)) == ["copy", "step1"]
    assert np.isfinite(yh.numpy()).all()
