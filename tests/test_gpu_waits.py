"""Bounded device waits, made to run out on purpose through the library's test
knob (moe_debug_wait_knob): the call reports MOE_ERR_TIMEOUT through the
workspace status instead of hanging, and the same context then runs a normal
step that is bit for bit the step of a fresh workspace.

The failure is injected from the host (a tag no CTA publishes, an mbarrier
arrival withheld); nothing here faults or traps the GPU, and every wait that
runs out is bounded by a short poll budget."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, gpu_layer

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = -6


def _names(B, fn):
    tr = B.KernelTrace(capacity=64)
    with tr:
        fn()
    torch.cuda.synchronize()
    return [B.lib().moe_kernel_name(i).decode() for i in tr.ids]


def test_step1_logit_poll_runs_out_and_context_recovers():
    """The one-token step polls for a logit tag that no CTA publishes."""
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 90, ntok=1, device="cuda")
    fresh = B.Workspace.for_layer(layer, 1)
    y_ref = B.moe_forward(layer, wr, x, fresh).cpu().numpy()
    assert B.moe_check_status(fresh) == 0

    ws = B.Workspace.for_layer(layer, 1)
    B.moe_debug_wait_knob(ws, 1, 2000)
    assert _names(B, lambda: B.moe_forward(layer, wr, x, ws)) == ["step1"]
    assert B.moe_check_status(ws) == MOE_ERR_TIMEOUT
    assert B.moe_check_status(ws) == 0  # read and cleared

    B.moe_debug_wait_knob(ws, 0, 0)
    for _ in range(2):
        y = B.moe_forward(layer, wr, x, ws).cpu().numpy()
        assert B.moe_check_status(ws) == 0
        assert np.array_equal(y, y_ref)


def test_tc_mbarrier_waits_run_out_and_context_recovers():
    """The tensor-core mat-vecs' gather warp withholds its first arrival: the
    MMA and fixup warps' mbarrier waits run out, the kernels drain their
    copies, free tensor memory and report MOE_ERR_TIMEOUT."""
    B = bm()
    wl = synthetic.WORKLOADS["30b-b16"]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 91, ntok=16, device="cuda")
    xq, xd = B.moe_quant_act_q8(x)
    idx, wts = B.moe_route_topk(x, wr, wl.top_k)
    fresh = B.Workspace.for_layer(layer, 16, prefill=False)
    y_ref = B.moe_debug_ffn_blocksums(layer, xq, xd, idx, wts, fresh)[0].cpu().numpy()
    assert B.moe_check_status(fresh) == 0

    ws = B.Workspace.for_layer(layer, 16, prefill=False)
    B.moe_debug_wait_knob(ws, 2, 50)
    names = _names(B, lambda: B.moe_debug_ffn_blocksums(layer, xq, xd, idx, wts, ws))
    assert names == ["group", "tc_gateup", "tc_down"]
    assert B.moe_check_status(ws) == MOE_ERR_TIMEOUT

    B.moe_debug_wait_knob(ws, 0, 0)
    for _ in range(2):
        y = B.moe_debug_ffn_blocksums(layer, xq, xd, idx, wts, ws)[0].cpu().numpy()
        assert B.moe_check_status(ws) == 0
        assert np.array_equal(y, y_ref)


def test_wait_knob_rejects_bad_arguments():
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    layer, _ = gpu_layer(wl)
    ws = B.Workspace.for_layer(layer, 1)
    for mode, polls in ((-1, 0), (3, 0), (1, -5)):
        with pytest.raises(B.MoEError) as ei:
            B.moe_debug_wait_knob(ws, mode, polls)
        assert ei.value.code == -1
