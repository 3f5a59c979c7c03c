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


@pytest.mark.parametrize("name,ntok,mode,polls,kernels", [
    ("30b", 1, 1, 2000, ["step1"]),                                        # tagged logit poll
    ("30b-b16", 16, 2, 50, ["router_quant", "topk_group", "tc_gateup", "tc_down"]),  # mbarrier waits
])
def test_wait_runs_out_and_context_recovers(name, ntok, mode, polls, kernels):
    B = bm()
    wl = synthetic.WORKLOADS[name]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 90, ntok=ntok, device="cuda")
    fresh = B.Workspace.for_layer(layer, ntok)
    y_ref = B.moe_forward(layer, wr, x, fresh).cpu().numpy()
    assert B.moe_check_status(fresh) == 0

    ws = B.Workspace.for_layer(layer, ntok)
    B.moe_debug_wait_knob(ws, mode, polls)
    assert _names(B, lambda: B.moe_forward(layer, wr, x, ws)) == kernels
    assert B.moe_check_status(ws) == MOE_ERR_TIMEOUT
    assert B.moe_check_status(ws) == 0  # read and cleared

    B.moe_debug_wait_knob(ws, 0, 0)
    for _ in range(2):
        y = B.moe_forward(layer, wr, x, ws).cpu().numpy()
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
