"""Parity of the shared expert (8-bit blocks, added to the routed sum) on the
CUDA path with the CPU oracle: codes and scales bit-exact, the layer output
with the shared term within 2e-3 * RMS(ref)."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, gpu_layer, oracle_layer, rel_err_rms

pytestmark = pytest.mark.gpu

LAYER_TOL = 2e-3


def _shared_weights(H, Fs, seed):
    g = np.random.default_rng(seed)
    wg = (g.standard_normal((Fs, H)) * 0.02).astype(np.float32)
    wu = (g.standard_normal((Fs, H)) * 0.02).astype(np.float32)
    wd = (g.standard_normal((H, Fs)) * 0.02).astype(np.float32)
    return wg, wu, wd


@pytest.mark.parametrize("rows,k", [(32, 256), (100, 768), (7, 2048)])
def test_q8_weights_bytes(orc, rows, k):
    B = bm()
    w = (np.random.default_rng(rows + k).standard_normal((rows, k)) * 0.02).astype(np.float32)
    w[0, :32] = 0.0
    q, d = B.moe_quantize_weights_q8(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    oq, od = orc.quantize_weights_q8(w)
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(d.cpu().numpy().view(np.uint16), od)


@pytest.mark.parametrize("wl_name,ntok,Fs", [("tiny", 1, 256), ("tiny", 5, 512), ("30b", 3, 1024)])
def test_shared_expert_added_to_the_layer(orc, wl_name, ntok, Fs):
    B = bm()
    wl = synthetic.WORKLOADS[wl_name]
    H = wl.hidden
    layer, fn = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 71, ntok=ntok, device="cuda")
    wg, wu, wd = _shared_weights(H, Fs, 72 + ntok)
    sh = B.SharedExpert(torch.from_numpy(wg).cuda(), torch.from_numpy(wu).cuda(), torch.from_numpy(wd).cuda())
    ws = B.Workspace.for_layer(layer, ntok)
    y = B.moe_forward(layer, wr, x, ws)
    xq, xd = B.moe_quant_act_q8(x)
    sh.add(xq, xd, y)
    y = y.cpu().numpy()
    assert B.moe_check_status(ws) == 0
    # oracle: routed experts (routing by the oracle router) plus the shared term
    xs = x.cpu().numpy()
    oidx, owts = orc.route_topk(xs, wr.cpu().numpy(), wl.top_k)
    olayer, remap = oracle_layer(orc, wl, fn, oidx)
    oq, od = orc.quant_act_q8(xs)
    ref = orc.expert_ffn(olayer, oq, od, remap[oidx], owts.astype(np.float32))
    ref = orc.SharedExpert(H, Fs, wg, wu, wd).add_to(ref, oq, od)
    assert rel_err_rms(y, ref) <= LAYER_TOL


def test_shared_expert_alone(orc):
    """Added to zeros, the shared term matches the oracle's shared FFN."""
    B = bm()
    H, Fs, ntok = 512, 768, 4
    wg, wu, wd = _shared_weights(H, Fs, 73)
    sh = B.SharedExpert(torch.from_numpy(wg).cuda(), torch.from_numpy(wu).cuda(), torch.from_numpy(wd).cuda())
    x = np.random.default_rng(74).standard_normal((ntok, H)).astype(np.float32)
    xq, xd = B.moe_quant_act_q8(torch.from_numpy(x).cuda())
    y = sh.add(xq, xd, torch.zeros((ntok, H), dtype=torch.float32, device="cuda")).cpu().numpy()
    ref = orc.SharedExpert(H, Fs, wg, wu, wd).add_to(np.zeros((ntok, H)), xq.cpu().numpy(), xd.cpu().numpy())
    assert rel_err_rms(y, ref) <= LAYER_TOL


@pytest.mark.parametrize("wl_name,ntok", [("30b", 1), ("tiny", 1), ("30b", 5), ("tiny", 70)])
def test_workspace_act_is_the_step_quantization(wl_name, ntok):
    """moe_forward leaves x's int8 codes and scales in its workspace (the
    one-token step, the batched decode and the prefill path each write them):
    bit for bit those of moe_quant_act_q8, so the shared expert can take them
    without quantizing x again."""
    B = bm()
    wl = synthetic.WORKLOADS[wl_name]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 75 + ntok, ntok=ntok, device="cuda")
    ws = B.Workspace.for_layer(layer, ntok)
    B.moe_forward(layer, wr, x, ws)
    assert B.moe_check_status(ws) == 0
    wq, wd = ws.act(layer, ntok)
    xq, xd = B.moe_quant_act_q8(x)
    assert np.array_equal(wq.cpu().numpy(), xq.cpu().numpy())
    assert np.array_equal(wd.cpu().numpy().view(np.uint32), xd.cpu().numpy().view(np.uint32))


def _names(B, fn):
    tr = B.KernelTrace(capacity=64)
    with tr:
        fn()
    torch.cuda.synchronize()
    return [B.lib().moe_kernel_name(i).decode() for i in tr.ids]


@pytest.mark.parametrize("wl_name,fmt,ntok,Fs", [
    ("30b", "ternary", 1, 768),     # slot-order down items, 24 shared blocks
    ("tiny", "ternary", 1, 256),
    ("tiny", "sign", 1, 2048),      # the most shared blocks the step takes (64)
    ("large", "ternary", 1, 1024),  # half-slot down items
    ("30b", "sign", 1, 96),
    ("30b", "e16", 1, 768),        # two-level scales in the step
    ("30b", "ternary", 3, 768),     # more tokens: the routed kernels, then the shared expert's
    ("tiny", "ternary", 1, 2080),   # more than 64 blocks: moe_forward, then the shared expert's
])
def test_forward_shared_equals_forward_then_shared_add(wl_name, fmt, ntok, Fs):
    """moe_forward_shared gives, bit for bit, moe_forward followed by the
    shared expert's add on the int8 x the step leaves in the workspace; one
    token of a layer the one-token step takes is one launch."""
    B = bm()
    wl = synthetic.WORKLOADS[wl_name]
    H = wl.hidden
    layer, _ = gpu_layer(wl, fmt=fmt)
    wr = synthetic.router(wl, 0, "cuda")
    wg, wu, wd = _shared_weights(H, Fs, 91 + Fs)
    sh = B.SharedExpert(torch.from_numpy(wg).cuda(), torch.from_numpy(wu).cuda(), torch.from_numpy(wd).cuda())
    ws = B.Workspace.for_layer(layer, ntok)
    ws2 = B.Workspace.for_layer(layer, ntok)
    sws = sh.workspace(ntok)
    fused = ntok == 1 and Fs // 32 <= 64
    for seed in range(3):
        x = synthetic.activations(wl, 300 + seed, ntok=ntok, device="cuda")
        y1 = torch.empty((ntok, H), device="cuda")
        names = _names(B, lambda: B.moe_forward_shared(layer, sh, wr, x, ws, sws, y=y1))
        if fused:
            assert names == ["step1"]
        else:
            assert names[-2:] == ["shared", "shared"]
        y2 = B.moe_forward(layer, wr, x, ws2)
        xq, xd = ws2.act(layer, ntok)
        sh.add(xq, xd, y2)
        assert B.moe_check_status(ws) == 0 and B.moe_check_status(ws2) == 0
        assert torch.equal(y1, y2), (wl_name, fmt, ntok, Fs, seed)


def test_forward_shared_refuses_a_hidden_mismatch():
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    wg, wu, wd = _shared_weights(512, 64, 5)
    sh = B.SharedExpert(torch.from_numpy(wg).cuda(), torch.from_numpy(wu).cuda(), torch.from_numpy(wd).cuda())
    x = synthetic.activations(wl, 1, ntok=1, device="cuda")
    with pytest.raises(RuntimeError):
        B.moe_forward_shared(layer, sh, wr, x, B.Workspace.for_layer(layer, 1))
