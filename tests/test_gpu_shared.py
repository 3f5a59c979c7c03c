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
