"""The tensor-core paths' exact int32 block sums against the oracle, bit for
bit (pxq_llama README, "PXQ vs MXFP4": one fixup per 32-value activation
block of an int8 dot product; Parakon Runtime README, "How it works").

moe_debug_ffn_blocksums runs the expert FFN through the grouped tensor-core
mat-vecs (decode) and writes sum(q * a) for every (pair, row, 32-block):
  - gate and up rows against the token's int8 codes: the oracle's block sums
    of its own quantization of the same fp32 weights, on its own int8 codes;
  - down rows against the int8 SwiGLU codes: compared with the oracle's block
    sums on the oracle's own SwiGLU codes wherever the two sides' codes of a
    32-block agree (they are taken from fp32 on the GPU and fp64 in the oracle,
    so a code may differ by one at a rounding boundary; almost all blocks
    agree, and the test requires that too).
All the GPU's inputs (codes, scales, ids, weights of the slots) are the
oracle's, so nothing on the oracle side comes from the GPU."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, gpu_layer, oracle_layer, rel_err_rms

pytestmark = pytest.mark.gpu

LAYER_TOL = 2e-3


def _cuda(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.to(dtype) if dtype is not None else t).cuda()


def _check_blocksums(orc, B, wl, layer, fn, x, wr, sample=None, prefill=False, seed=0):
    K, H, F = wl.top_k, wl.hidden, wl.ffn
    ntok = x.shape[0]
    oq, od = orc.quant_act_q8(x)
    oidx, owts = orc.route_topk(x, wr, K)
    ws = B.Workspace.for_layer(layer, ntok, prefill=prefill)
    y, gu, dn, aq = B.moe_debug_ffn_blocksums(layer, _cuda(oq), _cuda(od), _cuda(oidx, torch.int32),
                                              _cuda(owts, torch.float32), ws, prefill=prefill)
    assert B.moe_check_status(ws) == 0
    y, gu, dn, aq = y.cpu().numpy(), gu.cpu().numpy(), dn.cpu().numpy(), aq.cpu().numpy()
    pairs = np.arange(ntok * K)
    if sample is not None and sample < len(pairs):
        pairs = np.sort(np.random.default_rng(seed).choice(pairs, sample, replace=False))
    toks = sorted(set(int(p) // K for p in pairs))
    olayer, remap = oracle_layer(orc, wl, fn, oidx[toks])
    _, dbg = orc.expert_ffn(olayer, oq[toks], od[toks], remap[oidx[toks]], owts[toks].astype(np.float32),
                            debug=True)
    compared = agreed = 0
    for p in pairs:
        t, j = divmod(int(p), K)
        e = remap[oidx[t, j]]
        qg, _ = orc.unpack_weights(*olayer.gate[:2], olayer.n_experts * F, H, e * F, F)
        qu, _ = orc.unpack_weights(*olayer.up[:2], olayer.n_experts * F, H, e * F, F)
        qd, _ = orc.unpack_weights(*olayer.down[:2], olayer.n_experts * H, F, e * H, H)
        assert np.array_equal(gu[p, 0], orc.blocksums(qg, oq[t])), "gate block sums, pair %d" % p
        assert np.array_equal(gu[p, 1], orc.blocksums(qu, oq[t])), "up block sums, pair %d" % p
        ao = dbg["aq"][toks.index(t), j]
        ref = orc.blocksums(qd, ao)
        same = np.all(aq[p].reshape(-1, 32) == ao.reshape(-1, 32), axis=1)
        compared += same.size
        agreed += int(same.sum())
        assert np.array_equal(dn[p][:, same], ref[:, same]), "down block sums, pair %d" % p
    assert agreed >= 0.9 * compared, "only %d of %d SwiGLU code blocks agree" % (agreed, compared)
    return y, oq, od, oidx, owts


@pytest.mark.parametrize("name,ntok,sample", [("tiny", 1, None), ("tiny", 3, None), ("tiny", 17, None),
                                              ("30b-b16", 16, 24), ("large-b8", 8, 4)])
def test_tc_decode_blocksums_exact(orc, name, ntok, sample):
    B = bm()
    wl = synthetic.WORKLOADS[name]
    layer, fn = gpu_layer(wl)
    wr = synthetic.router(wl, 0)
    x = synthetic.activations(wl, 60, ntok=ntok).numpy()
    _check_blocksums(orc, B, wl, layer, fn, x, wr.numpy(), sample=sample, seed=ntok)


def test_tc_decode_blocksums_extreme_codes(orc):
    """All-(+-1) ternary weights against +-127 activation codes: every gate/up
    block sum reaches |sum| = 32 * 127."""
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    H, F, E = wl.hidden, wl.ffn, wl.n_experts

    def fn(role, e):
        rows, k = (H, F) if role == "down" else (F, H)
        w = torch.ones((rows, k), dtype=torch.float32, device="cuda")
        w[(e + (role == "up")) % 2::2] *= -1
        return w * 0.02

    from bit_moe_b200.layers import quantize_layer
    layer = quantize_layer(H, F, E, wl.top_k, fn)
    wr = synthetic.router(wl, 0).numpy()
    x = np.full((2, H), 127.0, np.float32)
    x[:, 1::3] *= -1
    x[1] *= -1
    y, oq, _, _, _ = _check_blocksums(orc, B, wl, layer, fn, x, wr)
    assert np.abs(oq).min() == 127


@pytest.mark.parametrize("ntok", [2, 5])
def test_tc_decode_layer_and_singles(orc, ntok):
    """The tensor-core decode of a batch against the oracle (every token), and
    bit for bit against the same tokens one at a time through the one-token
    step (same block split and fp32 summation order)."""
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, fn = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 70 + ntok, ntok=ntok, device="cuda")
    ws = B.Workspace.for_layer(layer, ntok)
    yb = B.moe_forward(layer, wr, x, ws).cpu().numpy()
    assert B.moe_check_status(ws) == 0
    for t in range(ntok):
        ws1 = B.Workspace.for_layer(layer, 1)
        ys = B.moe_forward(layer, wr, x[t:t + 1].contiguous(), ws1).cpu().numpy()
        assert np.array_equal(ys[0], yb[t]), "token %d" % t
    xc = x.cpu().numpy()
    oidx, _ = orc.route_topk(xc, wr.cpu().numpy(), wl.top_k)
    olayer, remap = oracle_layer(orc, wl, fn, oidx)
    oq, od = orc.quant_act_q8(xc)
    _, owts = orc.route_topk(xc, wr.cpu().numpy(), wl.top_k)
    ref = orc.expert_ffn(olayer, oq, od, remap[oidx], owts.astype(np.float32))
    assert rel_err_rms(yb, ref) <= LAYER_TOL


@pytest.mark.parametrize("name,ntok,sample", [("tiny", 65, None), ("tiny", 600, 48), ("30b", 160, 24)])
def test_tc_prefill_blocksums_exact(orc, name, ntok, sample):
    """The prefill GEMM's int32 accumulators (128-pair groups, full and
    ragged): every sampled pair's gate/up and down block sums bit for bit."""
    B = bm()
    wl = synthetic.WORKLOADS[name]
    layer, fn = gpu_layer(wl)
    wr = synthetic.router(wl, 0)
    x = synthetic.activations(wl, 61, ntok=ntok).numpy()
    y, oq, od, oidx, owts = _check_blocksums(orc, B, wl, layer, fn, x, wr.numpy(), sample=sample, prefill=True,
                                             seed=ntok)
    toks = np.arange(min(ntok, 6))
    olayer, remap = oracle_layer(orc, wl, fn, oidx[toks])
    ref = orc.expert_ffn(olayer, oq[toks], od[toks], remap[oidx[toks]], owts[toks].astype(np.float32))
    assert rel_err_rms(y[toks], ref) <= LAYER_TOL


def test_tc_prefill_blocksums_extreme_codes(orc):
    """+-127 codes against all-(+-1) weights through the prefill GEMM."""
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    H, F, E = wl.hidden, wl.ffn, wl.n_experts

    def fn(role, e):
        rows, k = (H, F) if role == "down" else (F, H)
        w = torch.ones((rows, k), dtype=torch.float32, device="cuda")
        w[(e + (role == "up")) % 2::2] *= -1
        return w * 0.02

    from bit_moe_b200.layers import quantize_layer
    layer = quantize_layer(H, F, E, wl.top_k, fn)
    wr = synthetic.router(wl, 0).numpy()
    x = np.full((70, H), 127.0, np.float32)
    x[:, 1::3] *= -1
    x[1::2] *= -1
    _check_blocksums(orc, B, wl, layer, fn, x, wr, prefill=True)
