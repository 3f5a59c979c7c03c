"""Parity of the two-level-scale format (MOE_FORMAT_E16: ternary digits with
an fp16 anchor per row and a 4-bit sub-scale per 16 weights) on the CUDA path
with the CPU oracle: digits, codes and anchors bit-exact, the weighted int32
block sums bit-exact, mat-vec outputs within 1e-5 of max(|ref|, RMS(ref))
elementwise, layer outputs within 2e-3 * RMS(ref) (the prefill GEMM on this
format: test_gpu_prefill_formats.py)."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, elementwise_rel, gpu_layer, oracle_layer, rel_err_rms

pytestmark = pytest.mark.gpu

MATVEC_TOL = 1e-5
LAYER_TOL = 2e-3


def _weights(rows, k, seed):
    g = np.random.default_rng(seed)
    w = (g.standard_normal((rows, k)) * 0.02).astype(np.float32)
    w[0] = 0.0                                   # all-zero row: anchor 0
    w[1, :16] *= 40.0                            # one dominant 16-block
    return w


@pytest.mark.parametrize("rows,k", [(32, 256), (64, 768), (96, 2048), (32, 4096)])
def test_e16_quantize_bytes(orc, rows, k):
    B = bm()
    w = _weights(rows, k, rows * 13 + k)
    m = B.moe_quantize_weights_e16(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    trits, codes, anchors = orc.quantize_weights_e16(w)
    assert np.array_equal(m.trits.cpu().numpy().view(np.uint32), trits)
    assert np.array_equal(m.codes.cpu().numpy().view(np.uint32), codes)
    assert np.array_equal(m.scales.cpu().numpy().view(np.uint16), anchors)


@pytest.mark.parametrize("rows,k,ntok", [(64, 512, 1), (96, 2048, 3), (32, 4096, 8)])
def test_e16_matvec_blocksums_and_outputs(orc, rows, k, ntok):
    B = bm()
    w = _weights(rows, k, rows + k + ntok)
    x = np.random.default_rng(ntok).standard_normal((ntok, k)).astype(np.float32)
    m = B.moe_quantize_weights_e16(torch.from_numpy(w).cuda())
    xq, xd = orc.quant_act_q8(x)
    out, isum = B.moe_debug_matvec(m, torch.from_numpy(xq).cuda(), torch.from_numpy(xd).cuda())
    torch.cuda.synchronize()
    trits, codes, anchors = orc.quantize_weights_e16(w)
    q, s16 = orc.unpack_weights_e16(trits, codes, anchors, rows, k)
    a = anchors.view(np.float16).astype(np.float64)
    cp1 = np.rint(16 * s16.astype(np.float64) / np.where(a == 0, 1, a)[:, None])   # c + 1
    cp1[a == 0] = 1
    isum = isum.cpu().numpy()
    out = out.cpu().numpy()
    for t in range(ntok):
        s16sum = (q.astype(np.int64) * xq[t].astype(np.int64)).reshape(rows, k // 16, 16).sum(axis=2)
        ref_isum = (cp1.astype(np.int64) * s16sum).reshape(rows, k // 32, 2).sum(axis=2)
        assert np.array_equal(isum[t], ref_isum)
        assert elementwise_rel(out[t], orc.matvec_e16(q, s16, xq[t], xd[t])) <= MATVEC_TOL


def _layer_parity(orc, wl, ntok, seed, rows, chunk=None):
    B = bm()
    layer, fn = gpu_layer(wl, fmt="e16")
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, seed, ntok=ntok, device="cuda")
    ws = B.Workspace.for_layer(layer, ntok)
    y = B.moe_forward(layer, wr, x, ws).cpu().numpy()
    assert B.moe_check_status(ws) == 0
    rows = np.asarray(rows)
    chunk = len(rows) if chunk is None else chunk
    refs = []
    for c0 in range(0, len(rows), chunk):  # only a chunk's experts in fp32 at once
        xs = x.cpu().numpy()[rows[c0:c0 + chunk]]
        oidx, owts = orc.route_topk(xs, wr.cpu().numpy(), wl.top_k)
        olayer, remap = oracle_layer(orc, wl, fn, oidx, fmt="e16")
        xq, xd = orc.quant_act_q8(xs)
        refs.append(orc.expert_ffn(olayer, xq, xd, remap[oidx], owts.astype(np.float32)))
    return y[rows], np.concatenate(refs)


@pytest.mark.parametrize("ntok", [1, 2, 8])
def test_e16_layer_tiny(orc, ntok):
    y, ref = _layer_parity(orc, synthetic.WORKLOADS["tiny"], ntok, 51, np.arange(ntok))
    assert rel_err_rms(y, ref) <= LAYER_TOL


@pytest.mark.parametrize("ntok", [1, 16])
def test_e16_layer_30b(orc, ntok):
    rows = np.arange(ntok)  # every token
    y, ref = _layer_parity(orc, synthetic.WORKLOADS["30b"], ntok, 52, rows)
    assert rel_err_rms(y, ref) <= LAYER_TOL


@pytest.mark.parametrize("ntok", [1, 8])
def test_e16_layer_large(orc, ntok):
    """The large layer (hidden 4096, ffn 2048, 256 experts, top-8) at 1 token
    (the one-token step with one ring slot per warp) and 8 tokens, the shape
    the benchmark times: every token, two at a time through the oracle."""
    y, ref = _layer_parity(orc, synthetic.WORKLOADS["large"], ntok, 54, np.arange(ntok), chunk=2)
    assert rel_err_rms(y, ref) <= LAYER_TOL


def test_e16_batch_equals_single_tokens():
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, _ = gpu_layer(wl, fmt="e16")
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 53, ntok=5, device="cuda")
    yb = B.moe_forward(layer, wr, x, B.Workspace.for_layer(layer, 5)).cpu().numpy()
    for t in range(5):
        ys = B.moe_forward(layer, wr, x[t:t + 1].contiguous(), B.Workspace.for_layer(layer, 1)).cpu().numpy()
        assert np.array_equal(ys[0], yb[t])


def test_e16_large_batch_equals_single_tokens():
    """The large layer: 3 tokens through the grouped kernels, each bit for bit
    the same token alone through the one-token step."""
    B = bm()
    wl = synthetic.WORKLOADS["large"]
    layer, _ = gpu_layer(wl, fmt="e16")
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 55, ntok=3, device="cuda")
    yb = B.moe_forward(layer, wr, x, B.Workspace.for_layer(layer, 3)).cpu().numpy()
    for t in range(3):
        ys = B.moe_forward(layer, wr, x[t:t + 1].contiguous(), B.Workspace.for_layer(layer, 1)).cpu().numpy()
        assert np.array_equal(ys[0], yb[t])


def test_e16_decode_entry_point():
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    layer, _ = gpu_layer(wl, fmt="e16")
    wr = synthetic.router(wl, 0, "cuda")
    for ntok in (1, 4):
        x = synthetic.activations(wl, 54, ntok=ntok, device="cuda")
        ws = B.Workspace.for_layer(layer, ntok)
        yf = B.moe_forward(layer, wr, x, ws).cpu().numpy()
        xq, xd = B.moe_quant_act_q8(x)
        idx, wts = B.moe_route_topk(x, wr, wl.top_k)
        yd = B.moe_expert_ffn_decode(layer, xq, xd, idx, wts, ws).cpu().numpy()
        assert B.moe_check_status(ws) == 0
        assert np.array_equal(yf, yd)
