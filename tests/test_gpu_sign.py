"""Parity of the 1-bit sign-code format (MOE_FORMAT_SIGN) on the CUDA path
with the CPU oracle: packed codes and scales bit-exact, int32 block sums
bit-exact, mat-vec outputs within 1e-5 of max(|ref|, RMS(ref)) elementwise,
layer outputs within 2e-3 * RMS(ref) (the prefill GEMM on this format:
test_gpu_prefill_formats.py)."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, elementwise_rel, gpu_layer, oracle_layer, rel_err_rms

pytestmark = pytest.mark.gpu

MATVEC_TOL = 1e-5
LAYER_TOL = 2e-3


@pytest.mark.parametrize("rows,k", [(32, 256), (64, 768), (96, 2048), (32, 4096)])
def test_sign_quantize_bytes(orc, rows, k):
    B = bm()
    g = np.random.default_rng(rows * 11 + k)
    w = (g.standard_normal((rows, k)) * 0.02).astype(np.float32)
    w[0, :256] = 0.0                      # all zero: codes +1, scale 0
    w[1, :7] = -0.0                       # negative zeros code +1
    m = B.moe_quantize_weights_sign(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    codes, scales = orc.quantize_weights_sign(w)
    assert np.array_equal(m.trits.cpu().numpy().view(np.uint32), codes)
    assert np.array_equal(m.scales.cpu().numpy().view(np.uint16), scales)


@pytest.mark.parametrize("rows,k,ntok", [(64, 512, 1), (96, 2048, 3), (32, 4096, 8)])
def test_sign_matvec_blocksums_and_outputs(orc, rows, k, ntok):
    B = bm()
    g = np.random.default_rng(rows + k + ntok)
    w = (g.standard_normal((rows, k)) * 0.02).astype(np.float32)
    x = g.standard_normal((ntok, k)).astype(np.float32)
    m = B.moe_quantize_weights_sign(torch.from_numpy(w).cuda())
    xq, xd = orc.quant_act_q8(x)
    out, isum = B.moe_debug_matvec(m, torch.from_numpy(xq).cuda(), torch.from_numpy(xd).cuda())
    torch.cuda.synchronize()
    codes, scales = orc.quantize_weights_sign(w)
    q, s = orc.unpack_weights_sign(codes, scales, rows, k)
    isum = isum.cpu().numpy()
    out = out.cpu().numpy()
    for t in range(ntok):
        assert np.array_equal(isum[t], orc.blocksums(q, xq[t]))
        assert elementwise_rel(out[t], orc.matvec(q, s, xq[t], xd[t])) <= MATVEC_TOL


def test_sign_matvec_extreme_codes(orc):
    """Activations at +-127 and weights all negative or all positive: the
    block sums are bit-exact and reach +-32*127 where the codes agree."""
    B = bm()
    rows, k = 32, 512
    w = np.where(np.arange(rows)[:, None] % 2 == 0, 1.0, -1.0).astype(np.float32) * np.ones((1, k), np.float32)
    # the first 256 activations all +1 (codes +127), the rest a +-1 pattern
    x = np.where((np.arange(k) < 256) | (np.arange(k) % 3 == 0), 1.0, -1.0).astype(np.float32)[None, :]
    m = B.moe_quantize_weights_sign(torch.from_numpy(w).cuda())
    xq, xd = orc.quant_act_q8(x)
    _, isum = B.moe_debug_matvec(m, torch.from_numpy(xq).cuda(), torch.from_numpy(xd).cuda())
    torch.cuda.synchronize()
    codes, scales = orc.quantize_weights_sign(w)
    q, _ = orc.unpack_weights_sign(codes, scales, rows, k)
    assert np.array_equal(isum.cpu().numpy()[0], orc.blocksums(q, xq[0]))
    assert np.abs(isum.cpu().numpy()).max() == 32 * 127


def _layer_parity(orc, wl, ntok, seed, rows, chunk=None):
    B = bm()
    layer, fn = gpu_layer(wl, fmt="sign")
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
        olayer, remap = oracle_layer(orc, wl, fn, oidx, fmt="sign")
        xq, xd = orc.quant_act_q8(xs)
        refs.append(orc.expert_ffn(olayer, xq, xd, remap[oidx], owts.astype(np.float32)))
    return y[rows], np.concatenate(refs)


@pytest.mark.parametrize("ntok", [1, 2, 8])
def test_sign_layer_tiny(orc, ntok):
    y, ref = _layer_parity(orc, synthetic.WORKLOADS["tiny"], ntok, 31, np.arange(ntok))
    assert rel_err_rms(y, ref) <= LAYER_TOL


@pytest.mark.parametrize("ntok", [1, 16])
def test_sign_layer_30b(orc, ntok):
    rows = np.arange(ntok)  # every token
    y, ref = _layer_parity(orc, synthetic.WORKLOADS["30b"], ntok, 32, rows)
    assert rel_err_rms(y, ref) <= LAYER_TOL


@pytest.mark.parametrize("ntok", [1, 8])
def test_sign_layer_large(orc, ntok):
    """The large layer (hidden 4096, ffn 2048, 256 experts, top-8) at one
    token (the fused one-token step) and at 8 tokens, the shape the benchmark
    times: every token, two at a time through the oracle."""
    y, ref = _layer_parity(orc, synthetic.WORKLOADS["large"], ntok, 34, np.arange(ntok), chunk=2)
    assert rel_err_rms(y, ref) <= LAYER_TOL


def test_sign_batch_equals_single_tokens():
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, _ = gpu_layer(wl, fmt="sign")
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 33, ntok=5, device="cuda")
    yb = B.moe_forward(layer, wr, x, B.Workspace.for_layer(layer, 5)).cpu().numpy()
    for t in range(5):
        ys = B.moe_forward(layer, wr, x[t:t + 1].contiguous(), B.Workspace.for_layer(layer, 1)).cpu().numpy()
        assert np.array_equal(ys[0], yb[t])


def test_sign_decode_entry_point(orc):
    """moe_expert_ffn_decode on a sign-code layer (1 and 4 tokens) equals
    moe_forward's routing of the same tokens (the prefill GEMM on this format
    is tested in test_gpu_prefill_formats.py)."""
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    layer, _ = gpu_layer(wl, fmt="sign")
    wr = synthetic.router(wl, 0, "cuda")
    for ntok in (1, 4):
        x = synthetic.activations(wl, 34, ntok=ntok, device="cuda")
        ws = B.Workspace.for_layer(layer, ntok)
        yf = B.moe_forward(layer, wr, x, ws).cpu().numpy()
        xq, xd = B.moe_quant_act_q8(x)
        idx, wts = B.moe_route_topk(x, wr, wl.top_k)
        yd = B.moe_expert_ffn_decode(layer, xq, xd, idx, wts, ws).cpu().numpy()
        assert B.moe_check_status(ws) == 0
        assert np.array_equal(yf, yd)
