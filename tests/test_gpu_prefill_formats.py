"""The prefill GEMM (tcgen05, exact int32 block sums) on the two other weight
formats: 1-bit sign codes (pxq_llama README, "What's PXQ?": the PXQ1 tier)
and ternary digits with two-level (E16) scales (the same page: a per-row
anchor and a 4-bit sub-scale per 16 weights).

- the gate and up rows' exact block sums of every pair (through
  moe_debug_ffn_blocksums) bit for bit against the oracle's own quantization
  of the same fp32 weights and its own int8 codes (for two-level scales the
  sum over the block's 16-weight halves of (c + 1) * sum(q * a));
- layer outputs within 2e-3 * RMS of the oracle on every token of ragged
  prefills of the tiny layer, and on a sample of a 300-token prefill of the
  30B-class layer;
- prefill within 1e-4 * RMS of the decode path on the same inputs."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, gpu_layer, oracle_layer, rel_err_rms

pytestmark = pytest.mark.gpu

LAYER_TOL = 2e-3
FORMATS = ["sign", "e16"]


def _cuda(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.to(dtype) if dtype is not None else t).cuda()


def _rows_blocksums(orc, fmt, mat, rows_total, k, row0, nrows, xq):
    """Exact block sums of rows [row0, row0 + nrows) of an oracle matrix."""
    if fmt == "sign":
        q, _ = orc.unpack_weights_sign(mat[0], mat[1], rows_total, k, row0, nrows)
        return orc.blocksums(q, xq)
    trits, anchors, codes = mat
    q, s16 = orc.unpack_weights_e16(trits, codes, anchors, rows_total, k, row0, nrows)
    a = anchors[row0:row0 + nrows].view(np.float16).astype(np.float64)
    cp1 = np.rint(16 * s16.astype(np.float64) / np.where(a == 0, 1, a)[:, None])  # c + 1
    cp1[a == 0] = 1
    s16sum = (q.astype(np.int64) * xq.astype(np.int64)).reshape(nrows, k // 16, 16).sum(axis=2)
    return (cp1.astype(np.int64) * s16sum).reshape(nrows, k // 32, 2).sum(axis=2)


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("ntok", [70, 129])
def test_prefill_formats_gateup_blocksums_exact(orc, fmt, ntok):
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    layer, fn = gpu_layer(wl, fmt=fmt)
    K, H, F = wl.top_k, wl.hidden, wl.ffn
    x = synthetic.activations(wl, 80 + ntok, ntok=ntok).numpy()
    wr = synthetic.router(wl, 0).numpy()
    oq, od = orc.quant_act_q8(x)
    oidx, owts = orc.route_topk(x, wr, K)
    ws = B.Workspace.for_layer(layer, ntok, prefill=True)
    _, gu, _, _ = B.moe_debug_ffn_blocksums(layer, _cuda(oq), _cuda(od), _cuda(oidx, torch.int32),
                                            _cuda(owts, torch.float32), ws, prefill=True)
    assert B.moe_check_status(ws) == 0
    gu = gu.cpu().numpy()
    olayer, remap = oracle_layer(orc, wl, fn, fmt=fmt)
    n = olayer.n_experts
    for p in range(ntok * K):
        t, j = divmod(p, K)
        e = remap[oidx[t, j]]
        assert np.array_equal(gu[p, 0], _rows_blocksums(orc, fmt, olayer.gate, n * F, H, e * F, F, oq[t])), p
        assert np.array_equal(gu[p, 1], _rows_blocksums(orc, fmt, olayer.up, n * F, H, e * F, F, oq[t])), p


def _oracle_y(orc, wl, fn, fmt, x, wr, rows, chunk):
    refs = []
    for c0 in range(0, len(rows), chunk):  # only a chunk's experts in fp32 at once
        xs = x[rows[c0:c0 + chunk]]
        oidx, owts = orc.route_topk(xs, wr, wl.top_k)
        olayer, remap = oracle_layer(orc, wl, fn, oidx, fmt=fmt)
        xq, xd = orc.quant_act_q8(xs)
        refs.append(orc.expert_ffn(olayer, xq, xd, remap[oidx], owts.astype(np.float32)))
    return np.concatenate(refs)


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("ntok", [65, 97])
def test_prefill_formats_tiny_all_tokens(orc, fmt, ntok):
    B = bm()
    wl = synthetic.WORKLOADS["tiny"]
    layer, fn = gpu_layer(wl, fmt=fmt)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 90 + ntok, ntok=ntok, device="cuda")
    ws = B.Workspace.for_layer(layer, ntok)
    y = B.moe_forward(layer, wr, x, ws).cpu().numpy()
    assert B.moe_check_status(ws) == 0
    ref = _oracle_y(orc, wl, fn, fmt, x.cpu().numpy(), wr.cpu().numpy(), np.arange(ntok), ntok)
    assert rel_err_rms(y, ref) <= LAYER_TOL


@pytest.mark.parametrize("fmt", FORMATS)
def test_prefill_formats_30b_sampled(orc, fmt):
    """300 tokens through the 30B-class layer (about 19 pairs per expert):
    24 sampled tokens against the oracle, 6 at a time."""
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, fn = gpu_layer(wl, fmt=fmt)
    wr = synthetic.router(wl, 0, "cuda")
    ntok = 300
    x = synthetic.activations(wl, 99, ntok=ntok, device="cuda")
    ws = B.Workspace.for_layer(layer, ntok)
    y = B.moe_forward(layer, wr, x, ws).cpu().numpy()
    assert B.moe_check_status(ws) == 0
    rows = np.sort(np.random.default_rng(7).choice(ntok, 24, replace=False))
    ref = _oracle_y(orc, wl, fn, fmt, x.cpu().numpy(), wr.cpu().numpy(), rows, 6)
    assert rel_err_rms(y[rows], ref) <= LAYER_TOL


@pytest.mark.parametrize("fmt", FORMATS)
def test_prefill_formats_equal_decode(fmt):
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, _ = gpu_layer(wl, fmt=fmt)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 12, ntok=40, device="cuda")
    xq, xd = B.moe_quant_act_q8(x)
    idx, wts = B.moe_route_topk(x, wr, wl.top_k)
    ws = B.Workspace.for_layer(layer, 40, prefill=True)
    yd = B.moe_expert_ffn_decode(layer, xq, xd, idx, wts, ws).cpu().numpy()
    yp = B.moe_expert_ffn_prefill(layer, xq, xd, idx, wts, ws).cpu().numpy()
    assert B.moe_check_status(ws) == 0
    assert rel_err_rms(yp, yd) <= 1e-4
