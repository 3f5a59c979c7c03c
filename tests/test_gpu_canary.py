"""Guard canaries around every output and workspace of the entry points: each
buffer is the middle of a larger allocation whose margins hold a known byte
pattern, and after the call (and a synchronize) the margins must be intact.
A kernel that writes past the end (or before the start) of an output, a
workspace region or a packed weight array is caught here without a memory
checker (compute-sanitizer is not available on this machine's GPUs)."""
import numpy as np
import pytest
import torch

import synthetic
from gpu_helpers import bm, gpu_layer

pytestmark = pytest.mark.gpu

PAD = 4096  # bytes of canary on each side (a multiple of 256 keeps the middle aligned)
CANARY = 0xA5


class Guarded:
    """A tensor of `shape`/`dtype` inside a byte buffer with canary margins."""

    def __init__(self, shape, dtype, init=None):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((PAD + n + PAD,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[PAD:PAD + n].view(dtype).view(*shape)
        if init is not None:
            self.t.copy_(init)

    def intact(self):
        torch.cuda.synchronize()
        head = self.raw[:PAD].cpu().numpy()
        tail = self.raw[-PAD:].cpu().numpy()
        return bool((head == CANARY).all() and (tail == CANARY).all())


def _guarded_ws(B, layer, ntok, prefill=None):
    ws = B.Workspace.for_layer(layer, ntok, prefill=prefill)
    g = Guarded((ws.nbytes,), torch.uint8, ws.buf)
    ws.buf = g.t  # the library writes the workspace through ws.buf's pointer
    return ws, g


@pytest.mark.parametrize("name,ntok", [("tiny", 1), ("30b", 1), ("30b-b16", 16), ("30b", 5), ("tiny", 70),
                                       ("tiny", 200)])
def test_forward_writes_stay_inside_buffers(name, ntok):
    B = bm()
    wl = synthetic.WORKLOADS[name]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 95, ntok=ntok, device="cuda")
    ws, gws = _guarded_ws(B, layer, ntok)
    y = Guarded((ntok, wl.hidden), torch.float32)
    B.moe_forward(layer, wr, x, ws, y=y.t)
    assert B.moe_check_status(ws) == 0
    assert y.intact(), "y margins overwritten"
    assert gws.intact(), "workspace margins overwritten"
    assert np.isfinite(y.t.cpu().numpy()).all()


@pytest.mark.parametrize("ntok", [1, 3, 16])
def test_decode_entry_points_write_inside_buffers(ntok):
    B = bm()
    wl = synthetic.WORKLOADS["30b"]
    layer, _ = gpu_layer(wl)
    wr = synthetic.router(wl, 0, "cuda")
    x = synthetic.activations(wl, 96, ntok=ntok, device="cuda")
    xq = Guarded((ntok, wl.hidden), torch.int8)
    xd = Guarded((ntok, wl.hidden // 32), torch.float32)
    B.lib().moe_quant_act_q8(x.data_ptr(), ntok, wl.hidden, xq.t.data_ptr(), xd.t.data_ptr(), None)
    assert xq.intact() and xd.intact()
    idx, wts = B.moe_route_topk(x, wr, wl.top_k)
    ws, gws = _guarded_ws(B, layer, ntok, prefill=False)
    y = Guarded((ntok, wl.hidden), torch.float32)
    B.moe_expert_ffn_decode(layer, xq.t, xd.t, idx, wts, ws, y=y.t)
    assert B.moe_check_status(ws) == 0
    assert y.intact() and gws.intact()


def test_quantizers_write_inside_packed_arrays():
    B = bm()
    from bit_moe_b200 import TernaryMatrix, e16_code_words, packed_words, scale_words
    rows, k = 96, 768
    w = torch.randn(rows, k, device="cuda") * 0.02
    for fmt, fn in (("ternary", B.moe_quantize_weights), ("sign", B.moe_quantize_weights_sign),
                    ("e16", B.moe_quantize_weights_e16)):
        tr = Guarded((packed_words(rows, k, fmt),), torch.int32)
        sc = Guarded((scale_words(rows, k, fmt),), torch.int16)
        cd = Guarded((e16_code_words(rows, k),), torch.int32) if fmt == "e16" else None
        m = TernaryMatrix(rows, k, tr.t, sc.t, fmt, cd.t if cd is not None else None)
        fn(w, out=m)
        assert tr.intact() and sc.intact() and (cd is None or cd.intact()), fmt
