"""Packing a whole MoE layer: every expert's fp32 matrices quantized in place
into one packed matrix per role (through moe_quantize_weights, or
moe_quantize_weights_sign for 1-bit sign codes)."""
import torch

from . import (MoELayer, TernaryMatrix, moe_quantize_weights, moe_quantize_weights_sign, packed_words,
               scale_count)


def _expert_view(mat, e, rows_per_expert, k):
    tw, sc = packed_words(rows_per_expert, k, mat.fmt), scale_count(rows_per_expert, k)
    return TernaryMatrix(rows_per_expert, k, mat.trits[e * tw:(e + 1) * tw],
                         mat.scales[e * sc:(e + 1) * sc], mat.fmt)


def quantize_layer(hidden, ffn, n_experts, top_k, expert_fn, device="cuda", stream=None, fmt="ternary"):
    """expert_fn(role, e) -> fp32 CUDA tensor, [ffn][hidden] for "gate"/"up"
    and [hidden][ffn] for "down".  Experts are quantized one at a time, so the
    fp32 weights of only one expert are alive at once.  fmt: "ternary" or
    "sign"."""
    quant = moe_quantize_weights_sign if fmt == "sign" else moe_quantize_weights
    gate = TernaryMatrix.empty(n_experts * ffn, hidden, device, fmt)
    up = TernaryMatrix.empty(n_experts * ffn, hidden, device, fmt)
    down = TernaryMatrix.empty(n_experts * hidden, ffn, device, fmt)
    for e in range(n_experts):
        for role, mat, rows, k in (("gate", gate, ffn, hidden), ("up", up, ffn, hidden),
                                   ("down", down, hidden, ffn)):
            w = expert_fn(role, e)
            assert w.shape == (rows, k) and w.dtype == torch.float32
            quant(w.contiguous(), out=_expert_view(mat, e, rows, k), stream=stream)
    return MoELayer(hidden, ffn, n_experts, top_k, gate, up, down)
