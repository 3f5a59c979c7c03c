"""Packing a whole MoE layer: every expert's fp32 matrices quantized in place
into one packed matrix per role (through moe_quantize_weights, or
moe_quantize_weights_sign for 1-bit sign codes)."""
import torch

from . import (MoELayer, TernaryMatrix, e16_code_words, moe_quantize_weights, moe_quantize_weights_e16,
               moe_quantize_weights_sign, packed_words, scale_words)


def _expert_view(mat, e, rows_per_expert, k):
    tw, sc = packed_words(rows_per_expert, k, mat.fmt), scale_words(rows_per_expert, k, mat.fmt)
    codes = None
    if mat.codes is not None:
        cw = e16_code_words(rows_per_expert, k)
        codes = mat.codes[e * cw:(e + 1) * cw]
    return TernaryMatrix(rows_per_expert, k, mat.trits[e * tw:(e + 1) * tw],
                         mat.scales[e * sc:(e + 1) * sc], mat.fmt, codes)


def quantize_layer(hidden, ffn, n_experts, top_k, expert_fn, device="cuda", stream=None, fmt="ternary"):
    """expert_fn(role, e) -> fp32 CUDA tensor, [ffn][hidden] for "gate"/"up"
    and [hidden][ffn] for "down".  Experts are quantized one at a time, so the
    fp32 weights of only one expert are alive at once.  fmt: "ternary",
    "sign" or "e16"."""
    quant = {"sign": moe_quantize_weights_sign, "e16": moe_quantize_weights_e16}.get(fmt, moe_quantize_weights)
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
