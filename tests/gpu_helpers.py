"""Shared set-up of the GPU parity tests: build the library, make layers from
the seeded generator on the device, and the matching oracle layer from copies
of the same fp32 weights."""
import numpy as np
import pytest
import torch

import synthetic


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def bm():
    need_gpu()
    import bit_moe_b200
    from bit_moe_b200 import build
    build.build()
    bit_moe_b200.lib()
    return bit_moe_b200


def gpu_layer(wl, layer=0, fmt="ternary"):
    """(device MoELayer, fp32 generator) for workload `wl`, weights drawn on cuda."""
    from bit_moe_b200.layers import quantize_layer
    fn = lambda role, e: synthetic.expert_matrix(wl, layer, role, e, "cuda")  # noqa: E731
    return quantize_layer(wl.hidden, wl.ffn, wl.n_experts, wl.top_k, fn, fmt=fmt), fn


def oracle_layer(orc, wl, fn, experts=None, fmt="ternary"):
    """Oracle layer with the same fp32 weights (copied from the device), holding
    only `experts` (all if None) renumbered 0..n-1.  Returns (layer, remap)
    with remap[e] the compact id of expert e (-1 if absent)."""
    H, F, E = wl.hidden, wl.ffn, wl.n_experts
    keep = list(range(E)) if experts is None else sorted(set(int(v) for v in np.ravel(experts)))
    n = len(keep)
    wg = np.zeros((n * F, H), np.float32)
    wu = np.zeros((n * F, H), np.float32)
    wd = np.zeros((n * H, F), np.float32)
    remap = -np.ones(E, np.int32)
    for i, e in enumerate(keep):
        remap[e] = i
        wg[i * F:(i + 1) * F] = fn("gate", e).cpu().numpy()
        wu[i * F:(i + 1) * F] = fn("up", e).cpu().numpy()
        wd[i * H:(i + 1) * H] = fn("down", e).cpu().numpy()
    return orc.Layer.from_float(H, F, n, wl.top_k, wg, wu, wd, fmt=fmt), remap


def rel_err_rms(y, ref):
    """max |y - ref| / RMS(ref)."""
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(np.asarray(y, np.float64) - ref))) / rms


def elementwise_rel(y, ref):
    """max |y - ref| / max(|ref|, RMS(ref)) elementwise."""
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    den = np.maximum(np.abs(ref), rms)
    return float(np.max(np.abs(np.asarray(y, np.float64) - ref) / den))
