"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle side.

This module holds no arithmetic of the method: it only draws Gaussian numbers.
It is the one module both the CUDA path's callers and the oracle's callers
use, so that both sides see the same inputs.

Every tensor is keyed by (seed, layer, role, expert) and drawn from its own
generator, so any expert of any layer can be regenerated alone.  Values depend
on the device they are drawn on (numpy's PCG64 on "cpu", torch's Philox on
"cuda"): a test draws once, on one device, and copies.

Workloads (the shapes, sizes and distributions of the MoE layers studied on the
pages; weights are random-init, not trained):
  moe-h256-f512-e8-k2       tiny layer, weights N(0, 0.02)
  moe-h2048-f768-e128-k8    30B-class layer, weights N(0, 0.02)
  moe-h4096-f2048-e256-k8   large layer, weights N(0, 0.015), 5-layer stack
Router weights N(0, 0.02); activations N(0, 1); a shared expert (where a
workload has one) N(0, w_std) like the routed experts.
"""
import hashlib
from dataclasses import dataclass, replace

import numpy as np
import torch

ROLE_IDS = {"gate": 1, "up": 2, "down": 3, "router": 4, "x": 5,
            "shared_gate": 6, "shared_up": 7, "shared_down": 8}


@dataclass(frozen=True)
class Workload:
    name: str
    hidden: int
    ffn: int
    n_experts: int
    top_k: int
    ntok: int
    w_std: float
    router_std: float = 0.02
    layers: int = 1          # layers in the stack the benchmark rotates through
    prefill: bool = False
    seed: int = 0
    fmt: str = "ternary"     # packed weight format: "ternary", "sign" (1-bit sign codes) or
                             # "e16" (ternary digits with two-level scales)
    shared_ffn: int = 0      # >0: a shared expert of this ffn width in 8-bit blocks beside the routed ones

    def with_(self, **kw):
        return replace(self, **kw)

    @property
    def block_bytes(self):
        """Packed bytes per 256 weights: 52 B of base-3 digits or 32 B of sign
        bits, plus the 2-byte scale (e16: 8 bytes of 4-bit sub-scales instead,
        the 2-byte anchor being per row)."""
        return {"sign": 34, "e16": 60}.get(self.fmt, 54)

    def matrix_bytes(self, rows, k):
        """Packed bytes of a [rows][k] matrix in this workload's format."""
        return rows * (k // 256) * self.block_bytes + (2 * rows if self.fmt == "e16" else 0)

    @property
    def expert_bytes(self):
        """Packed bytes of one expert's gate+up+down."""
        return 2 * self.matrix_bytes(self.ffn, self.hidden) + self.matrix_bytes(self.hidden, self.ffn)

    def describe(self):
        return "%s%s%s-t%d%s" % (self.name, "" if self.fmt == "ternary" else "-" + self.fmt,
                                 "-shared%d" % self.shared_ffn if self.shared_ffn else "", self.ntok,
                                 "-prefill" if self.prefill else "")


WORKLOADS = {
    # tiny layer, decode of 1 token
    "tiny": Workload("moe-h256-f512-e8-k2", 256, 512, 8, 2, 1, 0.02, seed=0),
    # 30B-class layer, decode of 1 token
    "30b": Workload("moe-h2048-f768-e128-k8", 2048, 768, 128, 8, 1, 0.02, layers=4, seed=1),
    # same layer, 16 independent tokens decoded together
    "30b-b16": Workload("moe-h2048-f768-e128-k8", 2048, 768, 128, 8, 16, 0.02, layers=4, seed=2),
    # large layer, decode of 1 token (and 8 with ntok=8), 5-layer stack
    "large": Workload("moe-h4096-f2048-e256-k8", 4096, 2048, 256, 8, 1, 0.015, layers=5, seed=3),
    "large-b8": Workload("moe-h4096-f2048-e256-k8", 4096, 2048, 256, 8, 8, 0.015, layers=5, seed=3),
    # the same layers with 1-bit sign codes instead of ternary digits
    "30b-sign": Workload("moe-h2048-f768-e128-k8", 2048, 768, 128, 8, 1, 0.02, layers=4, seed=5,
                         fmt="sign"),
    "large-sign-b8": Workload("moe-h4096-f2048-e256-k8", 4096, 2048, 256, 8, 8, 0.015, layers=5,
                              seed=6, fmt="sign"),
    # and with ternary digits under two-level (per-row anchor, per-16 sub-scale) scales
    "30b-e16": Workload("moe-h2048-f768-e128-k8", 2048, 768, 128, 8, 1, 0.02, layers=4, seed=7,
                        fmt="e16"),
    "large-e16-b8": Workload("moe-h4096-f2048-e256-k8", 4096, 2048, 256, 8, 8, 0.015, layers=5,
                             seed=8, fmt="e16"),
    "large-e16": Workload("moe-h4096-f2048-e256-k8", 4096, 2048, 256, 8, 1, 0.015, layers=6,
                          seed=8, fmt="e16"),
    # the 30B-class layer with a shared expert (ffn 768, 8-bit blocks) beside the routed ones
    "30b-shared": Workload("moe-h2048-f768-e128-k8", 2048, 768, 128, 8, 1, 0.02, layers=4, seed=1,
                           shared_ffn=768),
    # prefill of 2048 tokens through the 30B-class layer
    "30b-prefill": Workload("moe-h2048-f768-e128-k8", 2048, 768, 128, 8, 2048, 0.02,
                            layers=1, prefill=True, seed=4),
    # the same prefill on 1-bit sign codes and on two-level (E16) scales
    "30b-sign-prefill": Workload("moe-h2048-f768-e128-k8", 2048, 768, 128, 8, 2048, 0.02,
                                 layers=1, prefill=True, seed=9, fmt="sign"),
    "30b-e16-prefill": Workload("moe-h2048-f768-e128-k8", 2048, 768, 128, 8, 2048, 0.02,
                                layers=1, prefill=True, seed=10, fmt="e16"),
}


def subseed(*key) -> int:
    """A 63-bit seed derived from a key of ints/strings (stable across runs)."""
    h = hashlib.sha256(repr(tuple(key)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def gaussian(key, shape, std, device="cpu"):
    """fp32 N(0, std^2) tensor of `shape`, drawn from the generator of `key`."""
    s = subseed(*key)
    if str(device) == "cpu":
        rng = np.random.Generator(np.random.PCG64(s))
        a = rng.standard_normal(size=shape, dtype=np.float32)
        if std != 1.0:
            a *= np.float32(std)
        return torch.from_numpy(a)
    g = torch.Generator(device=device)
    g.manual_seed(s)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def expert_matrix(wl: Workload, layer: int, role: str, expert: int, device="cpu"):
    """One expert's fp32 matrix: gate/up [ffn][hidden], down [hidden][ffn]."""
    rows, k = (wl.hidden, wl.ffn) if role == "down" else (wl.ffn, wl.hidden)
    return gaussian((wl.seed, layer, ROLE_IDS[role], expert), (rows, k), wl.w_std, device)


def shared_matrix(wl: Workload, layer: int, role: str, device="cpu"):
    """The shared expert's fp32 matrix: gate/up [shared_ffn][hidden], down
    [hidden][shared_ffn]; role "gate", "up" or "down"."""
    rows, k = (wl.hidden, wl.shared_ffn) if role == "down" else (wl.shared_ffn, wl.hidden)
    return gaussian((wl.seed, layer, ROLE_IDS["shared_" + role], 0), (rows, k), wl.w_std, device)


def router(wl: Workload, layer: int, device="cpu"):
    """Dense fp32 router [n_experts][hidden]."""
    return gaussian((wl.seed, layer, ROLE_IDS["router"], 0), (wl.n_experts, wl.hidden),
                    wl.router_std, device)


def activations(wl: Workload, step: int, ntok=None, device="cpu"):
    """fp32 x [ntok][hidden] ~ N(0, 1) for decode step `step`."""
    n = wl.ntok if ntok is None else ntok
    return gaussian((wl.seed, step, ROLE_IDS["x"], n), (n, wl.hidden), 1.0, device)


def layer_float(wl: Workload, layer: int = 0, device="cpu"):
    """All experts' fp32 matrices stacked: (wg, wu [E*ffn][hidden], wd [E*hidden][ffn]).

    Only for layers small enough to hold in fp32 at once.
    """
    wg = torch.cat([expert_matrix(wl, layer, "gate", e, device) for e in range(wl.n_experts)])
    wu = torch.cat([expert_matrix(wl, layer, "up", e, device) for e in range(wl.n_experts)])
    wd = torch.cat([expert_matrix(wl, layer, "down", e, device) for e in range(wl.n_experts)])
    return wg, wu, wd
