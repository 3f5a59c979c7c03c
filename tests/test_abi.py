"""The C-ABI library loads on a machine without a GPU, exports every entry
point that include/bitmoe.h declares, and rejects bad arguments on the host
before touching a device."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from bit_moe_b200 import build
    build.build()
    import bit_moe_b200
    return bit_moe_b200, bit_moe_b200.lib()


def declared_functions():
    with open(os.path.join(ROOT, "include", "bitmoe.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_and_binding_agree():
    import bit_moe_b200
    assert set(declared_functions()) == set(bit_moe_b200.EXPORTS)


def test_library_exports_every_declared_symbol():
    _, L = _lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def test_host_side_validation_without_device():
    B, L = _lib()
    # null pointers are rejected before any device call
    rc = L.moe_quant_act_q8(None, 1, 256, None, None, None)
    assert rc == -1
    assert b"NULL" in L.moe_last_error()
    # shape limits
    assert L.moe_trit_words(64, 512) == 64 * 2 * 13
    assert L.moe_scale_count(64, 512) == 128
    assert L.moe_route_workspace_bytes(0, 8) == 0
    lay = B.moe_layer(256, 512, 8, 9, B.moe_tmat(), B.moe_tmat(), B.moe_tmat())
    assert L.moe_workspace_bytes(ctypes.byref(lay), 1, 0) == 0   # top_k > E
    lay = B.moe_layer(300, 512, 8, 2, B.moe_tmat(), B.moe_tmat(), B.moe_tmat())
    assert L.moe_workspace_bytes(ctypes.byref(lay), 1, 0) == 0   # hidden % 256
    rc = L.moe_check_status(None, None)
    assert rc == -1


def test_sign_format_host_side_without_device():
    B, L = _lib()
    assert L.moe_sign_words(64, 512) == 64 * 2 * 8
    assert L.moe_sign_words(0, 512) == 0
    # argument checks of the sign-code quantizer come before any device call
    rc = L.moe_quantize_weights_sign(None, 32, 256, None, None, None)
    assert rc == -1 and b"NULL" in L.moe_last_error()
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.c_void_p((ctypes.addressof(buf) + 15) & ~15)
    assert L.moe_quantize_weights_sign(p, 31, 256, p, p, None) == -2     # rows % 32
    assert L.moe_quantize_weights_sign(p, 32, 200, p, p, None) == -2     # k % 256
    # a layer whose matrices mix formats, or name an unknown one, is rejected
    def tm(rows, k, fmt):
        return B.moe_tmat(rows, k, p.value, p.value, fmt)
    mixed = B.moe_layer(256, 256, 2, 1, tm(512, 256, 1), tm(512, 256, 1), tm(512, 256, 0))
    x = ctypes.c_void_p(p.value)
    rc = L.moe_forward(ctypes.byref(mixed), x, 1, x, x, x, 1 << 30, None)
    assert rc == -1 and b"format" in L.moe_last_error()
    bad = B.moe_layer(256, 256, 2, 1, tm(512, 256, 7), tm(512, 256, 7), tm(512, 256, 7))
    rc = L.moe_forward(ctypes.byref(bad), x, 1, x, x, x, 1 << 30, None)
    assert rc == -1 and b"format" in L.moe_last_error()
    # the binding's struct matches the header's field order
    assert [f[0] for f in B.moe_tmat._fields_] == ["rows", "k", "trits", "scales", "format", "codes"]
    assert L.moe_e16_code_words(64, 512) == 64 * 2 * 2
    # a two-level-scale layer without its sub-scale codes is rejected
    nocodes = B.moe_layer(256, 256, 2, 1, tm(512, 256, 2), tm(512, 256, 2), tm(512, 256, 2))
    rc = L.moe_forward(ctypes.byref(nocodes), x, 1, x, x, x, 1 << 30, None)
    assert rc == -1 and b"codes" in L.moe_last_error()
    rc = L.moe_quantize_weights_e16(p, 32, 200, p, p, p, None)
    assert rc == -2


def test_shared_expert_host_side_without_device():
    B, L = _lib()
    s = B.moe_shared(256, 512, None, None, None, None, None, None)
    assert L.moe_shared_workspace_bytes(ctypes.byref(s), 4) > 0
    assert L.moe_shared_workspace_bytes(ctypes.byref(s), 0) == 0
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.c_void_p((ctypes.addressof(buf) + 15) & ~15)
    rc = L.moe_shared_ffn_add(ctypes.byref(s), 1, p, p, p, p, 1 << 20, None)
    assert rc == -1 and b"NULL" in L.moe_last_error()
    bad = B.moe_shared(300, 512, p.value, p.value, p.value, p.value, p.value, p.value)
    assert L.moe_shared_ffn_add(ctypes.byref(bad), 1, p, p, p, p, 1 << 20, None) == -2
    assert L.moe_quantize_weights_q8(p, 4, 48, p, p, None) == -2


@pytest.mark.skipif(torch.cuda.is_available(), reason="would launch kernels on the placeholder pointers")
def test_forward_host_long_sign_call_passes_the_format_checks():
    """A 65-token call on a sign-code layer takes the prefill GEMM: its
    arguments pass the host checks and the call stops only at the device
    check (no CUDA device here), having launched nothing."""
    B, L = _lib()
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.c_void_p((ctypes.addressof(buf) + 15) & ~15)

    def tm(rows, k, fmt):
        return B.moe_tmat(rows, k, p.value, p.value, fmt, p.value)
    lay = B.moe_layer(256, 256, 2, 1, tm(512, 256, 1), tm(512, 256, 1), tm(512, 256, 1))
    n0 = L.moe_launch_count()
    rc = L.moe_forward_host(ctypes.byref(lay), p, 65, p, p, p, 1 << 30, None)
    assert rc in (-5, -8), L.moe_last_error()  # no usable device on this machine
    assert b"64 tokens" not in L.moe_last_error()
    assert L.moe_launch_count() == n0


def test_workspace_act_offsets():
    """The offsets of x's int8 codes and scales in a workspace: 256-byte
    aligned, past the header, inside the workspace, not overlapping; bad
    arguments refused."""
    B, L = _lib()
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.c_void_p((ctypes.addressof(buf) + 15) & ~15)

    def tm(rows, k):
        return B.moe_tmat(rows, k, p.value, p.value, 0, None)
    H, F, E, K = 2048, 768, 128, 8
    lay = B.moe_layer(H, F, E, K, tm(E * F, H), tm(E * F, H), tm(E * H, F))
    for ntok, prefill in ((1, 0), (16, 0), (2048, 1)):
        oq, od = ctypes.c_size_t(0), ctypes.c_size_t(0)
        assert L.moe_workspace_act(ctypes.byref(lay), ntok, prefill, ctypes.byref(oq), ctypes.byref(od)) == 0
        total = L.moe_workspace_bytes(ctypes.byref(lay), ntok, prefill)
        assert oq.value % 256 == 0 and od.value % 256 == 0 and oq.value >= 256
        assert oq.value + ntok * H <= od.value
        assert od.value + ntok * (H // 32) * 4 <= total
    oq, od = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert L.moe_workspace_act(ctypes.byref(lay), 0, 0, ctypes.byref(oq), ctypes.byref(od)) == -1
    assert L.moe_workspace_act(ctypes.byref(lay), 1, 0, None, ctypes.byref(od)) == -1
