"""CPU oracle for the ternary routed-expert MoE hot path (ctypes over oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It does not import the
product package and the product package does not import it; the two share only
the seeded input generators in ``synthetic``.

All arrays are numpy; every function copies its inputs to contiguous arrays of
the documented dtype, calls the C oracle, and returns fresh numpy arrays.
"""
import ctypes
import os

import numpy as np

from . import build as _build

BLOCK = 256
BLOCK_WORDS = 13
PANEL = 32
QBLOCK = 32

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        L.orc_f16_from_f64.restype = ctypes.c_uint16
        L.orc_f16_from_f64.argtypes = [ctypes.c_double]
        L.orc_f16_to_f32.restype = ctypes.c_float
        L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_trit_byte_encode.restype = ctypes.c_uint8
        L.orc_trit_byte_encode.argtypes = [p]
        L.orc_trit_byte_decode.restype = ctypes.c_int
        L.orc_trit_byte_decode.argtypes = [ctypes.c_uint8, p]
        for name in ("orc_trit_words", "orc_scale_count"):
            getattr(L, name).restype = i64
            getattr(L, name).argtypes = [i64, i64]
        L.orc_word_index.restype = i64
        L.orc_word_index.argtypes = [i64, i64, i64, ctypes.c_int]
        L.orc_scale_index.restype = i64
        L.orc_scale_index.argtypes = [i64, i64, i64]
        L.orc_quantize_weights.restype = ctypes.c_int
        L.orc_quantize_weights.argtypes = [p, i64, i64, p, p]
        L.orc_sign_words.restype = i64
        L.orc_sign_words.argtypes = [i64, i64]
        L.orc_sign_word_index.restype = i64
        L.orc_sign_word_index.argtypes = [i64, i64, i64, ctypes.c_int]
        L.orc_quantize_weights_sign.restype = ctypes.c_int
        L.orc_quantize_weights_sign.argtypes = [p, i64, i64, p, p]
        L.orc_unpack_weights_sign.restype = ctypes.c_int
        L.orc_unpack_weights_sign.argtypes = [p, p, i64, i64, i64, i64, p, p]
        L.orc_e16_code_words.restype = i64
        L.orc_e16_code_words.argtypes = [i64, i64]
        L.orc_e16_code_index.restype = i64
        L.orc_e16_code_index.argtypes = [i64, i64, i64, ctypes.c_int]
        L.orc_quantize_weights_e16.restype = ctypes.c_int
        L.orc_quantize_weights_e16.argtypes = [p, i64, i64, p, p, p]
        L.orc_unpack_weights_e16.restype = ctypes.c_int
        L.orc_unpack_weights_e16.argtypes = [p, p, p, i64, i64, i64, i64, p, p]
        L.orc_matvec_e16.restype = None
        L.orc_matvec_e16.argtypes = [p, p, i64, i64, p, p, p]
        L.orc_quantize_weights_q8.restype = ctypes.c_int
        L.orc_quantize_weights_q8.argtypes = [p, i64, i64, p, p]
        L.orc_matvec_q8.restype = None
        L.orc_matvec_q8.argtypes = [p, p, i64, i64, p, p, p]
        L.orc_shared_ffn.restype = ctypes.c_int
        L.orc_shared_ffn.argtypes = [i64, i64, p, p, p, p, p, p, i64, p, p, p]
        L.orc_unpack_weights.restype = ctypes.c_int
        L.orc_unpack_weights.argtypes = [p, p, i64, i64, i64, i64, p, p]
        L.orc_quant_act_q8.restype = ctypes.c_int
        L.orc_quant_act_q8.argtypes = [p, i64, i64, p, p]
        L.orc_blocksums.restype = None
        L.orc_blocksums.argtypes = [p, i64, i64, p, p]
        L.orc_matvec.restype = None
        L.orc_matvec.argtypes = [p, p, i64, i64, p, p, p]
        L.orc_router_logits.restype = ctypes.c_int
        L.orc_router_logits.argtypes = [p, p, i64, i64, i64, p]
        L.orc_route_topk.restype = ctypes.c_int
        L.orc_route_topk.argtypes = [p, p, i64, i64, i64, i64, p, p]
        L.orc_expert_ffn.restype = ctypes.c_int
        L.orc_expert_ffn.argtypes = [ctypes.POINTER(OrcLayer), i64, p, p, p, p, p, p, p, p, p]
        _lib = L
    return _lib


class OrcLayer(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int64), ("ffn", ctypes.c_int64),
        ("n_experts", ctypes.c_int64), ("top_k", ctypes.c_int64),
        ("gate_trits", ctypes.c_void_p), ("gate_scales", ctypes.c_void_p),
        ("up_trits", ctypes.c_void_p), ("up_scales", ctypes.c_void_p),
        ("down_trits", ctypes.c_void_p), ("down_scales", ctypes.c_void_p),
        ("format", ctypes.c_int64),
        ("gate_codes", ctypes.c_void_p), ("up_codes", ctypes.c_void_p),
        ("down_codes", ctypes.c_void_p),
    ]


FORMATS = {"ternary": 0, "sign": 1, "e16": 2}


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- binary16
def f16_from_f64(x):
    x = np.asarray(x, dtype=np.float64)
    f = lib().orc_f16_from_f64
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


def f16_to_f32(h):
    h = np.asarray(h, dtype=np.uint16)
    f = lib().orc_f16_to_f32
    return np.array([f(int(v)) for v in h.ravel()], dtype=np.float32).reshape(h.shape)


# ---------------------------------------------------------------- base-3 bytes
def trit_byte_encode(t):
    t = _c(t, np.int32)
    assert t.shape == (5,)
    return int(lib().orc_trit_byte_encode(_ptr(t)))


def trit_byte_decode(u):
    t = np.zeros(5, dtype=np.int32)
    rc = lib().orc_trit_byte_decode(int(u), _ptr(t))
    return None if rc else t


# ---------------------------------------------------------------- weights
def trit_words(rows, k):
    return int(lib().orc_trit_words(rows, k))


def scale_count(rows, k):
    return int(lib().orc_scale_count(rows, k))


def word_index(k, r, b, w):
    return int(lib().orc_word_index(k, r, b, w))


def scale_index(k, r, b):
    return int(lib().orc_scale_index(k, r, b))


def quantize_weights(w):
    """w [rows][k] fp32 -> (trits uint32 [rows*(k/256)*13], scales uint16 [rows*(k/256)])."""
    w = _c(w, np.float32)
    rows, k = w.shape
    trits = np.zeros(trit_words(rows, k), dtype=np.uint32)
    scales = np.zeros(scale_count(rows, k), dtype=np.uint16)
    rc = lib().orc_quantize_weights(_ptr(w), rows, k, _ptr(trits), _ptr(scales))
    if rc:
        raise ValueError("orc_quantize_weights: bad shape %r" % (w.shape,))
    return trits, scales


def unpack_weights(trits, scales, rows, k, row0=0, nrows=None):
    """-> (q int8 [nrows][k], s float32 [nrows][k/256])."""
    if nrows is None:
        nrows = rows - row0
    trits = _c(trits, np.uint32)
    scales = _c(scales, np.uint16)
    q = np.zeros((nrows, k), dtype=np.int8)
    s = np.zeros((nrows, k // BLOCK), dtype=np.float32)
    rc = lib().orc_unpack_weights(_ptr(trits), _ptr(scales), rows, k, row0, nrows, _ptr(q), _ptr(s))
    if rc:
        raise ValueError("orc_unpack_weights failed")
    return q, s


# ---------------------------------------------------------------- 1-bit sign codes
def sign_words(rows, k):
    return int(lib().orc_sign_words(rows, k))


def sign_word_index(k, r, b, w):
    return int(lib().orc_sign_word_index(k, r, b, w))


def quantize_weights_sign(w):
    """w [rows][k] fp32 -> (codes uint32 [rows*(k/256)*8], scales uint16 [rows*(k/256)])."""
    w = _c(w, np.float32)
    rows, k = w.shape
    codes = np.zeros(sign_words(rows, k), dtype=np.uint32)
    scales = np.zeros(scale_count(rows, k), dtype=np.uint16)
    if lib().orc_quantize_weights_sign(_ptr(w), rows, k, _ptr(codes), _ptr(scales)):
        raise ValueError("orc_quantize_weights_sign: bad shape %r" % (w.shape,))
    return codes, scales


def unpack_weights_sign(codes, scales, rows, k, row0=0, nrows=None):
    """-> (q int8 [nrows][k] in {-1, +1}, s float32 [nrows][k/256])."""
    if nrows is None:
        nrows = rows - row0
    codes = _c(codes, np.uint32)
    scales = _c(scales, np.uint16)
    q = np.zeros((nrows, k), dtype=np.int8)
    s = np.zeros((nrows, k // BLOCK), dtype=np.float32)
    if lib().orc_unpack_weights_sign(_ptr(codes), _ptr(scales), rows, k, row0, nrows, _ptr(q), _ptr(s)):
        raise ValueError("orc_unpack_weights_sign failed")
    return q, s


# ---------------------------------------------------------------- two-level scales (E16)
def e16_code_words(rows, k):
    return int(lib().orc_e16_code_words(rows, k))


def e16_code_index(k, r, b, u):
    return int(lib().orc_e16_code_index(k, r, b, u))


def quantize_weights_e16(w):
    """w [rows][k] fp32 -> (trits uint32 [rows*(k/256)*13], codes uint32
    [rows*(k/256)*2], anchors uint16 [rows])."""
    w = _c(w, np.float32)
    rows, k = w.shape
    trits = np.zeros(trit_words(rows, k), dtype=np.uint32)
    codes = np.zeros(e16_code_words(rows, k), dtype=np.uint32)
    anchors = np.zeros(rows, dtype=np.uint16)
    if lib().orc_quantize_weights_e16(_ptr(w), rows, k, _ptr(trits), _ptr(codes), _ptr(anchors)):
        raise ValueError("orc_quantize_weights_e16: bad shape %r" % (w.shape,))
    return trits, codes, anchors


def unpack_weights_e16(trits, codes, anchors, rows, k, row0=0, nrows=None):
    """-> (q int8 [nrows][k], s16 float32 [nrows][k/16])."""
    if nrows is None:
        nrows = rows - row0
    trits, codes, anchors = _c(trits, np.uint32), _c(codes, np.uint32), _c(anchors, np.uint16)
    q = np.zeros((nrows, k), dtype=np.int8)
    s16 = np.zeros((nrows, k // 16), dtype=np.float32)
    if lib().orc_unpack_weights_e16(_ptr(trits), _ptr(codes), _ptr(anchors), rows, k, row0, nrows,
                                    _ptr(q), _ptr(s16)):
        raise ValueError("orc_unpack_weights_e16 failed")
    return q, s16


def matvec_e16(q, s16, xq, xd):
    """fp64 [rows]: sum_j xd_j * sum_{16-blocks h of j} s16[h] * sum_{k in h} q*xq."""
    q = _c(q, np.int8)
    s16 = _c(s16, np.float32)
    rows, k = q.shape
    out = np.zeros(rows, dtype=np.float64)
    lib().orc_matvec_e16(_ptr(q), _ptr(s16), rows, k, _ptr(_c(xq, np.int8)), _ptr(_c(xd, np.float32)), _ptr(out))
    return out


# ---------------------------------------------------------------- shared expert (q8 blocks)
def quantize_weights_q8(w):
    """w [rows][k] fp32 -> (q int8 [rows][k], d uint16 fp16 bits [rows][k/32])."""
    w = _c(w, np.float32)
    rows, k = w.shape
    q = np.zeros((rows, k), dtype=np.int8)
    d = np.zeros((rows, k // QBLOCK), dtype=np.uint16)
    if lib().orc_quantize_weights_q8(_ptr(w), rows, k, _ptr(q), _ptr(d)):
        raise ValueError("orc_quantize_weights_q8: bad shape %r" % (w.shape,))
    return q, d


def matvec_q8(q, d, xq, xd):
    q, d = _c(q, np.int8), _c(d, np.uint16)
    rows, k = q.shape
    out = np.zeros(rows, dtype=np.float64)
    lib().orc_matvec_q8(_ptr(q), _ptr(d), rows, k, _ptr(_c(xq, np.int8)), _ptr(_c(xd, np.float32)), _ptr(out))
    return out


class SharedExpert:
    """The shared expert in q8 blocks: gate/up [ffn][hidden], down [hidden][ffn]."""

    def __init__(self, hidden, ffn, wg, wu, wd):
        self.hidden, self.ffn = hidden, ffn
        self.gate, self.up, self.down = quantize_weights_q8(wg), quantize_weights_q8(wu), quantize_weights_q8(wd)

    def add_to(self, y, xq, xd):
        """y [ntok][hidden] fp64 += the shared expert's FFN of the tokens."""
        xq, xd = _c(xq, np.int8), _c(xd, np.float32)
        if xq.ndim == 1:
            xq, xd = xq[None], xd[None]
        y = np.ascontiguousarray(y, dtype=np.float64)
        (gq, gd), (uq, ud), (dq, dd) = self.gate, self.up, self.down
        rc = lib().orc_shared_ffn(self.hidden, self.ffn, _ptr(gq), _ptr(gd), _ptr(uq), _ptr(ud), _ptr(dq),
                                  _ptr(dd), xq.shape[0], _ptr(xq), _ptr(xd), _ptr(y))
        if rc:
            raise ValueError("orc_shared_ffn: bad shape")
        return y


# ---------------------------------------------------------------- activations
def quant_act_q8(x):
    """x [ntok][k] fp32 -> (xq int8 [ntok][k], xd fp32 [ntok][k/32])."""
    x = _c(x, np.float32)
    if x.ndim == 1:
        x = x[None, :]
    ntok, k = x.shape
    xq = np.zeros((ntok, k), dtype=np.int8)
    xd = np.zeros((ntok, k // QBLOCK), dtype=np.float32)
    rc = lib().orc_quant_act_q8(_ptr(x), ntok, k, _ptr(xq), _ptr(xd))
    if rc:
        raise ValueError("orc_quant_act_q8: k must be a multiple of 32")
    return xq, xd


def blocksums(q, xq):
    """q [rows][k] int8 ternary, xq [k] int8 -> isum int32 [rows][k/32]."""
    q = _c(q, np.int8)
    xq = _c(xq, np.int8).ravel()
    rows, k = q.shape
    isum = np.zeros((rows, k // QBLOCK), dtype=np.int32)
    lib().orc_blocksums(_ptr(q), rows, k, _ptr(xq), _ptr(isum))
    return isum


def matvec(q, s, xq, xd):
    """fp64 out [rows] = sum_b s[r][b] * sum_j xd[j] * isum[r][j]."""
    q = _c(q, np.int8)
    s = _c(s, np.float32)
    xq = _c(xq, np.int8).ravel()
    xd = _c(xd, np.float32).ravel()
    rows, k = q.shape
    out = np.zeros(rows, dtype=np.float64)
    lib().orc_matvec(_ptr(q), _ptr(s), rows, k, _ptr(xq), _ptr(xd), _ptr(out))
    return out


# ---------------------------------------------------------------- router
def router_logits(x, wr):
    x = _c(x, np.float32)
    if x.ndim == 1:
        x = x[None, :]
    wr = _c(wr, np.float32)
    ntok, hidden = x.shape
    E = wr.shape[0]
    lg = np.zeros((ntok, E), dtype=np.float32)
    if lib().orc_router_logits(_ptr(x), _ptr(wr), ntok, hidden, E, _ptr(lg)):
        raise ValueError("orc_router_logits: hidden must be a multiple of 32")
    return lg


def route_topk(x, wr, top_k):
    """-> (idx int32 [ntok][k], wts float64 [ntok][k])."""
    x = _c(x, np.float32)
    if x.ndim == 1:
        x = x[None, :]
    wr = _c(wr, np.float32)
    ntok, hidden = x.shape
    E = wr.shape[0]
    idx = np.zeros((ntok, top_k), dtype=np.int32)
    wts = np.zeros((ntok, top_k), dtype=np.float64)
    if lib().orc_route_topk(_ptr(x), _ptr(wr), ntok, hidden, E, top_k, _ptr(idx), _ptr(wts)):
        raise ValueError("orc_route_topk: bad arguments")
    return idx, wts


# ---------------------------------------------------------------- layer
class Layer:
    """A packed MoE layer in the storage format of orc_quantize_weights
    (fmt "ternary") or orc_quantize_weights_sign (fmt "sign").

    gate/up: rows E*ffn, k hidden; down: rows E*hidden, k ffn.  Expert e owns
    rows [e*ffn, (e+1)*ffn) of gate/up and [e*hidden, (e+1)*hidden) of down.
    """

    def __init__(self, hidden, ffn, n_experts, top_k, gate, up, down, fmt="ternary"):
        self.hidden, self.ffn, self.n_experts, self.top_k = hidden, ffn, n_experts, top_k
        self.fmt = fmt
        if fmt == "e16":  # (trits, codes, anchors): kept as (trits, anchors, codes)
            gate, up, down = [(m[0], m[2], m[1]) for m in (gate, up, down)]
        self.gate = (_c(gate[0], np.uint32), _c(gate[1], np.uint16)) + tuple(_c(m, np.uint32) for m in gate[2:])
        self.up = (_c(up[0], np.uint32), _c(up[1], np.uint16)) + tuple(_c(m, np.uint32) for m in up[2:])
        self.down = (_c(down[0], np.uint32), _c(down[1], np.uint16)) + tuple(_c(m, np.uint32) for m in down[2:])
        words = sign_words if fmt == "sign" else trit_words
        assert self.gate[0].size == words(n_experts * ffn, hidden)
        assert self.up[0].size == words(n_experts * ffn, hidden)
        assert self.down[0].size == words(n_experts * hidden, ffn)

    @classmethod
    def from_float(cls, hidden, ffn, n_experts, top_k, wg, wu, wd, fmt="ternary"):
        """wg, wu [E*ffn][hidden], wd [E*hidden][ffn] fp32."""
        quant = {"sign": quantize_weights_sign, "e16": quantize_weights_e16}.get(fmt, quantize_weights)
        return cls(hidden, ffn, n_experts, top_k, quant(wg), quant(wu), quant(wd), fmt=fmt)

    def c_struct(self, top_k=None):
        return OrcLayer(self.hidden, self.ffn, self.n_experts,
                        self.top_k if top_k is None else top_k,
                        _ptr(self.gate[0]).value, _ptr(self.gate[1]).value,
                        _ptr(self.up[0]).value, _ptr(self.up[1]).value,
                        _ptr(self.down[0]).value, _ptr(self.down[1]).value,
                        FORMATS[self.fmt],
                        *[(_ptr(m[2]).value if len(m) > 2 else None) for m in (self.gate, self.up, self.down)])


def expert_ffn(layer, xq, xd, idx, wts, debug=False):
    """y fp64 [ntok][hidden]; with debug=True also a dict of g, u, aq, ad."""
    xq = _c(xq, np.int8)
    xd = _c(xd, np.float32)
    idx = _c(idx, np.int32)
    wts = _c(wts, np.float32)
    if xq.ndim == 1:
        xq, xd = xq[None], xd[None]
    if idx.ndim == 1:
        idx, wts = idx[None], wts[None]
    ntok = xq.shape[0]
    K = idx.shape[1]
    H, F = layer.hidden, layer.ffn
    y = np.zeros((ntok, H), dtype=np.float64)
    dbg = None
    ptrs = [None] * 4
    if debug:
        dbg = dict(g=np.zeros((ntok, K, F)), u=np.zeros((ntok, K, F)),
                   aq=np.zeros((ntok, K, F), dtype=np.int8),
                   ad=np.zeros((ntok, K, F // QBLOCK), dtype=np.float32))
        ptrs = [_ptr(dbg[n]) for n in ("g", "u", "aq", "ad")]
    st = layer.c_struct(top_k=K)
    rc = lib().orc_expert_ffn(ctypes.byref(st), ntok, _ptr(xq), _ptr(xd), _ptr(idx),
                              _ptr(wts), _ptr(y), *ptrs)
    if rc == -2:
        raise IndexError("orc_expert_ffn: expert id out of range")
    if rc:
        raise ValueError("orc_expert_ffn: bad shape")
    return (y, dbg) if debug else y


def moe_forward(layer, wr, x, debug=False, shared=None):
    """The whole decode step on the CPU: act quant, router, expert FFN, and
    the shared expert's FFN added when `shared` (a SharedExpert) is given.

    Returns y fp64 [ntok][hidden], idx, wts (fp64) and, with debug, the
    intermediates.
    """
    xq, xd = quant_act_q8(x)
    idx, wts = route_topk(x, wr, layer.top_k)
    out = expert_ffn(layer, xq, xd, idx, wts.astype(np.float32), debug=debug)
    y = out[0] if debug else out
    if shared is not None:
        y = shared.add_to(y, xq, xd)
    if debug:
        dbg = out[1]
        dbg.update(xq=xq, xd=xd)
        return y, idx, wts, dbg
    return y, idx, wts
