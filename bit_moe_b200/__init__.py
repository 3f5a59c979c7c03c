"""Python binding of libbitmoe (the sm_100a ternary MoE hot path).

Argument marshalling only: every function below checks the tensors it is
given, passes their device pointers to the C entry point of the same name
(declared in include/bitmoe.h) on the current torch CUDA stream, and raises
MoEError on a negative status.  All arithmetic runs in the CUDA kernels of
libbitmoe.so; there is no other implementation behind these functions.  If the
library has not been built, `lib()` raises instead of falling back.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitmoe.so")
CHECKED_LIB_PATH = os.path.join(_HERE, "libbitmoe_checked.so")  # -DMOE_CHECKED, for the tests

BLOCK = 256
BLOCK_WORDS = 13
PANEL = 32
QBLOCK = 32
MAX_DECODE_TOKENS = 64

STATUS = {
    0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED_SHAPE",
    -3: "MOE_ERR_ALIGNMENT", -4: "MOE_ERR_WORKSPACE", -5: "MOE_ERR_CUDA",
    -6: "MOE_ERR_TIMEOUT", -7: "MOE_ERR_BAD_INDEX", -8: "MOE_ERR_DEVICE", -9: "MOE_ERR_BOUNDS",
}

# every symbol include/bitmoe.h declares
EXPORTS = (
    "moe_trit_words", "moe_sign_words", "moe_scale_count", "moe_workspace_bytes", "moe_workspace_init",
    "moe_quantize_weights", "moe_quantize_weights_sign", "moe_quant_act_q8", "moe_route_topk", "moe_route_workspace_bytes",
    "moe_expert_ffn_decode", "moe_expert_ffn_prefill", "moe_forward", "moe_forward_host",
    "moe_check_status", "moe_last_error", "moe_debug_matvec", "moe_launch_count",
    "moe_trace_begin", "moe_trace_end", "moe_kernel_name", "moe_expert_ffn_decode_static",
    "moe_sign_words", "moe_quantize_weights_sign", "moe_e16_code_words", "moe_quantize_weights_e16",
    "moe_quantize_weights_q8", "moe_shared_workspace_bytes", "moe_shared_ffn_add", "moe_forward_shared",
    "moe_debug_ffn_blocksums", "moe_debug_wait_knob", "moe_workspace_act",
)


class MoEError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("%s (%d): %s" % (STATUS.get(code, "?"), code, msg))
        self.code = code


class moe_tmat(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int32), ("k", ctypes.c_int32),
                ("trits", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("format", ctypes.c_int32), ("codes", ctypes.c_void_p)]


FORMATS = {"ternary": 0, "sign": 1, "e16": 2}   # moe_format


class moe_shared(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("gate_q", ctypes.c_void_p), ("gate_d", ctypes.c_void_p),
                ("up_q", ctypes.c_void_p), ("up_d", ctypes.c_void_p),
                ("down_q", ctypes.c_void_p), ("down_d", ctypes.c_void_p)]


class moe_layer(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("gate", moe_tmat), ("up", moe_tmat), ("down", moe_tmat)]


_lib = None


def lib():
    """Load libbitmoe.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libbitmoe.so is not built (run `python -m bit_moe_b200.build`); "
                               "the ternary MoE path has no other implementation")
        _lib = load_library(LIB_PATH)
    return _lib


def load_library(path):
    """A ctypes handle of a build of the library at `path` (the normal build,
    or the bounds-checked one that the tests load), with every entry point's
    signature set."""
    L = ctypes.CDLL(path)
    p, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "moe_trit_words": (sz, [i64, i64]),
        "moe_sign_words": (sz, [i64, i64]),
        "moe_e16_code_words": (sz, [i64, i64]),
        "moe_scale_count": (sz, [i64, i64]),
        "moe_workspace_bytes": (sz, [p, i32, i32]),
        "moe_workspace_init": (ctypes.c_int, [p, sz, p]),
        "moe_quantize_weights": (ctypes.c_int, [p, i64, i64, p, p, p]),
        "moe_quantize_weights_sign": (ctypes.c_int, [p, i64, i64, p, p, p]),
        "moe_quantize_weights_e16": (ctypes.c_int, [p, i64, i64, p, p, p, p]),
        "moe_quantize_weights_q8": (ctypes.c_int, [p, i64, i64, p, p, p]),
        "moe_shared_workspace_bytes": (sz, [p, i32]),
        "moe_shared_ffn_add": (ctypes.c_int, [p, i32, p, p, p, p, sz, p]),
        "moe_forward_shared": (ctypes.c_int, [p, p, p, i32, p, p, p, sz, p, sz, p]),
        "moe_quant_act_q8": (ctypes.c_int, [p, i32, i32, p, p, p]),
        "moe_route_topk": (ctypes.c_int, [p, p, i32, i32, i32, i32, p, p, p, sz, p]),
        "moe_route_workspace_bytes": (sz, [i32, i32]),
        "moe_expert_ffn_decode": (ctypes.c_int, [p, i32, p, p, p, p, p, p, sz, p]),
        "moe_expert_ffn_prefill": (ctypes.c_int, [p, i32, p, p, p, p, p, p, sz, p]),
        "moe_forward": (ctypes.c_int, [p, p, i32, p, p, p, sz, p]),
        "moe_forward_host": (ctypes.c_int, [p, p, i32, p, p, p, sz, p]),
        "moe_check_status": (ctypes.c_int, [p, p]),
        "moe_last_error": (ctypes.c_char_p, []),
        "moe_debug_matvec": (ctypes.c_int, [p, i32, p, p, p, p, p]),
        "moe_launch_count": (i64, []),
        "moe_trace_begin": (ctypes.c_int, [p, i32]),
        "moe_trace_end": (ctypes.c_int, [p, i32]),
        "moe_kernel_name": (ctypes.c_char_p, [i32]),
        "moe_expert_ffn_decode_static": (ctypes.c_int, [p, i32, p, p, p, p, p, p]),
        "moe_debug_ffn_blocksums": (ctypes.c_int, [p, i32, p, p, p, p, p, p, sz, i32, p, p, p, p]),
        "moe_debug_wait_knob": (ctypes.c_int, [p, sz, i32, i32, p]),
        "moe_workspace_act": (ctypes.c_int, [p, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    return L


def _check(rc):
    if rc != 0:
        raise MoEError(rc, lib().moe_last_error().decode())
    return rc


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return ctypes.c_void_p(t.data_ptr())


# ---------------------------------------------------------------- sizes
def trit_words(rows, k):
    return int(lib().moe_trit_words(rows, k))


def sign_words(rows, k):
    return int(lib().moe_sign_words(rows, k))


def e16_code_words(rows, k):
    return int(lib().moe_e16_code_words(rows, k))


def packed_words(rows, k, fmt="ternary"):
    return sign_words(rows, k) if fmt == "sign" else trit_words(rows, k)


def scale_words(rows, k, fmt="ternary"):
    """fp16 values in a matrix's `scales`: one per block, or one anchor per row (e16)."""
    return rows if fmt == "e16" else scale_count(rows, k)


def scale_count(rows, k):
    return int(lib().moe_scale_count(rows, k))


# ---------------------------------------------------------------- weights
class TernaryMatrix:
    """Packed matrix: trits (int32 view of the uint32 words: base-3 digits,
    or 1-bit sign codes when fmt is "sign"), scales (int16 view of the fp16
    bits: block scales, or per-row anchors when fmt is "e16") and, for "e16",
    codes (int32 view of the 4-bit sub-scale words), in the storage formats of
    bitmoe.h."""

    def __init__(self, rows, k, trits, scales, fmt="ternary", codes=None):
        self.rows, self.k, self.trits, self.scales, self.fmt = rows, k, trits, scales, fmt
        self.codes = codes

    @classmethod
    def empty(cls, rows, k, device="cuda", fmt="ternary"):
        codes = (torch.empty(e16_code_words(rows, k), dtype=torch.int32, device=device)
                 if fmt == "e16" else None)
        return cls(rows, k, torch.empty(packed_words(rows, k, fmt), dtype=torch.int32, device=device),
                   torch.empty(scale_words(rows, k, fmt), dtype=torch.int16, device=device), fmt, codes)

    def c_struct(self):
        return moe_tmat(self.rows, self.k, self.trits.data_ptr(), self.scales.data_ptr(), FORMATS[self.fmt],
                        self.codes.data_ptr() if self.codes is not None else None)

    @property
    def nbytes(self):
        n = self.trits.numel() * 4 + self.scales.numel() * 2
        return n + (self.codes.numel() * 4 if self.codes is not None else 0)


def moe_quantize_weights(w, out=None, stream=None):
    """w [rows][k] fp32 CUDA -> TernaryMatrix (or into `out`)."""
    rows, k = w.shape
    m = TernaryMatrix.empty(rows, k, w.device) if out is None else out
    _check(lib().moe_quantize_weights(_dev(w, torch.float32, "w"), rows, k,
                                      ctypes.c_void_p(m.trits.data_ptr()),
                                      ctypes.c_void_p(m.scales.data_ptr()), _stream(stream)))
    return m


def moe_quantize_weights_sign(w, out=None, stream=None):
    """w [rows][k] fp32 CUDA -> 1-bit sign-code TernaryMatrix (fmt "sign")."""
    rows, k = w.shape
    m = TernaryMatrix.empty(rows, k, w.device, fmt="sign") if out is None else out
    _check(lib().moe_quantize_weights_sign(_dev(w, torch.float32, "w"), rows, k,
                                           ctypes.c_void_p(m.trits.data_ptr()),
                                           ctypes.c_void_p(m.scales.data_ptr()), _stream(stream)))
    return m


def moe_quantize_weights_e16(w, out=None, stream=None):
    """w [rows][k] fp32 CUDA -> ternary digits with two-level scales
    (TernaryMatrix, fmt "e16": per-row anchors in `scales`, sub-scale codes)."""
    rows, k = w.shape
    m = TernaryMatrix.empty(rows, k, w.device, fmt="e16") if out is None else out
    _check(lib().moe_quantize_weights_e16(_dev(w, torch.float32, "w"), rows, k,
                                          ctypes.c_void_p(m.trits.data_ptr()),
                                          ctypes.c_void_p(m.codes.data_ptr()),
                                          ctypes.c_void_p(m.scales.data_ptr()), _stream(stream)))
    return m


def moe_quantize_weights_q8(w, stream=None):
    """w [rows][k] fp32 CUDA -> (q int8 [rows][k], d int16 view of fp16 [rows][k/32])."""
    rows, k = w.shape
    q = torch.empty((rows, k), dtype=torch.int8, device=w.device)
    d = torch.empty((rows, k // QBLOCK), dtype=torch.int16, device=w.device)
    _check(lib().moe_quantize_weights_q8(_dev(w, torch.float32, "w"), rows, k, ctypes.c_void_p(q.data_ptr()),
                                         ctypes.c_void_p(d.data_ptr()), _stream(stream)))
    return q, d


class SharedExpert:
    """The shared expert in 8-bit blocks (gate/up [ffn][hidden], down
    [hidden][ffn]), quantized from fp32 CUDA tensors."""

    def __init__(self, wg, wu, wd, stream=None):
        self.ffn, self.hidden = wg.shape
        self.gate = moe_quantize_weights_q8(wg.contiguous(), stream)
        self.up = moe_quantize_weights_q8(wu.contiguous(), stream)
        self.down = moe_quantize_weights_q8(wd.contiguous(), stream)
        self._c = moe_shared(self.hidden, self.ffn, *[t.data_ptr() for m in (self.gate, self.up, self.down) for t in m])

    def c_ref(self):
        return ctypes.byref(self._c)

    def workspace(self, ntok, device="cuda"):
        n = lib().moe_shared_workspace_bytes(self.c_ref(), ntok)
        if n == 0:
            _check(-1)
        return torch.empty(int(n), dtype=torch.uint8, device=device)

    def add(self, xq, xd, y, ws=None, stream=None):
        """y [ntok][hidden] += the shared expert's FFN of (xq, xd); returns y."""
        ntok = xq.shape[0]
        if ws is None:
            ws = self.workspace(ntok, y.device)
        _check(lib().moe_shared_ffn_add(self.c_ref(), ntok, _dev(xq, torch.int8, "xq"), _dev(xd, torch.float32, "xd"),
                                        _dev(y, torch.float32, "y"), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                        _stream(stream)))
        return y


class MoELayer:
    """Gate, up and down of E experts (expert e owns rows [e*ffn, (e+1)*ffn)
    of gate/up and [e*hidden, (e+1)*hidden) of down)."""

    def __init__(self, hidden, ffn, n_experts, top_k, gate, up, down):
        self.hidden, self.ffn, self.n_experts, self.top_k = hidden, ffn, n_experts, top_k
        self.gate, self.up, self.down = gate, up, down
        self._c = moe_layer(hidden, ffn, n_experts, top_k, gate.c_struct(), up.c_struct(),
                            down.c_struct())

    def c_ref(self):
        return ctypes.byref(self._c)

    @property
    def nbytes(self):
        return self.gate.nbytes + self.up.nbytes + self.down.nbytes

    def workspace_bytes(self, ntok, prefill=False):
        n = lib().moe_workspace_bytes(self.c_ref(), ntok, int(prefill))
        if n == 0:
            _check(-1)
        return int(n)


class Workspace:
    """Device workspace for calls of up to `ntok` tokens (zeroed once)."""

    def __init__(self, nbytes, device="cuda", stream=None):
        self.nbytes = int(nbytes)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        _check(lib().moe_workspace_init(ctypes.c_void_p(self.buf.data_ptr()), self.nbytes,
                                        _stream(stream)))

    @classmethod
    def for_layer(cls, layer, ntok, prefill=None, device="cuda"):
        if prefill is None:
            prefill = ntok > MAX_DECODE_TOKENS
        return cls(layer.workspace_bytes(ntok, prefill), device)

    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())

    def act(self, layer, ntok, prefill=None):
        """Views of x's int8 codes [ntok][hidden] and fp32 scales
        [ntok][hidden/32] that moe_forward left in this workspace."""
        if prefill is None:
            prefill = ntok > MAX_DECODE_TOKENS
        oq, od = ctypes.c_size_t(0), ctypes.c_size_t(0)
        _check(lib().moe_workspace_act(layer.c_ref(), ntok, int(bool(prefill)), ctypes.byref(oq), ctypes.byref(od)))
        H = layer.hidden
        xq = self.buf[oq.value:oq.value + ntok * H].view(torch.int8).view(ntok, H)
        xd = self.buf[od.value:od.value + ntok * (H // QBLOCK) * 4].view(torch.float32).view(ntok, H // QBLOCK)
        return xq, xd


# ---------------------------------------------------------------- the path
def moe_quant_act_q8(x, stream=None):
    ntok, k = x.shape
    xq = torch.empty((ntok, k), dtype=torch.int8, device=x.device)
    xd = torch.empty((ntok, k // QBLOCK), dtype=torch.float32, device=x.device)
    _check(lib().moe_quant_act_q8(_dev(x, torch.float32, "x"), ntok, k, ctypes.c_void_p(xq.data_ptr()),
                                  ctypes.c_void_p(xd.data_ptr()), _stream(stream)))
    return xq, xd


def moe_route_topk(x, w_router, top_k, ws=None, stream=None):
    ntok, hidden = x.shape
    E = w_router.shape[0]
    if ws is None:
        ws = Workspace(lib().moe_route_workspace_bytes(ntok, E), x.device)
    idx = torch.empty((ntok, top_k), dtype=torch.int32, device=x.device)
    wts = torch.empty((ntok, top_k), dtype=torch.float32, device=x.device)
    _check(lib().moe_route_topk(_dev(x, torch.float32, "x"), _dev(w_router, torch.float32, "w_router"),
                                ntok, hidden, E, top_k, ctypes.c_void_p(idx.data_ptr()),
                                ctypes.c_void_p(wts.data_ptr()), ws.ptr(), ws.nbytes, _stream(stream)))
    return idx, wts


def _ffn(fn, layer, xq, xd, idx, wts, ws, y, stream):
    ntok = xq.shape[0]
    if y is None:
        y = torch.empty((ntok, layer.hidden), dtype=torch.float32, device=xq.device)
    _check(fn(layer.c_ref(), ntok, _dev(xq, torch.int8, "xq"), _dev(xd, torch.float32, "xd"),
              _dev(idx, torch.int32, "idx"), _dev(wts, torch.float32, "wts"),
              _dev(y, torch.float32, "y"), ws.ptr(), ws.nbytes, _stream(stream)))
    return y


def moe_expert_ffn_decode(layer, xq, xd, idx, wts, ws, y=None, stream=None):
    return _ffn(lib().moe_expert_ffn_decode, layer, xq, xd, idx, wts, ws, y, stream)


def moe_expert_ffn_decode_static(layer, xq, xd, idx, wts, y=None, stream=None):
    """Decode FFN for callers that cannot allocate device memory: no workspace
    argument; the library's own fixed 4 MiB device scratch is used instead
    (see include/bitmoe.h for its limits)."""
    ntok = xq.shape[0]
    if y is None:
        y = torch.empty((ntok, layer.hidden), dtype=torch.float32, device=xq.device)
    _check(lib().moe_expert_ffn_decode_static(
        layer.c_ref(), ntok, _dev(xq, torch.int8, "xq"), _dev(xd, torch.float32, "xd"),
        _dev(idx, torch.int32, "idx"), _dev(wts, torch.float32, "wts"),
        _dev(y, torch.float32, "y"), _stream(stream)))
    return y


def moe_expert_ffn_prefill(layer, xq, xd, idx, wts, ws, y=None, stream=None):
    return _ffn(lib().moe_expert_ffn_prefill, layer, xq, xd, idx, wts, ws, y, stream)


def moe_forward(layer, w_router, x, ws, y=None, stream=None):
    ntok = x.shape[0]
    if y is None:
        y = torch.empty((ntok, layer.hidden), dtype=torch.float32, device=x.device)
    _check(lib().moe_forward(layer.c_ref(), _dev(w_router, torch.float32, "w_router"), ntok,
                             _dev(x, torch.float32, "x"), _dev(y, torch.float32, "y"), ws.ptr(),
                             ws.nbytes, _stream(stream)))
    return y


def moe_forward_shared(layer, shared, w_router, x, ws, shared_ws=None, y=None, stream=None):
    """y = the routed experts' sum plus the shared expert's FFN of x (one
    launch for one token where the one-token step applies)."""
    ntok = x.shape[0]
    if y is None:
        y = torch.empty((ntok, layer.hidden), dtype=torch.float32, device=x.device)
    if shared_ws is None:
        shared_ws = shared.workspace(ntok, x.device)
    _check(lib().moe_forward_shared(layer.c_ref(), shared.c_ref(), _dev(w_router, torch.float32, "w_router"), ntok,
                                    _dev(x, torch.float32, "x"), _dev(y, torch.float32, "y"), ws.ptr(), ws.nbytes,
                                    ctypes.c_void_p(shared_ws.data_ptr()), shared_ws.numel(), _stream(stream)))
    return y


def moe_forward_host(layer, w_router, x_host, y_host, ws, stream=None):
    """x_host, y_host: CPU fp32 tensors (pinned for asynchronous copies)."""
    for t, n in ((x_host, "x_host"), (y_host, "y_host")):
        if t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError("%s must be a contiguous CPU fp32 tensor" % n)
    _check(lib().moe_forward_host(layer.c_ref(), _dev(w_router, torch.float32, "w_router"),
                                  x_host.shape[0], ctypes.c_void_p(x_host.data_ptr()),
                                  ctypes.c_void_p(y_host.data_ptr()), ws.ptr(), ws.nbytes,
                                  _stream(stream)))
    return y_host


def moe_check_status(ws, stream=None):
    """Synchronize and return (and clear) the device status code."""
    return int(lib().moe_check_status(ws.ptr(), _stream(stream)))


def moe_debug_matvec(mat, xq, xd, want_isum=True, stream=None):
    ntok = xq.shape[0]
    out = torch.empty((ntok, mat.rows), dtype=torch.float32, device=xq.device)
    isum = None
    if want_isum:
        isum = torch.empty((ntok, mat.rows, mat.k // QBLOCK), dtype=torch.int32, device=xq.device)
    m = mat.c_struct()
    _check(lib().moe_debug_matvec(ctypes.byref(m), ntok, _dev(xq, torch.int8, "xq"),
                                  _dev(xd, torch.float32, "xd"), ctypes.c_void_p(out.data_ptr()),
                                  ctypes.c_void_p(isum.data_ptr()) if isum is not None else None,
                                  _stream(stream)))
    return out, isum


def moe_debug_ffn_blocksums(layer, xq, xd, idx, wts, ws, prefill=False, stream=None):
    """The expert FFN through the tensor-core path (decode mat-vecs, or the
    prefill GEMM with prefill=True) with its exact int32 block sums:
    returns (y, isum_gu [pairs][2][ffn][hidden/32], isum_dn
    [pairs][hidden][ffn/32], aq [pairs][ffn])."""
    ntok = xq.shape[0]
    K, H, F = idx.shape[1], layer.hidden, layer.ffn
    dev = xq.device
    y = torch.empty((ntok, H), dtype=torch.float32, device=dev)
    gu = torch.zeros((ntok * K, 2, F, H // QBLOCK), dtype=torch.int32, device=dev)
    dn = torch.zeros((ntok * K, H, F // QBLOCK), dtype=torch.int32, device=dev)
    aq = torch.zeros((ntok * K, F), dtype=torch.int8, device=dev)
    _check(lib().moe_debug_ffn_blocksums(
        layer.c_ref(), ntok, _dev(xq, torch.int8, "xq"), _dev(xd, torch.float32, "xd"),
        _dev(idx, torch.int32, "idx"), _dev(wts, torch.float32, "wts"), _dev(y, torch.float32, "y"),
        ws.ptr(), ws.nbytes, int(bool(prefill)), ctypes.c_void_p(gu.data_ptr()),
        ctypes.c_void_p(dn.data_ptr()), ctypes.c_void_p(aq.data_ptr()), _stream(stream)))
    return y, gu, dn, aq


def moe_debug_wait_knob(ws, mode, polls=0, stream=None):
    """Test knob of the bounded device waits (see include/bitmoe.h): mode 1
    makes the one-token step's logit poll run out, mode 2 the tensor-core
    mat-vecs' mbarrier waits; 0 restores normal operation."""
    _check(lib().moe_debug_wait_knob(ws.ptr(), ws.nbytes, int(mode), int(polls), _stream(stream)))


# ---------------------------------------------------------------- tracing
def moe_launch_count():
    """Kernels this thread has launched through the library so far."""
    return int(lib().moe_launch_count())


class KernelTrace:
    """Per-kernel CUDA-event timing of library launches.

    While the context is active, the library records one of `capacity`
    events on the launching stream after every kernel; `durations()` then
    gives, per kernel name, the elapsed time since the previous event (or
    since `start`, recorded on entry) -- i.e. each kernel's time on its
    stream when the stream runs the library's kernels back to back."""

    def __init__(self, capacity=4096):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(capacity)]
        for e in self.events:  # torch creates the CUDA event on first record
            e.record()
        torch.cuda.current_stream().synchronize()
        self.handles = (ctypes.c_void_p * capacity)(*[e.cuda_event for e in self.events])
        self.start = torch.cuda.Event(enable_timing=True)
        self.n = 0
        self.ids = []

    def __enter__(self):
        self.start.record()
        _check(lib().moe_trace_begin(self.handles, len(self.events)))
        return self

    def __exit__(self, *exc):
        ids = (ctypes.c_int32 * len(self.events))()
        self.n = int(lib().moe_trace_end(ids, len(self.events)))
        self.ids = list(ids[:self.n])
        return False

    def durations(self):
        """{kernel name: [ms per launch, ...]} (call after synchronizing)."""
        out = {}
        prev = self.start
        for i in range(self.n):
            ev = self.events[i]
            name = lib().moe_kernel_name(self.ids[i]).decode()
            out.setdefault(name, []).append(prev.elapsed_time(ev))
            prev = ev
        return out
