"""Pins for the oracle's shared expert (CPU only): the higher-precision
expert beside the low-bit routed ones (llama-modchip page, "The interesting
bit"), read as 8-bit blocks of 32 weights with an fp16 scale.  Each test
checks the oracle against something other than itself: numpy's binary16
rounding and the quantization error bound, a dense fp64 product, a dense
evaluation of the FFN, and the additivity of the shared term."""
import numpy as np
import pytest

from test_oracle_router_ffn import _tiny


def test_q8_weights_scale_and_error_bound(orc):
    rng = np.random.default_rng(61)
    rows, k = 16, 256
    w = (rng.standard_normal((rows, k)) * 0.05).astype(np.float32)
    w[3, 32:64] = 0.0                                   # one all-zero block
    q, d = orc.quantize_weights_q8(w)
    amax = np.abs(w.astype(np.float64)).reshape(rows, k // 32, 32).max(axis=2)
    assert np.array_equal(d, (amax / 127.0).astype(np.float16).view(np.uint16))
    df = np.repeat(d.view(np.float16).astype(np.float64), 32, axis=1)
    err = np.abs(w.astype(np.float64) - q.astype(np.float64) * df)
    assert np.all(err <= 0.5 * df + 1e-12)
    # the largest element of every nonzero block codes +-127
    qa = np.abs(q.astype(np.int64)).reshape(rows, k // 32, 32).max(axis=2)
    assert np.all(qa[amax > 0] == 127)
    assert not q[3, 32:64].any() and d[3, 1] == 0
    with pytest.raises(ValueError):
        orc.quantize_weights_q8(np.zeros((4, 48), np.float32))


def test_q8_matvec_dense(orc):
    rng = np.random.default_rng(62)
    rows, k = 48, 512
    w = (rng.standard_normal((rows, k)) * 0.05).astype(np.float32)
    q, d = orc.quantize_weights_q8(w)
    xq, xd = orc.quant_act_q8(rng.standard_normal((1, k)).astype(np.float32))
    out = orc.matvec_q8(q, d, xq[0], xd[0])
    wdeq = q.astype(np.float64) * np.repeat(d.view(np.float16).astype(np.float64), 32, axis=1)
    xdeq = xq[0].astype(np.float64) * np.repeat(xd[0].astype(np.float64), 32)
    ref = wdeq @ xdeq
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_shared_ffn_dense(orc):
    """The shared term equals Wd (q8(silu(Wg x^) * Wu x^))^ evaluated densely
    from the dequantized 8-bit weights."""
    rng = np.random.default_rng(63)
    H, Fs = 256, 384
    wg = (rng.standard_normal((Fs, H)) * 0.05).astype(np.float32)
    wu = (rng.standard_normal((Fs, H)) * 0.05).astype(np.float32)
    wd = (rng.standard_normal((H, Fs)) * 0.05).astype(np.float32)
    x = rng.standard_normal((3, H)).astype(np.float32)
    sh = orc.SharedExpert(H, Fs, wg, wu, wd)
    xq, xd = orc.quant_act_q8(x)
    y = sh.add_to(np.zeros((3, H)), xq, xd)

    def deq(m):
        q, d = m
        return q.astype(np.float64) * np.repeat(d.view(np.float16).astype(np.float64), 32, axis=1)

    xdeq = xq.astype(np.float64) * np.repeat(xd.astype(np.float64), 32, axis=1)
    g = xdeq @ deq(sh.gate).T
    u = xdeq @ deq(sh.up).T
    a = (g / (1.0 + np.exp(-g)) * u).astype(np.float32)
    aq, ad = orc.quant_act_q8(a)
    ref = (aq.astype(np.float64) * np.repeat(ad.astype(np.float64), 32, axis=1)) @ deq(sh.down).T
    scale = np.abs(ref).max()
    assert scale > 1e-3
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * scale)


def test_shared_term_adds_to_the_routed_sum(orc):
    """moe_forward with a shared expert = the routed output + the shared FFN
    (exactly, in fp64); a zero shared expert changes nothing; with all routed
    weights zero the output is the shared FFN alone."""
    H, F, E, K = 256, 512, 4, 2
    wg, wu, wd, wr, x = _tiny(orc, H, F, E, seed=64)
    rng = np.random.default_rng(65)
    Fs = 256
    sg = (rng.standard_normal((Fs, H)) * 0.05).astype(np.float32)
    su = (rng.standard_normal((Fs, H)) * 0.05).astype(np.float32)
    sd = (rng.standard_normal((H, Fs)) * 0.05).astype(np.float32)
    sh = orc.SharedExpert(H, Fs, sg, su, sd)
    layer = orc.Layer.from_float(H, F, E, K, wg, wu, wd)
    y0, i0, _ = orc.moe_forward(layer, wr, x)
    y1, i1, _ = orc.moe_forward(layer, wr, x, shared=sh)
    xq, xd = orc.quant_act_q8(x)
    only = sh.add_to(np.zeros_like(y0), xq, xd)
    assert np.array_equal(i0, i1)
    assert np.array_equal(y1, y0 + only)
    z = np.zeros
    zero_sh = orc.SharedExpert(H, Fs, z((Fs, H), np.float32), z((Fs, H), np.float32), z((H, Fs), np.float32))
    y2, _, _ = orc.moe_forward(layer, wr, x, shared=zero_sh)
    assert np.array_equal(y2, y0)
    zl = orc.Layer.from_float(H, F, E, K, z((E * F, H), np.float32), z((E * F, H), np.float32),
                              z((E * H, F), np.float32))
    y3, _, _ = orc.moe_forward(zl, wr, x, shared=sh)
    assert np.array_equal(y3, only)
