"""Pins for the oracle's two-level (E16) scales (CPU only).

The E16-row scales of the pxq_llama README ("What's PXQ?": a per-row fp16
anchor plus a 4-bit sub-scale per 16-element block), read onto the ternary
digits.  Each test checks the oracle against something other than itself: a
hand-built row whose codes and anchor are known in advance, the definition of
the anchor, a brute-force dense fp64 product, and the ternary format on
weights of one magnitude.
"""
import numpy as np
import pytest
import scipy.special


def test_e16_hand_row(orc):
    """Row 0: 16-block h holds |w| = (h+1)/32 with alternating signs, so the
    block means are (h+1)/32, the anchor is 0.5, code h is h and the
    sub-scale reproduces each block's mean exactly."""
    rows, k = 32, 256
    w = np.full((rows, k), 0.25, np.float32)
    sgn = np.where(np.arange(16) % 2 == 0, 1.0, -1.0)
    for h in range(16):
        w[0, 16 * h:16 * h + 16] = sgn * (h + 1) / 32.0
    trits, codes, anchors = orc.quantize_weights_e16(w)
    assert anchors[0] == np.float16(0.5).view(np.uint16)
    assert codes[orc.e16_code_index(k, 0, 0, 0)] == 0x76543210
    assert codes[orc.e16_code_index(k, 0, 0, 1)] == 0xFEDCBA98
    q, s16 = orc.unpack_weights_e16(trits, codes, anchors, rows, k)
    assert np.array_equal(s16[0], (np.arange(16) + 1) / 32.0)
    assert np.array_equal(q[0], np.sign(w[0]).astype(np.int8))
    # constant rows: anchor 0.25, every code 15, q = +1
    assert anchors[1] == np.float16(0.25).view(np.uint16)
    assert codes[orc.e16_code_index(k, 1, 0, 0)] == 0xFFFFFFFF
    assert np.all(q[1] == 1)


def test_e16_anchor_codes_and_zero_rows(orc):
    rng = np.random.default_rng(41)
    rows, k = 64, 512
    w = (rng.standard_normal((rows, k)) * 0.02).astype(np.float32)
    w[7] = 0.0
    trits, codes, anchors = orc.quantize_weights_e16(w)
    m = np.abs(w.astype(np.float64)).reshape(rows, k // 16, 16).mean(axis=2)
    assert np.array_equal(anchors, m.max(axis=1).astype(np.float16).view(np.uint16))
    q, s16 = orc.unpack_weights_e16(trits, codes, anchors, rows, k)
    a = anchors.view(np.float16).astype(np.float64)
    # codes: c = clamp(rint(16 m / A) - 1, 0, 15); the largest block gets 15
    c = np.rint(16 * s16.astype(np.float64) / np.where(a == 0, 1, a)[:, None]) - 1
    ref_c = np.clip(np.rint(16 * m / np.where(a == 0, 1, a)[:, None]) - 1, 0, 15)
    ref_c[7] = 0
    assert np.array_equal(c[a > 0], ref_c[a > 0])
    assert np.all(ref_c[a > 0].max(axis=1) == 15)
    # the all-zero row: anchor 0, scales 0, digits 0
    assert anchors[7] == 0 and not s16[7].any() and not q[7].any()
    # q = sign(w) where |w| >= s/2 (fp32), else 0
    half = 0.5 * np.repeat(s16, 16, axis=1)
    ref_q = np.where((np.abs(w) >= half) & (w != 0), np.sign(w), 0).astype(np.int8)
    assert np.array_equal(q, ref_q)
    # a row range unpacks the same rows
    q2, s2 = orc.unpack_weights_e16(trits, codes, anchors, rows, k, row0=33, nrows=5)
    assert np.array_equal(q2, q[33:38]) and np.array_equal(s2, s16[33:38])


def test_e16_matvec_brute_force(orc):
    """The E16 mat-vec equals the dense fp64 product of the dequantized
    weights (q * s16 per weight) with the dequantized activations."""
    rng = np.random.default_rng(42)
    rows, k = 64, 768
    w = (rng.standard_normal((rows, k)) * 0.02).astype(np.float32)
    trits, codes, anchors = orc.quantize_weights_e16(w)
    q, s16 = orc.unpack_weights_e16(trits, codes, anchors, rows, k)
    xq, xd = orc.quant_act_q8(rng.standard_normal((1, k)).astype(np.float32))
    out = orc.matvec_e16(q, s16, xq[0], xd[0])
    wdeq = q.astype(np.float64) * np.repeat(s16.astype(np.float64), 16, axis=1)
    xdeq = xq[0].astype(np.float64) * np.repeat(xd[0].astype(np.float64), 32)
    ref = wdeq @ xdeq
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def _layer_inputs(seed, H=256, F=512, E=4):
    rng = np.random.default_rng(seed)
    wg = (rng.standard_normal((E * F, H)) * 0.05).astype(np.float32)
    wu = (rng.standard_normal((E * F, H)) * 0.05).astype(np.float32)
    wd = (rng.standard_normal((E * H, F)) * 0.05).astype(np.float32)
    wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    x = rng.standard_normal((3, H)).astype(np.float32)
    return wg, wu, wd, wr, x


def test_e16_ffn_route_all_equals_dense_mixture(orc):
    """Every expert routed: y = sum_e softmax_e * Wd_e q8(silu(Wg_e x^) * Wu_e x^)^
    evaluated densely from the unpacked E16 weights."""
    H, F, E = 256, 512, 4
    wg, wu, wd, wr, x = _layer_inputs(43, H, F, E)
    layer = orc.Layer.from_float(H, F, E, E, wg, wu, wd, fmt="e16")
    y, _, _ = orc.moe_forward(layer, wr, x)
    xq, xd = orc.quant_act_q8(x)
    p = scipy.special.softmax(orc.router_logits(x, wr).astype(np.float64), axis=1)
    xdeq = xq.astype(np.float64) * np.repeat(xd.astype(np.float64), 32, axis=1)

    def deq(mat, rows, k, e):
        q, s16 = orc.unpack_weights_e16(mat[0], mat[2], mat[1], E * rows, k, e * rows, rows)
        return q.astype(np.float64) * np.repeat(s16.astype(np.float64), 16, axis=1)

    ref = np.zeros((x.shape[0], H))
    for e in range(E):
        g = xdeq @ deq(layer.gate, F, H, e).T
        u = xdeq @ deq(layer.up, F, H, e).T
        a = (g / (1.0 + np.exp(-g)) * u).astype(np.float32)
        aq, ad = orc.quant_act_q8(a)
        adeq = aq.astype(np.float64) * np.repeat(ad.astype(np.float64), 32, axis=1)
        ref += p[:, e:e + 1].astype(np.float32).astype(np.float64) * (adeq @ deq(layer.down, H, F, e).T)
    scale = np.abs(ref).max()
    assert scale > 1e-3
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * scale)


def test_e16_and_ternary_agree_on_one_magnitude(orc):
    """Weights of one magnitude m: every 16-block mean is m, so the anchor is
    fp16(m), every code 15 and every sub-scale m; the ternary block scale is
    also fp16(m): both formats give the same layer output."""
    H, F, E, K = 256, 512, 4, 2
    rng = np.random.default_rng(44)
    m = np.float32(0.03125)

    def pm(shape):
        return np.where(rng.random(shape) < 0.5, -m, m).astype(np.float32)

    wg, wu, wd = pm((E * F, H)), pm((E * F, H)), pm((E * H, F))
    wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    x = rng.standard_normal((3, H)).astype(np.float32)
    yt, it, _ = orc.moe_forward(orc.Layer.from_float(H, F, E, K, wg, wu, wd), wr, x)
    ye, ie, _ = orc.moe_forward(orc.Layer.from_float(H, F, E, K, wg, wu, wd, fmt="e16"), wr, x)
    assert np.array_equal(it, ie)
    assert np.array_equal(yt, ye)


def test_e16_bad_shapes(orc):
    with pytest.raises(ValueError):
        orc.quantize_weights_e16(np.zeros((31, 256), np.float32))
    with pytest.raises(ValueError):
        orc.quantize_weights_e16(np.zeros((32, 200), np.float32))
