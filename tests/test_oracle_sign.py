"""Pins for the oracle's 1-bit sign-code format (CPU only).

The 1-bit tier of the pxq_llama README ("What's PXQ?", the PXQ1 row) stores
one sign per weight times a scale; this build reads it with the ternary
format's 256-weight block and fp16 absmean scale.  Each test checks the oracle
against something other than itself: a hand-placed bit, the least-squares
optimum of a sign code's scale, an fp64 dense evaluation from the unpacked
values, closed forms of all-positive and all-zero blocks.
"""
import numpy as np
import pytest

from test_oracle_router_ffn import _dense_mixture, _tiny


def test_sign_bit_position_hand_case(orc):
    """One negative weight at k = 32*1 + 4*i + l with i = 3, l = 2 of row 5:
    in word 1 of that row's block only bit 8*2 + 3 is clear."""
    rows, k = 32, 256
    w = np.full((rows, k), 0.5, np.float32)
    w[5, 32 + 4 * 3 + 2] = -0.25
    codes, scales = orc.quantize_weights_sign(w)
    for r in range(rows):
        for j in range(8):
            word = int(codes[orc.sign_word_index(k, r, 0, j)])
            want = 0xFFFFFFFF & ~(1 << (8 * 2 + 3)) if (r, j) == (5, 1) else 0xFFFFFFFF
            assert word == want, (r, j, hex(word))
    # the words of a block sit 32 apart (one per row of the panel), the rows
    # of a panel are consecutive
    assert orc.sign_word_index(k, 5, 0, 1) == 1 * 32 + 5
    assert orc.sign_word_index(512, 33, 1, 7) == ((1 * 2 + 1) * 8 + 7) * 32 + 1
    # scale of row 5: (255 * 0.5 + 0.25) / 256, rounded to fp16
    assert scales[orc.scale_index(k, 5, 0)] == np.float16((255 * 0.5 + 0.25) / 256).view(np.uint16)


def test_sign_roundtrip_and_signs(orc):
    rng = np.random.default_rng(11)
    rows, k = 64, 768
    w = rng.standard_normal((rows, k)).astype(np.float32)
    w[3, :10] = 0.0
    w[4, 7] = -0.0
    codes, scales = orc.quantize_weights_sign(w)
    assert codes.size == rows * (k // 256) * 8
    q, s = orc.unpack_weights_sign(codes, scales, rows, k)
    assert np.array_equal(q, np.where(w < 0, -1, 1).astype(np.int8))   # zeros (and -0) code +1
    mean_abs = np.abs(w.astype(np.float64)).reshape(rows, k // 256, 256).mean(axis=2)
    assert np.array_equal(s, mean_abs.astype(np.float16).astype(np.float32))
    # unpacking a row range gives the same rows
    q2, s2 = orc.unpack_weights_sign(codes, scales, rows, k, row0=33, nrows=7)
    assert np.array_equal(q2, q[33:40]) and np.array_equal(s2, s[33:40])


def test_sign_scale_is_least_squares_optimum(orc):
    """For codes of +-1 the squared error sum (w - s*sign w)^2 is a parabola
    in s with its minimum at mean|w|: the stored fp16 scale beats both fp16
    neighbours."""
    rng = np.random.default_rng(12)
    w = (rng.standard_normal((32, 256)) * 0.03).astype(np.float32)
    codes, scales = orc.quantize_weights_sign(w)
    q, s = orc.unpack_weights_sign(codes, scales, 32, 256)
    for r in range(32):
        h = scales[orc.scale_index(256, r, 0)]
        err = lambda hh: np.sum((w[r].astype(np.float64)
                                 - float(np.uint16(hh).view(np.float16)) * q[r]) ** 2)
        assert err(h) <= err(h + 1) and err(h) <= err(h - 1)


def test_sign_matvec_all_positive_closed_form(orc):
    """All-positive weights: every code is +1, so row r gives
    s_r * sum_j xd_j * sum(xq in block j)."""
    rng = np.random.default_rng(13)
    rows, k = 32, 512
    w = np.abs(rng.standard_normal((rows, k))).astype(np.float32) + np.float32(0.01)
    codes, scales = orc.quantize_weights_sign(w)
    q, s = orc.unpack_weights_sign(codes, scales, rows, k)
    assert np.all(q == 1)
    xq, xd = orc.quant_act_q8(rng.standard_normal((1, k)).astype(np.float32))
    out = orc.matvec(q, s, xq[0], xd[0])
    bsum = xd[0].astype(np.float64) * xq[0].reshape(-1, 32).astype(np.int64).sum(axis=1)
    ref = (s.astype(np.float64) * bsum.reshape(-1, 8).sum(axis=1)[None, :]).sum(axis=1)
    assert np.allclose(out, ref, rtol=1e-14, atol=0)


def test_sign_ffn_route_all_equals_dense_mixture(orc):
    H, F, E = 256, 512, 4
    wg, wu, wd, wr, x = _tiny(orc, H, F, E, seed=21)
    layer = orc.Layer.from_float(H, F, E, E, wg, wu, wd, fmt="sign")
    y, idx, wts = orc.moe_forward(layer, wr, x)
    ref = _dense_mixture(orc, layer, wr, x, unpack=orc.unpack_weights_sign)
    scale = np.abs(ref).max()
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * scale)
    assert scale > 1e-3


def test_sign_ffn_zero_weights_give_zero(orc):
    """All-zero weights code +1 everywhere but get scale 0: y = 0."""
    H, F, E, K = 256, 256, 4, 2
    z = np.zeros
    layer = orc.Layer.from_float(H, F, E, K, z((E * F, H), np.float32), z((E * F, H), np.float32),
                                 z((E * H, F), np.float32), fmt="sign")
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, H)).astype(np.float32)
    wr = rng.standard_normal((E, H)).astype(np.float32)
    y, _, _ = orc.moe_forward(layer, wr, x)
    assert not y.any()


def test_sign_and_ternary_agree_on_sign_valued_weights(orc):
    """Weights of equal magnitude m in every block: the ternary code is
    sign(w) with scale m, the sign code the same, so both formats give the
    same layer output."""
    H, F, E, K = 256, 512, 4, 2
    rng = np.random.default_rng(23)
    m = np.float32(0.03125)

    def pm(shape):
        return np.where(rng.random(shape) < 0.5, -m, m).astype(np.float32)

    wg, wu, wd = pm((E * F, H)), pm((E * F, H)), pm((E * H, F))
    wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    x = rng.standard_normal((3, H)).astype(np.float32)
    yt, it, _ = orc.moe_forward(orc.Layer.from_float(H, F, E, K, wg, wu, wd), wr, x)
    ys, is_, _ = orc.moe_forward(orc.Layer.from_float(H, F, E, K, wg, wu, wd, fmt="sign"), wr, x)
    assert np.array_equal(it, is_)
    assert np.array_equal(yt, ys)


def test_sign_bad_shapes(orc):
    with pytest.raises(ValueError):
        orc.quantize_weights_sign(np.zeros((31, 256), np.float32))
    with pytest.raises(ValueError):
        orc.quantize_weights_sign(np.zeros((32, 255), np.float32))
