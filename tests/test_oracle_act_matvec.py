"""Pins for the oracle's int8 activation blocks and its block-sum mat-vec (CPU)."""
import numpy as np
import pytest


# ------------------------------------------------------------------ q8 activations
def test_q8_integer_grid_roundtrip(orc):
    """x = c * m with integers |m| <= 127, max |m| = 127 and c a power of two:
    d = 127c/127 = c exactly and every code is m."""
    rng = np.random.default_rng(11)
    m = rng.integers(-127, 128, size=(4, 256)).astype(np.int64)
    m[:, ::32] = 127 * np.where(np.arange(8) % 2, 1, -1)
    for c in (1.0, 2.0 ** -7, 2.0 ** 5):
        x = (m * c).astype(np.float32)
        xq, xd = orc.quant_act_q8(x)
        assert np.array_equal(xq.astype(np.int64), m)
        assert np.all(xd == np.float32(c))


def test_q8_amax_and_bounds(orc):
    rng = np.random.default_rng(12)
    x = rng.standard_normal((8, 512)).astype(np.float32) * 3
    xq, xd = orc.quant_act_q8(x)
    xb = x.reshape(8, 16, 32)
    qb = xq.reshape(8, 16, 32).astype(np.int32)
    amax_pos = np.abs(xb).argmax(-1)
    for t in range(8):
        for j in range(16):
            i = amax_pos[t, j]
            assert qb[t, j, i] == (127 if xb[t, j, i] > 0 else -127)
    assert np.abs(qb).max() <= 127
    # the scale is amax/127 as an fp32 quotient
    assert np.array_equal(xd, (np.abs(xb).max(-1) / np.float32(127)).astype(np.float32))
    # round to nearest: every reconstruction error is at most half a step
    err = np.abs(xb.astype(np.float64) - qb * xd[..., None].astype(np.float64))
    assert np.all(err <= xd[..., None].astype(np.float64) * (0.5 + 1e-6))


def test_q8_ties_to_even_and_zero_block(orc):
    x = np.zeros((1, 64), np.float32)
    x[0, 0] = 127.0                      # d = 1 exactly
    x[0, 1:7] = [2.5, 3.5, -2.5, -3.5, 0.5, 126.5]
    xq, xd = orc.quant_act_q8(x)
    assert xd[0, 0] == 1.0 and xd[0, 1] == 0.0
    assert list(xq[0, 1:7]) == [2, 4, -2, -4, 0, 126]
    assert not xq[0, 32:].any()
    # amax/127 underflows to 0: the block is treated as the zero block
    x2 = np.zeros((1, 32), np.float32)
    x2[0, 3] = np.float32(1e-44)
    xq2, xd2 = orc.quant_act_q8(x2)
    assert xd2[0, 0] == 0.0 and not xq2.any()


def test_q8_scale_invariance(orc):
    rng = np.random.default_rng(13)
    x = rng.standard_normal((3, 256)).astype(np.float32)
    q1, d1 = orc.quant_act_q8(x)
    q2, d2 = orc.quant_act_q8(x * np.float32(8))
    assert np.array_equal(q1, q2)
    assert np.array_equal(d2, d1 * 8)


def test_q8_rejects_bad_k(orc):
    with pytest.raises(ValueError):
        orc.quant_act_q8(np.zeros((1, 40), np.float32))


# ------------------------------------------------------------------ block sums / mat-vec
def _rand_layer(rng, rows, k, std=0.02):
    w = (rng.standard_normal((rows, k)) * std).astype(np.float32)
    return w


def test_blocksums_brute_force(orc):
    rng = np.random.default_rng(21)
    rows, k = 64, 768
    q = rng.integers(-1, 2, size=(rows, k)).astype(np.int8)
    xq = rng.integers(-127, 128, size=k).astype(np.int8)
    isum = orc.blocksums(q, xq)
    ref = np.zeros((rows, k // 32), np.int64)
    for r in range(rows):
        for kk in range(k):
            ref[r, kk // 32] += int(q[r, kk]) * int(xq[kk])
    assert np.array_equal(isum.astype(np.int64), ref)


def test_matvec_equals_dense_dequantized_product(orc):
    """Block-wise fixups equal the dense product of dequantized vectors (exact
    arithmetic), so the two fp64 results agree to rounding."""
    rng = np.random.default_rng(22)
    rows, k = 96, 1024
    w = _rand_layer(rng, rows, k)
    trits, scales = orc.quantize_weights(w)
    q, s = orc.unpack_weights(trits, scales, rows, k)
    x = rng.standard_normal(k).astype(np.float32)
    xq, xd = orc.quant_act_q8(x)
    out = orc.matvec(q, s, xq[0], xd[0])
    wdeq = q.astype(np.float64) * np.repeat(s.astype(np.float64), 256, axis=1)
    xdeq = xq[0].astype(np.float64) * np.repeat(xd[0].astype(np.float64), 32)
    ref = wdeq @ xdeq
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # against the unquantized product: for Gaussian w the absmean ternary
    # reconstruction w^ = s*q has E[w w^]/E[w^2] = sqrt(2/pi) * 2*phi(t) with
    # t = sqrt(2/pi)/2 (phi the normal density), i.e. 0.588, and correlation
    # 0.588 / sqrt(0.439) = 0.887; a missing, doubled or misplaced scale
    # breaks one of the two
    w2 = _rand_layer(rng, 1024, 1024)
    q2, s2 = orc.unpack_weights(*orc.quantize_weights(w2), 1024, 1024)
    xs = rng.standard_normal((8, 1024)).astype(np.float32)
    xq2, xd2 = orc.quant_act_q8(xs)
    out = np.concatenate([orc.matvec(q2, s2, xq2[i], xd2[i]) for i in range(8)])
    exact = (w2.astype(np.float64) @ xs.astype(np.float64).T).T.ravel()
    t = np.sqrt(2 / np.pi) / 2
    beta_th = np.sqrt(2 / np.pi) * 2 * np.exp(-t * t / 2) / np.sqrt(2 * np.pi)
    beta = float(out @ exact / (exact @ exact))
    corr = float(np.corrcoef(out, exact)[0, 1])
    assert abs(beta - beta_th) < 0.02, (beta, beta_th)
    assert corr > 0.85, corr


def test_matvec_linear_in_activation_scale(orc):
    rng = np.random.default_rng(23)
    q = rng.integers(-1, 2, size=(32, 512)).astype(np.int8)
    s = rng.uniform(0.001, 0.01, size=(32, 2)).astype(np.float32)
    xq = rng.integers(-127, 128, size=512).astype(np.int8)
    xd = rng.uniform(0.01, 0.1, size=16).astype(np.float32)
    a = orc.matvec(q, s, xq, xd)
    b = orc.matvec(q, s, xq, xd * np.float32(4))
    assert np.allclose(b, 4 * a, rtol=1e-14, atol=0)
