"""Pins for the oracle's weight format: binary16 rounding, the base-3 byte, and
the absmean ternary block (CPU only).

Each test checks the oracle against something other than itself: numpy's own
binary16 conversion, exhaustive enumeration, or closed forms of the absmean
rule.
"""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ------------------------------------------------------------------ binary16
def test_f16_to_f32_exhaustive(orc):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.f16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f16_from_f64_roundtrip_and_midpoints(orc):
    # every finite half converts back to itself
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = h.view(np.float16).astype(np.float64)
    fin = np.isfinite(vals)
    back = orc.f16_from_f64(vals[fin])
    assert np.array_equal(back, h[fin])
    # midpoints of consecutive positive finite halves: ties go to even (numpy
    # rounds float64 -> float16 correctly, ties to even)
    pos = np.arange(0, 0x7C00, dtype=np.uint16)
    lo = pos[:-1].view(np.float16).astype(np.float64)
    hi = pos[1:].view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2.0                        # exact in fp64
    ours = orc.f16_from_f64(np.concatenate([mid, -mid]))
    ref = np.concatenate([mid, -mid]).astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    # even mantissa wins at a tie: 1 + 2^-11 is halfway between 1 and 1 + 2^-10
    assert orc.f16_from_f64(np.array([1.0 + 2.0 ** -11]))[0] == 0x3C00
    assert orc.f16_from_f64(np.array([1.0 + 3 * 2.0 ** -11]))[0] == 0x3C02


def test_f16_from_f64_random_and_edges(orc):
    rng = np.random.default_rng(7)
    x = np.exp(rng.uniform(np.log(1e-9), np.log(7e4), 20000)) * rng.choice([-1, 1], 20000)
    ours = orc.f16_from_f64(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    edges = np.array([65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -24, 2.0 ** -25,
                      2.0 ** -25 * 1.0000001, 2.0 ** -14, 0.0, -0.0])
    assert np.array_equal(orc.f16_from_f64(edges), edges.astype(np.float16).view(np.uint16))


# ------------------------------------------------------------------ base-3 byte
def _all_digit_tuples():
    for v in range(243):
        t = [(v // 3 ** (4 - i)) % 3 for i in range(5)]
        yield v, t


def test_trit_byte_roundtrip_exhaustive(orc):
    seen = set()
    prev = -1
    for v, t in _all_digit_tuples():
        u = orc.trit_byte_encode(np.array(t))
        assert 0 <= u <= 255
        assert u > prev, "codes must increase with the base-3 value"
        prev = u
        seen.add(u)
        back = orc.trit_byte_decode(u)
        assert back is not None and list(back) == t
    # exactly 243 of the 256 byte values are codes; the rest are rejected
    assert len(seen) == 243
    for u in range(256):
        assert (orc.trit_byte_decode(u) is not None) == (u in seen)


def test_fixed_point_peel_off_property(orc):
    """The byte is ceil(v*256/243): multiplying by 3^i and keeping the high
    byte gives H_i = floor(v / 3^(5-i)), so digit i = H_(i+1) - 3*H_i.  A
    16-bit lane holds u*3^5 and 3*H_i fits a byte (no borrow between lanes)."""
    for v, t in _all_digit_tuples():
        u = orc.trit_byte_encode(np.array(t))
        H = [(u * 3 ** i) >> 8 for i in range(6)]
        assert H[0] == 0
        for i in range(6):
            assert H[i] == v // 3 ** (5 - i)
        assert [H[i + 1] - 3 * H[i] for i in range(5)] == t
        assert u * 3 ** 5 <= 0xFFFF
        assert all(3 * H[i] <= 0xFF for i in range(5))


# ------------------------------------------------------------------ absmean blocks
def _quant(orc, w):
    trits, scales = orc.quantize_weights(w)
    q, s = orc.unpack_weights(trits, scales, *w.shape)
    return q, s, trits, scales


def test_roundtrip_ternary_patterns(orc):
    """w = c * q with q ternary and c a power of two: the absmean rule gives
    back q exactly, with s = c * nnz / 256 (every nonzero has |w| = c >= s/2)."""
    rng = np.random.default_rng(1)
    rows, k = 64, 1024
    q0 = rng.integers(-1, 2, size=(rows, k)).astype(np.int8)
    q0[:, ::256] = 1                                  # every block has a nonzero
    c = 0.25
    q, s, _, _ = _quant(orc, q0.astype(np.float32) * np.float32(c))
    assert np.array_equal(q, q0)
    nnz = np.abs(q0.reshape(rows, k // 256, 256)).sum(-1)
    exp_s = (c * nnz / 256.0).astype(np.float16).astype(np.float32)
    assert np.array_equal(s, exp_s)


def test_closed_forms(orc):
    rows, k = 32, 256
    w = np.zeros((rows, k), np.float32)
    # row 0: constant magnitude c, random signs -> s = c, q = sign
    signs = np.where(np.arange(k) % 3 == 0, -1.0, 1.0).astype(np.float32)
    w[0] = 0.375 * signs
    # row 1: a single nonzero v -> s = |v|/256, q = sign(v) there, 0 elsewhere
    w[1, 77] = -3.0
    # row 2: all zero -> s = 0, q = 0
    q, s, _, _ = _quant(orc, w)
    assert s[0, 0] == np.float32(0.375)
    assert np.array_equal(q[0], signs.astype(np.int8))
    assert s[1, 0] == np.float16(3.0 / 256).astype(np.float32)
    assert q[1, 77] == -1 and np.count_nonzero(q[1]) == 1
    assert s[2, 0] == 0 and not q[2].any()


def test_threshold_tie_exact(orc):
    """A weight exactly at half the block scale rounds away from zero."""
    w = np.zeros((32, 256), np.float32)
    # sum of |w| = 256 exactly with entries at exactly 0.5
    w[0, :63] = 2.0        # 126
    w[0, 63:192] = 1.0     # 129 -> 255
    w[0, 192] = 0.5        # 255.5
    w[0, 193] = -0.5       # 256.0 -> s = 1.0, threshold 0.5 exactly
    q, s, _, _ = _quant(orc, w)
    assert s[0, 0] == 1.0
    assert q[0, 192] == 1 and q[0, 193] == -1
    w[0, 192] = np.nextafter(np.float32(0.5), np.float32(0))
    w[0, 194] = 0.5 - w[0, 192]  # keep the sum 256 exactly in fp64
    q, s, _, _ = _quant(orc, w)
    assert s[0, 0] == 1.0
    assert q[0, 192] == 0 and q[0, 194] == 0


def test_gaussian_zero_fraction(orc):
    """For w ~ N(0, s^2) the absmean is s*sqrt(2/pi), so the zero fraction is
    P(|z| < sqrt(2/pi)/2) = erf(sqrt(2/pi)/2/sqrt(2)) = 0.3101."""
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((256, 4096)) * 0.02).astype(np.float32)
    q, s, _, _ = _quant(orc, w)
    frac = np.mean(q == 0)
    expected = math.erf(math.sqrt(2 / math.pi) / 2 / math.sqrt(2))
    assert abs(frac - expected) < 0.003, (frac, expected)
    # the scale is the block absmean rounded to fp16
    absmean = np.abs(w.astype(np.float64)).reshape(256, 16, 256).mean(-1)
    assert np.array_equal(s, absmean.astype(np.float16).astype(np.float32))


def test_scale_invariance(orc):
    """Scaling w by 2 doubles every scale exactly and keeps every q."""
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    q1, s1, _, _ = _quant(orc, w)
    q2, s2, _, _ = _quant(orc, w * np.float32(2))
    assert np.array_equal(q1, q2)
    assert np.array_equal(s2, s1 * 2)


def test_storage_layout_is_a_bijection_with_pad_digit(orc):
    rows, k = 64, 768
    idx = set()
    for r in range(rows):
        for b in range(k // 256):
            for w in range(13):
                idx.add(orc.word_index(k, r, b, w))
    assert idx == set(range(orc.trit_words(rows, k)))
    sidx = {orc.scale_index(k, r, b) for r in range(rows) for b in range(k // 256)}
    assert sidx == set(range(orc.scale_count(rows, k)))
    # the unused level of the last word of each block is the zero weight (digit 1)
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((rows, k)) * 0.02).astype(np.float32)
    trits, _ = orc.quantize_weights(w)
    for r in (0, 17, 63):
        for b in range(k // 256):
            word = int(trits[orc.word_index(k, r, b, 12)])
            for lane in range(4):
                t = orc.trit_byte_decode((word >> (8 * lane)) & 0xFF)
                assert t[4] == 1


def test_quantize_rejects_bad_shapes(orc):
    with pytest.raises(ValueError):
        orc.quantize_weights(np.zeros((33, 256), np.float32))
    with pytest.raises(ValueError):
        orc.quantize_weights(np.zeros((32, 300), np.float32))
