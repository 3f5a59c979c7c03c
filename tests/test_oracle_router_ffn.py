"""Pins for the oracle's router and expert FFN (CPU only)."""
import numpy as np
import pytest
import scipy.special

import synthetic


# ------------------------------------------------------------------ router
def test_router_fixed_order_hand_case(orc):
    """hidden = 64: products 2^24 at k=0, 1 at k=32 (both in partial 0) and
    -2^24 at k=16 (partial 16).  In the fixed order partial 0 is
    fmaf(1, 1, 2^24) = 2^24 (the tie rounds to even), and the first pairwise
    round cancels it with partial 16: the logit is 0, not the exact sum 1."""
    x = np.zeros(64, np.float32)
    w = np.zeros((1, 64), np.float32)
    x[0], w[0, 0] = 2.0 ** 12, 2.0 ** 12
    x[32], w[0, 32] = 1.0, 1.0
    x[16], w[0, 16] = -(2.0 ** 12), 2.0 ** 12
    assert orc.router_logits(x, w)[0, 0] == 0.0
    # moving the 1 into its own partial makes every step exact
    x2, w2 = x.copy(), w.copy()
    x2[32], w2[0, 32] = 0.0, 0.0
    x2[33], w2[0, 33] = 1.0, 1.0
    assert orc.router_logits(x2, w2)[0, 0] == 1.0


def test_router_logits_error_bound(orc):
    rng = np.random.default_rng(31)
    H, E = 2048, 64
    x = rng.standard_normal((4, H)).astype(np.float32)
    wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    lg = orc.router_logits(x, wr).astype(np.float64)
    exact = x.astype(np.float64) @ wr.astype(np.float64).T
    mag = np.abs(x.astype(np.float64)) @ np.abs(wr.astype(np.float64)).T
    n = H // 32 + 5
    assert np.all(np.abs(lg - exact) <= n * 2.0 ** -24 * mag * 1.01)


def test_topk_matches_stable_argsort_and_softmax(orc):
    rng = np.random.default_rng(32)
    H, E, K = 256, 32, 6
    x = rng.standard_normal((16, H)).astype(np.float32)
    wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    wr[7] = wr[3]                       # a guaranteed tie: id 3 ranks before 7
    idx, wts = orc.route_topk(x, wr, K)
    lg = orc.router_logits(x, wr)
    for t in range(16):
        order = np.argsort(-lg[t].astype(np.float64), kind="stable")[:K]
        assert list(idx[t]) == list(order)
        sel = lg[t, idx[t]].astype(np.float64)
        assert np.allclose(wts[t], scipy.special.softmax(sel), rtol=1e-13, atol=0)
        assert abs(wts[t].sum() - 1.0) < 1e-14
        where3 = np.where(idx[t] == 3)[0]
        where7 = np.where(idx[t] == 7)[0]
        if len(where7):
            assert len(where3) and where3[0] + 1 == where7[0]


def test_topk_all_and_one(orc):
    rng = np.random.default_rng(33)
    H, E = 512, 8
    x = rng.standard_normal((3, H)).astype(np.float32)
    wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    idx, wts = orc.route_topk(x, wr, 1)
    assert np.all(wts == 1.0)
    idx, wts = orc.route_topk(x, wr, E)
    lg = orc.router_logits(x, wr).astype(np.float64)
    full = scipy.special.softmax(lg, axis=1)
    for t in range(3):
        assert np.allclose(wts[t], full[t, idx[t]], rtol=1e-13, atol=0)
    # permuting the router rows permutes the chosen ids
    perm = rng.permutation(E)
    idx2, wts2 = orc.route_topk(x, wr[perm], 3)
    idx3, wts3 = orc.route_topk(x, wr, 3)
    assert np.array_equal(perm[idx2], idx3)
    assert np.array_equal(wts2, wts3)
    with pytest.raises(ValueError):
        orc.route_topk(x, wr, E + 1)


# ------------------------------------------------------------------ expert FFN
def _tiny(orc, H=256, F=512, E=4, K=2, seed=5, std=0.05):
    rng = np.random.default_rng(seed)
    wg = (rng.standard_normal((E * F, H)) * std).astype(np.float32)
    wu = (rng.standard_normal((E * F, H)) * std).astype(np.float32)
    wd = (rng.standard_normal((E * H, F)) * std).astype(np.float32)
    wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    x = rng.standard_normal((3, H)).astype(np.float32)
    return (wg, wu, wd, wr, x)


def _dense_mixture(orc, layer, wr, x, unpack=None):
    """Independent dense evaluation of a layer that routes to every expert:
    y = sum_e softmax(logits)_e * Wd_e (q8(silu(Wg_e x^) * Wu_e x^))^.
    `unpack` expands a packed matrix (the ternary unpacking by default)."""
    unpack = orc.unpack_weights if unpack is None else unpack
    H, F, E = layer.hidden, layer.ffn, layer.n_experts
    xq, xd = orc.quant_act_q8(x)
    lg = orc.router_logits(x, wr).astype(np.float64)
    p = scipy.special.softmax(lg, axis=1)
    xdeq = xq.astype(np.float64) * np.repeat(xd.astype(np.float64), 32, axis=1)

    def deq(mat, rows, k, e):
        q, s = unpack(mat[0], mat[1], E * rows, k, e * rows, rows)
        return q.astype(np.float64) * np.repeat(s.astype(np.float64), 256, axis=1)

    y = np.zeros((x.shape[0], H))
    for e in range(E):
        G, U, D = deq(layer.gate, F, H, e), deq(layer.up, F, H, e), deq(layer.down, H, F, e)
        g = xdeq @ G.T
        u = xdeq @ U.T
        a = (g / (1.0 + np.exp(-g)) * u).astype(np.float32)
        aq, ad = orc.quant_act_q8(a)
        adeq = aq.astype(np.float64) * np.repeat(ad.astype(np.float64), 32, axis=1)
        y += p[:, e:e + 1].astype(np.float32).astype(np.float64) * (adeq @ D.T)
    return y


def test_ffn_route_all_equals_dense_mixture(orc):
    H, F, E = 256, 512, 4
    wg, wu, wd, wr, x = _tiny(orc, H, F, E)
    layer = orc.Layer.from_float(H, F, E, E, wg, wu, wd)
    y, idx, wts = orc.moe_forward(layer, wr, x)
    ref = _dense_mixture(orc, layer, wr, x)
    scale = np.abs(ref).max()
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * scale)
    assert scale > 1e-3


def test_ffn_zero_weights_give_zero(orc):
    H, F, E, K = 256, 256, 4, 2
    z = np.zeros
    layer = orc.Layer.from_float(H, F, E, K, z((E * F, H), np.float32),
                                 z((E * F, H), np.float32), z((E * H, F), np.float32))
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, H)).astype(np.float32)
    wr = rng.standard_normal((E, H)).astype(np.float32)
    y, _, _ = orc.moe_forward(layer, wr, x)
    assert not y.any()


def test_ffn_expert_permutation_invariance(orc):
    H, F, E, K = 256, 256, 6, 3
    wg, wu, wd, wr, x = _tiny(orc, H, F, E, seed=9)
    perm = np.random.default_rng(1).permutation(E)

    def blocks(m, rows):
        return m.reshape(E, rows, -1)[perm].reshape(E * rows, -1)

    l1 = orc.Layer.from_float(H, F, E, K, wg, wu, wd)
    l2 = orc.Layer.from_float(H, F, E, K, blocks(wg, F), blocks(wu, F), blocks(wd, H))
    y1, i1, _ = orc.moe_forward(l1, wr, x)
    y2, i2, _ = orc.moe_forward(l2, wr[perm], x)
    assert np.array_equal(perm[i2], i1)
    assert np.array_equal(y1, y2)


def test_ffn_batch_equals_single_tokens(orc):
    H, F, E, K = 256, 512, 4, 2
    wg, wu, wd, wr, x = _tiny(orc, H, F, E)
    layer = orc.Layer.from_float(H, F, E, K, wg, wu, wd)
    y, _, _ = orc.moe_forward(layer, wr, x)
    for t in range(x.shape[0]):
        yt, _, _ = orc.moe_forward(layer, wr, x[t:t + 1])
        assert np.array_equal(yt[0], y[t])


def test_ffn_exact_scaling_of_up_and_down(orc):
    """Doubling Wu doubles u, a, the q8 scale of a and y exactly; doubling Wd
    doubles y exactly."""
    H, F, E, K = 256, 512, 4, 2
    wg, wu, wd, wr, x = _tiny(orc, H, F, E)
    two = np.float32(2)
    y0, _, _ = orc.moe_forward(orc.Layer.from_float(H, F, E, K, wg, wu, wd), wr, x)
    y1, _, _ = orc.moe_forward(orc.Layer.from_float(H, F, E, K, wg, wu * two, wd), wr, x)
    y2, _, _ = orc.moe_forward(orc.Layer.from_float(H, F, E, K, wg, wu, wd * two), wr, x)
    assert np.array_equal(y1, 2 * y0)
    assert np.array_equal(y2, 2 * y0)


def test_ffn_single_expert_closed_form(orc):
    """One expert, top-1, ternary diagonal weights: each 256-block of row r
    holds a single +1 at column r, so every nonzero dequantizes to c/256 and
    g = u = (c/256) x^, y = (c/256) q8(silu(g) * u)^, all by hand."""
    H = F = 256
    c = 64.0
    eye = (np.eye(H) * c).astype(np.float32)
    layer = orc.Layer.from_float(H, F, 1, 1, eye, eye, eye)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((1, H)).astype(np.float32)
    wr = np.zeros((1, H), np.float32)
    y, idx, wts = orc.moe_forward(layer, wr, x)
    assert idx[0, 0] == 0 and wts[0, 0] == 1.0
    xq, xd = orc.quant_act_q8(x)
    xh = xq[0].astype(np.float64) * np.repeat(xd[0].astype(np.float64), 32)
    g = (c / 256) * xh
    a = (g / (1 + np.exp(-g)) * g).astype(np.float32)
    aq, ad = orc.quant_act_q8(a)
    ref = (c / 256) * aq[0].astype(np.float64) * np.repeat(ad[0].astype(np.float64), 32)
    assert np.array_equal(y[0], ref)


def test_ffn_rejects_bad_expert_ids(orc):
    H, F, E, K = 256, 256, 2, 1
    wg, wu, wd, wr, x = _tiny(orc, H, F, E)
    layer = orc.Layer.from_float(H, F, E, K, wg, wu, wd)
    xq, xd = orc.quant_act_q8(x[:1])
    with pytest.raises(IndexError):
        orc.expert_ffn(layer, xq, xd, np.array([[E]], np.int32), np.ones((1, 1), np.float32))


def test_synthetic_inputs_are_deterministic():
    wl = synthetic.WORKLOADS["tiny"]
    a = synthetic.expert_matrix(wl, 0, "gate", 3).numpy()
    b = synthetic.expert_matrix(wl, 0, "gate", 3).numpy()
    c = synthetic.expert_matrix(wl, 0, "gate", 4).numpy()
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert abs(a.std() - 0.02) < 0.002


def test_swiglu_against_fixed_values(orc):
    """The activation between gate/up and down, pinned to literal values of
    SiLU (a = g * sigmoid(g) * u; pxq_llama README, "Updates -- 2026-07-28":
    the SiLU unary of the gate), so that a wrong activation shared with a
    numpy restatement cannot pass.  One expert, top-1; single-nonzero weight
    blocks and integer activation blocks with amax 127 make g and u exact:
      - up: every row holds 4 at column 0 (scale 1/64), x[0] = 64, so u = 1;
      - gate rows 32..35 hold 4 at their own column (scale 1/64), x = 127, 64,
        -64, 0, so g = 1.984375, 1, -1, 0;
      - gate rows 64, 65 hold 256 at their own column (scale 1), x = 127, -127,
        so g = 127, -127 (the large-|g| limits);
      - gate rows 0..31 are zero, so that activation block is all zeros.
    The SwiGLU output is observed through its int8 requantization, within half
    a quantization step of the literal values."""
    H = F = 256
    wg = np.zeros((F, H), np.float32)
    for r in (32, 33, 34, 35):
        wg[r, r] = 4.0
    for r in (64, 65):
        wg[r, r] = 256.0
    wu = np.zeros((F, H), np.float32)
    wu[:, 0] = 4.0
    wd = np.zeros((H, F), np.float32)
    layer = orc.Layer.from_float(H, F, 1, 1, wg, wu, wd)
    x = np.zeros((1, H), np.float32)
    x[0, 0], x[0, 1] = 64.0, 127.0
    x[0, 32:36] = [127.0, 64.0, -64.0, 0.0]
    x[0, 64], x[0, 65] = 127.0, -127.0
    xq, xd = orc.quant_act_q8(x)
    assert np.array_equal(xq[0].astype(np.float32) * np.repeat(xd[0], 32), x[0])  # exact inputs
    _, dbg = orc.expert_ffn(layer, xq, xd, np.array([[0]], np.int32), np.ones((1, 1), np.float32), debug=True)
    g, u, aq, ad = dbg["g"][0, 0], dbg["u"][0, 0], dbg["aq"][0, 0].astype(np.int64), dbg["ad"][0, 0]
    assert np.all(u == 1.0)
    assert list(g[32:36]) == [1.984375, 1.0, -1.0, 0.0] and list(g[64:66]) == [127.0, -127.0]
    assert np.all(g[:32] == 0.0) and np.all(aq[:32] == 0) and ad[0] == 0.0
    # block 1: amax = silu(1.984375) = 1.7445568667767222..., so ad = amax / 127
    assert abs(float(ad[1]) * 127 - 1.7445568667767222) < 1e-6
    step = float(ad[1])
    assert aq[32] == 127
    assert abs(aq[33] * step - 0.7310585786300049) <= step / 2    # silu(1)
    assert abs(aq[34] * step - (-0.2689414213699951)) <= step / 2  # silu(-1)
    assert aq[35] == 0                                              # silu(0) = 0
    # block 2: silu(127) = 127 to fp32 precision, silu(-127) ~ -8.9e-54
    assert float(ad[2]) == 1.0 and aq[64] == 127 and aq[65] == 0
