"""Pins for the oracle's elementary operators (CPU only).

Each check compares against something other than the oracle's own formula:
brute-force loops over tiny inputs, closed forms, invariants and special cases.
"""
import math
import itertools

import numpy as np
import pytest

import oracle
from oracle import ops


def rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------- conv

def conv_brute(x, w, b, stride, pad):
    C, H, W = x.shape
    O, _, k, _ = w.shape
    Ho = (H + 2 * pad - k) // stride + 1
    Wo = (W + 2 * pad - k) // stride + 1
    y = np.zeros((O, Ho, Wo))
    for o in range(O):
        for i in range(Ho):
            for j in range(Wo):
                acc = 0.0 if b is None else float(b[o])
                for c in range(C):
                    for u in range(k):
                        for v in range(k):
                            yy = stride * i + u - pad
                            xx = stride * j + v - pad
                            if 0 <= yy < H and 0 <= xx < W:
                                acc += float(w[o, c, u, v]) * float(x[c, yy, xx])
                y[o, i, j] = acc
    return y


def conv_im2col(x, w, b, stride, pad):
    """Independent im2col + one matrix product."""
    C, H, W = x.shape
    O, _, k, _ = w.shape
    Ho = (H + 2 * pad - k) // stride + 1
    Wo = (W + 2 * pad - k) // stride + 1
    cols = np.zeros((C * k * k, Ho * Wo))
    for c in range(C):
        for u in range(k):
            for v in range(k):
                r = (c * k + u) * k + v
                for i in range(Ho):
                    for j in range(Wo):
                        yy, xx = stride * i + u - pad, stride * j + v - pad
                        if 0 <= yy < H and 0 <= xx < W:
                            cols[r, i * Wo + j] = x[c, yy, xx]
    y = (w.reshape(O, -1) @ cols).reshape(O, Ho, Wo)
    return y + (0 if b is None else b.reshape(O, 1, 1))


@pytest.mark.parametrize("C,O,H,W,stride,pad,k", [
    (3, 4, 5, 6, 1, 1, 3), (5, 2, 7, 5, 2, 1, 3), (4, 3, 6, 6, 1, 0, 1), (8, 5, 5, 7, 2, 1, 3),
    (2, 3, 4, 4, 1, 1, 3)])
def test_conv_matches_brute_force_and_im2col(C, O, H, W, stride, pad, k):
    r = rng(C * 100 + H)
    x = r.standard_normal((C, H, W))
    w = r.standard_normal((O, C, k, k))
    b = r.standard_normal(O)
    y = ops.conv2d(x, w, b, stride, pad)
    np.testing.assert_allclose(y, conv_brute(x, w, b, stride, pad), rtol=0, atol=1e-9)
    np.testing.assert_allclose(y, conv_im2col(x, w, b, stride, pad), rtol=0, atol=1e-9)


def test_conv_delta_kernel_is_identity_and_shift():
    r = rng(1)
    C, H, W = 3, 5, 6
    x = r.standard_normal((C, H, W))
    w = np.zeros((C, C, 3, 3))
    for c in range(C):
        w[c, c, 1, 1] = 1.0
    np.testing.assert_array_equal(ops.conv2d(x, w, None, 1, 1), x)
    # tap (0, 0) reads the pixel up-left: y[i, j] = x[i-1, j-1], zero on the border
    w2 = np.zeros((C, C, 3, 3))
    for c in range(C):
        w2[c, c, 0, 0] = 1.0
    y = ops.conv2d(x, w2, None, 1, 1)
    np.testing.assert_array_equal(y[:, 1:, 1:], x[:, :-1, :-1])
    assert np.all(y[:, 0, :] == 0) and np.all(y[:, :, 0] == 0)


def test_conv_all_ones_counts_padding():
    C, H, W = 4, 6, 7
    y = ops.conv2d(np.ones((C, H, W)), np.ones((1, C, 3, 3)), None, 1, 1)[0]
    assert y[2, 3] == 9 * C
    assert y[0, 3] == 6 * C and y[H - 1, 3] == 6 * C and y[2, 0] == 6 * C and y[2, W - 1] == 6 * C
    assert y[0, 0] == 4 * C and y[H - 1, W - 1] == 4 * C and y[0, W - 1] == 4 * C


def test_stride2_is_subsampled_stride1():
    r = rng(2)
    x = r.standard_normal((6, 8, 10))
    w = r.standard_normal((4, 6, 3, 3))
    b = r.standard_normal(4)
    s1 = ops.conv2d(x, w, b, 1, 1)
    s2 = ops.conv2d(x, w, b, 2, 1)
    assert s2.shape == (4, 4, 5)
    np.testing.assert_array_equal(s2, s1[:, ::2, ::2])


def test_upsample_nearest_brute():
    r = rng(3)
    x = r.standard_normal((3, 4, 5))
    u = ops.upsample_nearest2x(x)
    assert u.shape == (3, 8, 10)
    for c, i, j in itertools.product(range(3), range(8), range(10)):
        assert u[c, i, j] == x[c, i // 2, j // 2]


def test_upsample_conv_equals_conv_of_materialised():
    r = rng(4)
    x = r.standard_normal((3, 3, 4))
    w = r.standard_normal((2, 3, 3, 3))
    b = r.standard_normal(2)
    big = np.zeros((3, 6, 8))
    for i in range(6):
        for j in range(8):
            big[:, i, j] = x[:, i // 2, j // 2]
    p = {"u.weight": w, "u.bias": b}
    np.testing.assert_allclose(oracle.upsample(x, p, "u"), conv_brute(big, w, b, 1, 1), atol=1e-9)


# ----------------------------------------------------------------------------- norms

@pytest.mark.parametrize("C,G", [(64, 32), (96, 32), (8, 8), (12, 1)])
def test_group_norm_moments(C, G):
    r = rng(C + G)
    sigma = 3.0
    x = 1.5 + sigma * r.standard_normal((C, 5, 7))
    eps = 1e-5
    y = ops.group_norm(x, np.ones(C), np.zeros(C), G, eps)
    cpg = C // G
    for g in range(G):
        blk = y[g * cpg:(g + 1) * cpg]
        xb = x[g * cpg:(g + 1) * cpg]
        assert abs(blk.mean()) < 1e-10
        v = xb.var()
        assert abs(blk.var() - v / (v + eps)) < 1e-10


def test_group_norm_brute_with_affine():
    r = rng(7)
    C, G, H, W = 8, 4, 3, 3
    x = r.standard_normal((C, H, W))
    gam = r.standard_normal(C)
    bet = r.standard_normal(C)
    y = ops.group_norm(x, gam, bet, G, 1e-5)
    for g in range(G):
        vals = [x[c, i, j] for c in range(2 * g, 2 * g + 2) for i in range(H) for j in range(W)]
        m = sum(vals) / len(vals)
        var = sum((v - m) ** 2 for v in vals) / len(vals)
        for c in range(2 * g, 2 * g + 2):
            for i in range(H):
                for j in range(W):
                    ref = (x[c, i, j] - m) / math.sqrt(var + 1e-5) * gam[c] + bet[c]
                    assert abs(y[c, i, j] - ref) < 1e-12


def test_group_norm_g_equals_c_is_instance_norm():
    r = rng(8)
    x = r.standard_normal((6, 4, 4)) * 2 + 1
    y = ops.group_norm(x, np.ones(6), np.zeros(6), 6, 0.0)
    for c in range(6):
        assert abs(y[c].mean()) < 1e-12 and abs(y[c].std() - 1) < 1e-12


def test_layer_norm_per_token():
    r = rng(9)
    t = 4 + 2 * r.standard_normal((11, 64))
    y = ops.layer_norm(t, np.ones(64), np.zeros(64), 1e-5)
    v = t.var(axis=1)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose(y.var(axis=1), v / (v + 1e-5), atol=1e-12)
    g = r.standard_normal(64)
    b = r.standard_normal(64)
    np.testing.assert_allclose(ops.layer_norm(t, g, b, 1e-5), y * g + b, atol=1e-12)


# ----------------------------------------------------------------------------- attention

def attention_brute(q, k, v, hd):
    Nq, C = q.shape
    out = np.zeros((Nq, C))
    for h in range(C // hd):
        for i in range(Nq):
            s = [sum(q[i, h * hd + d] * k[j, h * hd + d] for d in range(hd)) / math.sqrt(hd)
                 for j in range(k.shape[0])]
            m = max(s)
            e = [math.exp(z - m) for z in s]
            tot = sum(e)
            for d in range(hd):
                out[i, h * hd + d] = sum(e[j] * v[j, h * hd + d] for j in range(k.shape[0])) / tot
    return out


def test_layer_norm_folds_into_the_following_linear():
    """The identity the GPU path uses instead of a LayerNorm kernel:
    LN(x) W^T + b = rstd (x (W*gamma)^T - mean c1) + c2, c1 = rowsum(W*gamma),
    c2 = W beta + b, with mean and rstd of each row of x (biased variance) and
    the row statistics taken from sum x and sum x^2 as the GPU accumulates them."""
    rng = np.random.default_rng(7)
    N, C, O, eps = 11, 48, 20, 1e-5
    x = rng.normal(0.3, 1.7, (N, C))
    gamma, beta = 1 + 0.2 * rng.normal(size=C), 0.3 * rng.normal(size=C)
    W, bias = rng.normal(size=(O, C)) / math.sqrt(C), rng.normal(size=O)
    ref = ops.linear(ops.layer_norm(x, gamma, beta, eps), W, bias)
    Wg = W * gamma[None, :]
    c1, c2 = Wg.sum(axis=1), W @ beta + bias
    s1, s2 = x.sum(axis=1), (x * x).sum(axis=1)
    mean = s1 / C
    rstd = 1 / np.sqrt(s2 / C - mean ** 2 + eps)
    folded = rstd[:, None] * (x @ Wg.T - mean[:, None] * c1[None, :]) + c2[None, :]
    np.testing.assert_allclose(folded, ref, rtol=1e-11, atol=1e-11)
    # a dropped term is caught: without c1 (or with gamma left out) the results differ
    assert not np.allclose(rstd[:, None] * (x @ Wg.T) + c2[None, :], ref, atol=1e-3)
    assert not np.allclose(rstd[:, None] * (x @ W.T - mean[:, None] * W.sum(axis=1)) + c2[None, :], ref, atol=1e-3)


def test_attention_brute_force_small():
    r = rng(10)
    q, k, v = (r.standard_normal((5, 8)) for _ in range(3))
    kk = r.standard_normal((7, 8))
    vv = r.standard_normal((7, 8))
    np.testing.assert_allclose(ops.attention(q, kk, vv, 4), attention_brute(q, kk, vv, 4), atol=1e-12)
    np.testing.assert_allclose(ops.attention(q, k, v, 8), attention_brute(q, k, v, 8), atol=1e-12)


def test_attention_rows_sum_to_one_single_key_and_mean():
    r = rng(11)
    q = 3 * r.standard_normal((9, 128))
    k = 3 * r.standard_normal((13, 128))
    # V = 1 everywhere: output = sum_j P_ij = 1 when rows of P sum to 1
    np.testing.assert_allclose(ops.attention(q, k, np.ones((13, 128))), 1.0, atol=1e-12)
    # one key: output is V exactly
    v1 = r.standard_normal((1, 128))
    np.testing.assert_array_equal(ops.attention(q, k[:1], v1), np.repeat(v1, 9, axis=0))
    # Q = 0: uniform weights, output is the mean of V
    v = r.standard_normal((13, 128))
    np.testing.assert_allclose(ops.attention(np.zeros((9, 128)), k, v), np.repeat(v.mean(0, keepdims=True), 9, 0),
                               atol=1e-12)


def test_attention_permutation_symmetries():
    r = rng(12)
    x = r.standard_normal((10, 64))
    perm = r.permutation(10)
    a = ops.attention(x, x, x)
    np.testing.assert_allclose(ops.attention(x[perm], x[perm], x[perm]), a[perm], atol=1e-12)
    ctx = r.standard_normal((77, 64))
    p2 = r.permutation(77)
    np.testing.assert_allclose(ops.attention(x, ctx[p2], ctx[p2] * 2), ops.attention(x, ctx, ctx * 2), atol=1e-12)


def test_attention_large_logits_stable():
    q = np.full((2, 64), 10.0)
    k = np.full((3, 64), 10.0)
    k[1] *= -1
    v = np.arange(3 * 64, dtype=float).reshape(3, 64)
    out = ops.attention(q, k, v)
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out[0], (v[0] + v[2]) / 2, atol=1e-9)


# ----------------------------------------------------------------------------- GELU / GEGLU

@pytest.mark.parametrize("x", [-6.0, -3.0, -1.0, -0.5, 0.0, 0.1, 0.7, 1.0, 2.5, 5.0])
def test_gelu_closed_form(x):
    ref = 0.5 * x * (1.0 + math.erf(x / math.sqrt(2.0)))
    assert abs(ops.gelu(np.array([x]))[0] - ref) < 1e-15


def test_gelu_limits():
    assert ops.gelu(np.array([0.0]))[0] == 0.0
    assert abs(ops.gelu(np.array([12.0]))[0] - 12.0) < 1e-12
    assert abs(ops.gelu(np.array([-12.0]))[0]) < 1e-12
    # GELU(1) = Phi(1) = 0.841344746068543 (standard normal CDF at 1)
    assert abs(ops.gelu(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15


def test_geglu_ff_brute():
    r = rng(13)
    C = 2
    t = r.standard_normal((3, C))
    w1 = r.standard_normal((8 * C, C))
    b1 = r.standard_normal(8 * C)
    w2 = r.standard_normal((C, 4 * C))
    b2 = r.standard_normal(C)
    y = ops.geglu_ff(t, w1, b1, w2, b2)
    for n in range(3):
        u = [sum(w1[o, i] * t[n, i] for i in range(C)) + b1[o] for o in range(8 * C)]
        m = [u[j] * 0.5 * u[4 * C + j] * (1 + math.erf(u[4 * C + j] / math.sqrt(2))) for j in range(4 * C)]
        for o in range(C):
            ref = sum(w2[o, j] * m[j] for j in range(4 * C)) + b2[o]
            assert abs(y[n, o] - ref) < 1e-12


# ----------------------------------------------------------------------------- timestep embedding

def test_timestep_embedding_properties():
    e0 = ops.timestep_embedding(0.0, 320)
    np.testing.assert_array_equal(e0[:160], 1.0)
    np.testing.assert_array_equal(e0[160:], 0.0)
    e = ops.timestep_embedding(500.0, 320)
    np.testing.assert_allclose(e[:160] ** 2 + e[160:] ** 2, 1.0, atol=1e-15)
    assert abs(e[0] - math.cos(500.0)) < 1e-15 and abs(e[160] - math.sin(500.0)) < 1e-15
    f_last = 10000.0 ** (-159 / 160)
    assert abs(e[159] - math.cos(500.0 * f_last)) < 1e-12


def test_bf16_round_known_values():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -7, -2.5, 3.0e38])
    r = ops.bf16_round(vals)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to even (1.0)
    assert r[0] == 1.0 and r[1] == 1.0
    assert r[2] == 1.0 + 2 ** -6  # tie between 1+2^-7 and 1+2^-6, rounds to even mantissa
    assert r[3] == 1.0 + 2 ** -7 and r[4] == -2.5


# ----------------------------------------------------------------------------- SiLU

@pytest.mark.parametrize("x,expected", [
    (0.0, 0.0),
    (1.0, 0.7310585786300049),    # 1 * logistic(1), tabulated
    (-1.0, -0.2689414213699951),  # -1 * logistic(-1)
    (2.0, 1.7615941559557649),    # 2 * logistic(2)
    (-2.0, -0.2384058440442351),
])
def test_silu_tabulated(x, expected):
    assert abs(float(ops.silu(np.array([x]))[0]) - expected) < 1e-15


def test_silu_limits_and_even_part():
    """SiLU(x) -> x for large x and -> 0 for very negative x; its even part
    SiLU(x) + SiLU(-x) equals x * tanh(x / 2) (a sign slip, a dropped x or a
    plain sigmoid breaks one of these)."""
    big = np.array([30.0, 40.0])
    np.testing.assert_allclose(ops.silu(big), big, rtol=1e-12)
    assert np.all(np.abs(ops.silu(-big)) < 1e-11)
    x = np.linspace(-6.0, 6.0, 49)
    np.testing.assert_allclose(ops.silu(x) + ops.silu(-x), x * np.tanh(x / 2.0), atol=1e-14)
    np.testing.assert_allclose(ops.silu(x) - ops.silu(-x), x, atol=1e-14)
