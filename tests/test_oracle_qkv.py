"""Pins of the oracle's fused residual add + RMSNorm + QKV projection.

"rvLLM 소개" (discuss.pytorch.kr), §퓨즈드 CUDA 커널 names the fused Add+RMSNorm+QKV
kernel that feeds attention and the cache write, and gives no formula. The readings
(oracle header, R9-R11): s = binary16(x + residual) is the new residual stream;
y = s / sqrt(mean(s^2) + eps) * gamma; qkv = W y (+ bias), W's rows ordered query
heads, key heads, value heads. Each pin holds by construction: binary16 rounding from
its definition and against NumPy's IEEE conversion, closed forms worked by hand,
row selection by unit vectors, and invariances of RMSNorm.
"""
import math

import numpy as np
import pytest

import oracle
import workloads as W

F16 = np.float16


def _run(x, r, gamma, w, bias=None, eps=0.0, Hq=None, Hkv=0, D=None):
    """The oracle on a bare [N, H] weight; returns (residual_out, qkv [T, N])."""
    N = w.shape[0]
    res, q, k, v = oracle.add_rmsnorm_qkv(np.asarray(x, F16), np.asarray(r, F16), np.asarray(gamma, F16),
                                          np.asarray(w, F16), None if bias is None else np.asarray(bias, F16),
                                          eps, Hq if Hq is not None else N, Hkv, D if D is not None else 1)
    T = res.shape[0]
    return res, np.concatenate([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], axis=1)


# ------------------------------------------------------------------ binary16 rounding
def test_f16_rounding_ties_and_limits():
    cases = {
        2049.0: 2048.0,            # tie between 2048 and 2050: even significand
        2051.0: 2052.0,            # tie between 2050 and 2052: even significand
        2050.5: 2050.0,            # below the tie
        65519.0: 65504.0,          # largest finite
        2.0 ** -25: 0.0,           # tie between 0 and the smallest subnormal
        3 * 2.0 ** -25: 2.0 ** -23,
        1.0 + 2.0 ** -11: 1.0,     # tie at 1: even
        1.0 + 3 * 2.0 ** -11: 1.0 + 2.0 ** -9,
    }
    for v, want in cases.items():
        for sgn in (1.0, -1.0):
            got = oracle.f16_from_f64([sgn * v]).view(F16)[0]
            assert float(got) == sgn * want, (v, got)
    inf = oracle.f16_from_f64([65520.0, -1e9])
    assert inf.tolist() == [0x7C00, 0xFC00]
    assert np.isnan(oracle.f16_from_f64([np.nan]).view(F16)[0])


def test_f16_rounding_matches_numpy_ieee_conversion():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(4000) * np.exp2(rng.integers(-30, 15, 4000)),
        # exact ties: a binary16 value plus half its spacing
        (rng.standard_normal(2000).astype(F16).astype(np.float64) *
         (1 + np.ldexp(1.0, -11))),
    ])
    want = v.astype(F16).view(np.uint16)
    assert np.array_equal(oracle.f16_from_f64(v), want)


def test_residual_add_rounds_once_to_nearest_even():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((5, 64)) * np.exp2(rng.integers(-20, 12, (5, 64)))).astype(F16)
    r = (rng.standard_normal((5, 64)) * np.exp2(rng.integers(-20, 12, (5, 64)))).astype(F16)
    x[0, :3] = [2048, 2048, 65504]
    r[0, :3] = [1, 3, 15]                   # 65519 is below the tie at 65520
    res, _ = _run(x, r, np.ones(64), np.eye(64))
    want = (x.astype(np.float64) + r.astype(np.float64)).astype(F16)      # exact sum, one rounding
    assert np.array_equal(res.view(np.uint16), want.view(np.uint16))
    assert res[0, :3].tolist() == [2048.0, 2052.0, 65504.0]


# ------------------------------------------------------------------ closed forms
def test_worked_example_by_hand():
    """s = (3, 4): mean(s^2) = 12.5; rows of W select and combine the normalised values."""
    x = np.array([[1.0, 4.0]])
    r = np.array([[2.0, 0.0]])
    w = np.array([[1, 0], [0, 1], [1, 1], [2, -1], [0.5, 0.25]])
    bias = np.array([0, 0, 0, 0, 1.0])
    _, out = _run(x, r, [1.0, 1.0], w, bias, eps=0.0)
    root = math.sqrt(12.5)
    want = [3 / root, 4 / root, 7 / root, 2 / root, 2.5 / root + 1]
    assert np.allclose(out[0], want, rtol=1e-15, atol=0)


def test_constant_row_and_eps():
    H = 48
    for c, eps in [(0.5, 0.0), (3.0, 1e-6), (2.0, 4.0)]:
        gamma = np.linspace(0.5, 2.0, H).astype(F16)
        _, out = _run(np.full((1, H), c), np.zeros((1, H)), gamma, np.eye(H), eps=eps)
        want = c / math.sqrt(c * c + eps) * gamma.astype(np.float64)
        assert np.allclose(out[0], want, rtol=1e-14, atol=0)


def test_zero_stream_gives_the_bias():
    H, N = 32, 40
    rng = np.random.default_rng(2)
    w = rng.standard_normal((N, H)).astype(F16)
    bias = rng.standard_normal(N).astype(F16)
    _, out = _run(np.zeros((2, H)), np.zeros((2, H)), np.ones(H), w, bias, eps=1e-6)
    assert np.array_equal(out, np.broadcast_to(bias.astype(np.float64), (2, N)))


def test_unit_rows_select_the_normalised_stream():
    """W = rows of a permuted identity, N != H: out[:, n] = y[perm[n]] (no transposed operand)."""
    H, N = 24, 10
    rng = np.random.default_rng(3)
    perm = rng.permutation(H)[:N]
    w = np.zeros((N, H))
    w[np.arange(N), perm] = 1.0
    x = rng.standard_normal((3, H)).astype(F16)
    r = rng.standard_normal((3, H)).astype(F16)
    gamma = rng.uniform(0.5, 1.5, H).astype(F16)
    res, out = _run(x, r, gamma, w, eps=1e-3)
    s = res.astype(np.float64)
    y = s / np.sqrt((s * s).sum(axis=1, keepdims=True) / H + 1e-3) * gamma.astype(np.float64)
    assert np.allclose(out, y[:, perm], rtol=1e-14, atol=0)


# ------------------------------------------------------------------ invariances
def test_scale_invariance_without_eps():
    rng = np.random.default_rng(4)
    H, N = 64, 16
    x, r = rng.standard_normal((4, H)).astype(F16), rng.standard_normal((4, H)).astype(F16)
    w = rng.standard_normal((N, H)).astype(F16)
    _, a = _run(x, r, np.ones(H), w)
    _, b = _run(x * F16(8), r * F16(8), np.ones(H), w)          # powers of two stay exact
    assert np.allclose(a, b, rtol=1e-13, atol=1e-13)


def test_linear_in_the_weights_and_gamma():
    rng = np.random.default_rng(5)
    H, N = 40, 12
    x, r = rng.standard_normal((3, H)).astype(F16), rng.standard_normal((3, H)).astype(F16)
    w1, w2 = rng.standard_normal((N, H)).astype(F16), rng.standard_normal((N, H)).astype(F16)
    g = rng.uniform(0.5, 1.5, H).astype(F16)
    _, a = _run(x, r, g, w1, eps=1e-6)
    _, b = _run(x, r, g, w2, eps=1e-6)
    _, c = _run(x, r, g, np.concatenate([w1, w2]), eps=1e-6)
    assert np.array_equal(c, np.concatenate([a, b], axis=1))
    _, d = _run(x, r, g * F16(2), w1, eps=1e-6)
    assert np.allclose(d, 2 * a, rtol=1e-13, atol=1e-13)


def test_tokens_are_independent():
    rng = np.random.default_rng(6)
    H, N = 32, 8
    x, r = rng.standard_normal((6, H)).astype(F16), rng.standard_normal((6, H)).astype(F16)
    w = rng.standard_normal((N, H)).astype(F16)
    _, a = _run(x, r, np.ones(H), w, eps=1e-6)
    p = rng.permutation(6)
    _, b = _run(x[p], r[p], np.ones(H), w, eps=1e-6)
    assert np.array_equal(b, a[p])


def test_qkv_split_follows_the_row_order():
    """With a zero stream the outputs are the bias; its three slices land in q, k and v by head."""
    Hq, Hkv, D, H = 6, 2, 8, 16
    N = (Hq + 2 * Hkv) * D
    bias = np.arange(N, dtype=np.float64).astype(F16)
    _, q, k, v = oracle.add_rmsnorm_qkv(np.zeros((2, H), F16), np.zeros((2, H), F16), np.ones(H, F16),
                                        np.ones((N, H), F16), bias, 1e-6, Hq, Hkv, D)
    for t in range(2):
        assert np.array_equal(q[t], np.arange(Hq * D).reshape(Hq, D))
        assert np.array_equal(k[t], Hq * D + np.arange(Hkv * D).reshape(Hkv, D))
        assert np.array_equal(v[t], (Hq + Hkv) * D + np.arange(Hkv * D).reshape(Hkv, D))


def test_empty_batch_and_bad_sizes():
    res, q, k, v = oracle.add_rmsnorm_qkv(np.zeros((0, 16), F16), np.zeros((0, 16), F16), np.ones(16, F16),
                                          np.ones((24, 16), F16), None, 1e-6, 1, 1, 8)
    assert res.shape == (0, 16) and q.shape == (0, 1, 8) and v.shape == (0, 1, 8)
    with pytest.raises(ValueError):
        oracle.add_rmsnorm_qkv(np.zeros((1, 16), F16), np.zeros((1, 16), F16), np.ones(16, F16),
                               np.ones((24, 16), F16), None, -1.0, 1, 1, 8)


def test_generated_inputs_have_the_stated_shapes():
    s = W.QKV_SHAPES["qwen2.5-1.5b"]
    d = W.make_qkv_inputs(3, s["H"], s["Hq"], s["Hkv"], s["D"], 0, outliers=True)
    N = (s["Hq"] + 2 * s["Hkv"]) * s["D"]
    assert d["x"].shape == (3, s["H"]) and d["w_qkv"].shape == (N, s["H"]) and d["bias"].shape == (N,)
    assert np.abs(d["residual"].astype(np.float32)).max() >= 1e4      # the planted outliers
