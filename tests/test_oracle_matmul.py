"""Pins for the oracle's matmul y = x . W^T (W4A16 linear layer, TinyChat
README "Speed Benchmarks": 4-bit weights, fp16 activations).

Checked against: one-hot activations (y must equal a column of W^ exactly),
exact rational arithmetic on tiny shapes (Python fractions), numpy's fp64
matmul, small-integer cases whose sums are exact, and a second, factored
route through the per-group codes.
"""
from fractions import Fraction

import numpy as np
import pytest

import awq_synth
import oracle

G = 128


def _layer(N, K, tag, G=G, std=0.02):
    W = awq_synth.matrix_f16(awq_synth.key(0, 98, f"{tag}/W"), N, K, std)
    q, z, s, _ = oracle.quantize(W, G)
    return q, z, s, oracle.dequant(q, z, s, G)


def test_one_hot_activations_select_a_column():
    N, K = 32, 3 * G
    q, z, s, wh = _layer(N, K, "onehot")
    ks = [0, 1, 127, 128, 200, K - 1]
    x = np.zeros((len(ks), K), np.float16)
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    y, b = oracle.matmul(x, wh)
    for m, k in enumerate(ks):
        assert (y[m] == wh[:, k].astype(np.float64)).all()
        assert (b[m] == np.abs(wh[:, k].astype(np.float64))).all()


def test_tiny_shapes_against_exact_rationals():
    for M, K, N in [(1, 128, 16), (2, 256, 16), (3, 128, 32)]:
        q, z, s, wh = _layer(N, K, f"tiny{M}{K}{N}")
        x = awq_synth.matrix_f16(awq_synth.key(0, 98, f"tiny{M}{K}{N}/x"), M, K, 1.0)
        y, b = oracle.matmul(x, wh)
        xf = [[Fraction(float(v)) for v in row] for row in x.astype(np.float64)]
        wf = [[Fraction(float(v)) for v in row] for row in wh.astype(np.float64)]
        for m in range(M):
            for n in range(N):
                exact = sum(a * c for a, c in zip(xf[m], wf[n]))
                babs = sum(abs(a * c) for a, c in zip(xf[m], wf[n]))
                # fp64 summation of K terms: |error| <= K * 2^-53 * sum|terms|
                assert abs(Fraction(y[m, n]) - exact) <= Fraction(K, 2 ** 53) * babs
                assert abs(Fraction(b[m, n]) - babs) <= Fraction(K, 2 ** 53) * babs


def test_matches_numpy_fp64_matmul():
    N, K, M = 64, 8 * G, 5
    q, z, s, wh = _layer(N, K, "np")
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, "np/x"), M, K, 1.0)
    y, b = oracle.matmul(x, wh)
    xd, wd = x.astype(np.float64), wh.astype(np.float64)
    assert np.allclose(y, xd @ wd.T, rtol=0, atol=1e-13 * b.max())
    assert np.allclose(b, np.abs(xd) @ np.abs(wd).T, rtol=1e-13, atol=0)


def test_small_integer_sums_are_exact():
    # x small integers, W^ = (q - z) * 2^-4: every partial sum is an exact
    # multiple of 2^-4 far below 2^53, so y equals integer arithmetic.
    rng = np.random.default_rng(2)
    N, K, M = 32, 2 * G, 3
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    z = rng.integers(0, 16, (N, K // G)).astype(np.uint8)
    s = np.full((N, K // G), 2.0 ** -4, np.float16)
    wh = oracle.dequant(q, z, s, G)
    x = rng.integers(-8, 9, (M, K)).astype(np.float16)
    y, _ = oracle.matmul(x, wh)
    qi = q.astype(np.int64) - np.repeat(z.astype(np.int64), G, axis=1)
    exact = (x.astype(np.int64) @ qi.T).astype(np.float64) * 2.0 ** -4
    assert (y == exact).all()


@pytest.mark.parametrize("G", [128, 64, 32])
def test_factored_route_agrees_exactly_when_w_hat_is_exact(G):
    # power-of-two scales make every (q - z) s an exact fp16 value, so the two
    # routes differ only by fp64 summation order
    rng = np.random.default_rng(9)
    N, K, M = 48, (6 * G if 6 * G % 128 == 0 else 8 * G), 4
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    z = rng.integers(0, 16, (N, K // G)).astype(np.uint8)
    s = np.exp2(rng.integers(-12, -4, (N, K // G))).astype(np.float16)
    wh = oracle.dequant(q, z, s, G)
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, "fact/x"), M, K, 1.0)
    y, b = oracle.matmul(x, wh)
    y2 = oracle.matmul_factored(x, q, z, s, G)
    assert (np.abs(y - y2) <= 1e-12 * b).all()


def test_factored_route_within_the_rounding_of_w_hat():
    # in general W^ = fp16((q - z) s) differs from the exact product by at
    # most 2^-11 of it, so the routes agree to 2^-11 sum|x (q - z) s|
    N, K, M = 48, 6 * G, 4
    q, z, s, wh = _layer(N, K, "fact")
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, "fact/x"), M, K, 1.0)
    y, b = oracle.matmul(x, wh)
    y2 = oracle.matmul_factored(x, q, z, s, G)
    exact_abs = np.abs(x.astype(np.float64)) @ np.abs(
        (q.astype(np.float64) - np.repeat(z, G, axis=1)) * np.repeat(s.astype(np.float64), G, axis=1)).T
    assert (np.abs(y - y2) <= 2.0 ** -11 * exact_abs * (1 + 1e-9)).all()
    assert np.abs(y - y2).max() > 0          # the rounding of W^ is visible


@pytest.mark.parametrize("G", [128, 64, 32])
def test_linear_from_packed_buffers_equals_dequant_then_matmul(G):
    N, K, M = 32, 4 * G, 3
    q, z, s, wh = _layer(N, K, "lin", G)
    qw, sc, ze = oracle.pack(q, z, s, G)
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, "lin/x"), M, K, 1.0)
    y, b = oracle.matmul(x, wh)
    y2, b2 = oracle.linear(x, qw, sc, ze, N, K, G)
    assert (y == y2).all() and (b == b2).all()
    y3, _ = oracle.linear(x, qw, sc, ze, N, K, G, rows=(16, 32))
    assert (y3 == y[:, 16:32]).all()
    ms = np.array([0, 2, 1, 2])
    ns = np.array([5, 5, 31, 0])
    ye, be = oracle.linear_entries(x, qw, sc, ze, N, K, ms, ns, G)
    assert (ye == y[ms, ns]).all() and (be == b[ms, ns]).all()


def test_linearity_in_x():
    N, K = 32, 2 * G
    q, z, s, wh = _layer(N, K, "linx")
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, "linx/x"), 2, K, 1.0)
    y, b = oracle.matmul(x, wh)
    x2 = (x.astype(np.float64) * 2.0).astype(np.float16)   # exact scaling by 2
    y2, _ = oracle.matmul(x2, wh)
    assert (y2 == 2 * y).all()
    xneg = (-x.astype(np.float64)).astype(np.float16)
    y3, _ = oracle.matmul(xneg, wh)
    assert (y3 == -y).all()


def test_empty_batch():
    N, K = 16, G
    q, z, s, wh = _layer(N, K, "empty")
    y, b = oracle.matmul(np.zeros((0, K), np.float16), wh)
    assert y.shape == (0, N)
