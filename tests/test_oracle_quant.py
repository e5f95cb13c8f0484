"""Pins for the oracle's group quantization (4-bit, group 128, asymmetric
min-max with fp16 scale and 4-bit zero point; TinyChat README, Usage step 3).

Each pin checks the oracle against something other than its own formula:
hand-derived groups (tests/golden/quant_groups.txt), groups built from exact
(q, z, s) that must come back unchanged with zero error, a brute-force search
over all 16 codes (every q is a nearest grid point), the per-element error
bound, and invariances (power-of-two scaling, permutation within a group).
"""
import numpy as np
import pytest

import awq_synth
import oracle
from golden_io import quant_groups

G = 128


def test_hand_derived_groups():
    for c in quant_groups(G):
        W = np.tile(c["v"], (16, 1))          # 16 identical rows, one group each
        q, z, s, _ = oracle.quantize(W, G)
        wh = oracle.dequant(q, z, s, G).view(np.uint16)
        for r in range(16):
            assert s.view(np.uint16)[r, 0] == c["s"], c["name"]
            assert z[r, 0] == c["z"], c["name"]
            assert (q[r] == c["q"]).all(), c["name"]
            for i, bits in c["w"].items():
                assert wh[r, i] == bits, (c["name"], i, hex(wh[r, i]), hex(bits))


def _exact_groups(rng, N, K, G=G):
    """W built from random (q, z, s) with s = m * 2^e (m odd <= 127) and every
    group spanning the whole grid (one q = 0 and one q = 15), so that every
    (q - z) * s is an exact fp16 value, hi - lo = 15 s and R / 15 = s exactly."""
    ng = K // G
    z = rng.integers(0, 16, (N, ng))
    m = rng.integers(0, 64, (N, ng)) * 2 + 1
    e = rng.integers(-14, -6, (N, ng))
    s = m * np.exp2(e)
    q = rng.integers(0, 16, (N, K))
    for n in range(N):
        for g in range(ng):
            a, b = rng.choice(G, 2, replace=False)
            q[n, g * G + a] = 0
            q[n, g * G + b] = 15
    w = (q - np.repeat(z, G, axis=1)) * np.repeat(s, G, axis=1)
    W = w.astype(np.float16)
    assert (W.astype(np.float64) == w).all()
    return W, q, z, s


@pytest.mark.parametrize("G", [128, 64, 32])
def test_exactly_representable_weights_have_zero_error(G):
    rng = np.random.default_rng(7)
    W, q0, z0, s0 = _exact_groups(rng, 64, 4 * G, G)
    q, z, s, _ = oracle.quantize(W, G)
    assert (q == q0).all()
    assert (z == z0).all()
    assert (s.astype(np.float64) == s0).all()
    wh = oracle.dequant(q, z, s, G)
    assert (wh.view(np.uint16) == W.view(np.uint16)).all()


def _random_weights(G=G):
    """Seeded weights with the value mixes the kernels meet: N(0, 0.02),
    outlier channels x20, all-positive and all-negative groups, groups whose
    range is so small that the scale is subnormal, and constant groups."""
    N, K = 64, 8 * G
    wl = awq_synth.WORKLOADS["llama2_70b_decode"]
    W = awq_synth.matrix_f16(awq_synth.key(0, 99, "pins/W"), N, K, 0.02).astype(np.float64)
    ch = awq_synth.pick_channels(awq_synth.key(0, 99, "pins/out"), K, 10)
    W[:, ch] *= wl.outlier_mult
    W[0:8, 0:G] = np.abs(W[0:8, 0:G]) + 0.01           # all positive -> z clamps to 0
    W[8:16, G:2 * G] = -np.abs(W[8:16, G:2 * G]) - 0.01  # all negative -> z clamps to 15
    W[16:24, 2 * G:3 * G] *= 1e-3                      # range < 15 * 2^-14 -> subnormal s
    W[24:32, 3 * G:4 * G] = 0.25                       # constant groups
    W[32:40, 4 * G:5 * G] = 0.0                        # all-zero groups
    return W.astype(np.float16)


@pytest.mark.parametrize("G", [128, 64, 32])
def test_codes_and_zero_points_in_range(G):
    q, z, s, _ = oracle.quantize(_random_weights(G), G)
    assert q.max() <= 15 and z.max() <= 15
    assert (s.astype(np.float64) > 0).all()


@pytest.mark.parametrize("G", [128, 64, 32])
def test_every_code_is_a_nearest_grid_point(G):
    """Brute force over the 16 codes: (q - z) s is a nearest point of the
    group's grid {(c - z) s : c = 0..15} to v, and exact ties go to even
    q - z (round half to even)."""
    W = _random_weights(G)
    q, z, s, _ = oracle.quantize(W, G)
    N, K = W.shape
    v = W.astype(np.float64)
    zz = np.repeat(z.astype(np.float64), G, axis=1)
    ss = np.repeat(s.astype(np.float64), G, axis=1)
    grid = (np.arange(16)[None, None, :] - zz[..., None]) * ss[..., None]   # exact in fp64
    dist = np.abs(v[..., None] - grid)
    best = dist.min(axis=-1)
    mine = np.take_along_axis(dist, q[..., None].astype(np.int64), axis=-1)[..., 0]
    assert (mine == best).all()
    # exact ties are rare in random data (the golden groups hold constructed
    # ones); where one occurs, q - z must be even
    ties = (dist == best[..., None]).sum(axis=-1) > 1
    d = (q.astype(np.int64) - zz.astype(np.int64))[ties]
    assert (d % 2 == 0).all()


@pytest.mark.parametrize("G", [128, 64, 32])
def test_scale_is_range_over_15_and_zero_point_centres_the_minimum(G):
    W = _random_weights(G)
    q, z, s, _ = oracle.quantize(W, G)
    N, K = W.shape
    v = W.astype(np.float64).reshape(N, K // G, G)
    lo, hi = v.min(-1), v.max(-1)
    R = np.maximum(hi - lo, 1e-5)
    sd = s.astype(np.float64)
    # s is the nearest fp16 of R/15 (numpy's own rounding)
    assert (s.view(np.uint16) == (R / 15.0).astype(np.float16).view(np.uint16)).all()
    # the zero point puts the group minimum within half a step of grid point 0
    free = (z > 0) & (z < 15)
    assert (np.abs(lo + z * sd)[free] <= sd[free] / 2).all()
    # all-positive groups clamp z at 0, all-negative ones at 15
    assert (z[(lo > 0) & (R > 1e-5)] == 0).all()
    assert (z[(hi < 0) & (hi - lo > 15 * sd)] == 15).all()


def _half_ulp(a):
    a = np.abs(a)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return np.exp2(e - 11)


@pytest.mark.parametrize("G", [128, 64, 32])
def test_error_bound_on_non_degenerate_groups(G):
    """|v - W^| <= s/2 + max(0, (hi - lo) - 15 s) + ulp(W^)/2 whenever the zero
    point is not clamped (q cannot clamp at 0 then; at 15 the overshoot of the
    range beyond 15 s is the only extra error)."""
    W = _random_weights(G)
    q, z, s, _ = oracle.quantize(W, G)
    wh = oracle.dequant(q, z, s, G).astype(np.float64)
    N, K = W.shape
    v = W.astype(np.float64)
    g = v.reshape(N, K // G, G)
    R = g.max(-1) - g.min(-1)
    sd = s.astype(np.float64)
    unclamped = np.repeat((z > 0) & (z < 15) & (R >= 1e-5), G, axis=1)
    bound = np.repeat(sd / 2 + np.maximum(0.0, R - 15 * sd), G, axis=1) + _half_ulp(wh)
    bound *= 1 + 1e-12
    err = np.abs(v - wh)
    assert (err[unclamped] <= bound[unclamped]).all()
    # and on the plain N(0, 0.02) rows the error never exceeds ~ one step
    assert (err[48:] <= np.repeat(sd[48:], G, axis=1) * 0.5 + _half_ulp(wh[48:]) + 1e-12).all()


def test_power_of_two_scaling_is_equivariant():
    W = awq_synth.matrix_f16(awq_synth.key(0, 99, "pins/scale"), 32, 4 * G, 0.02)
    q, z, s, _ = oracle.quantize(W, G)
    for j in (1, 3, -2):
        W2 = (W.astype(np.float64) * 2.0 ** j).astype(np.float16)
        q2, z2, s2, _ = oracle.quantize(W2, G)
        assert (q2 == q).all() and (z2 == z).all()
        assert (s2.astype(np.float64) == s.astype(np.float64) * 2.0 ** j).all()


def test_permutation_within_a_group_permutes_codes():
    rng = np.random.default_rng(3)
    W = awq_synth.matrix_f16(awq_synth.key(0, 99, "pins/perm"), 16, 2 * G, 0.02)
    q, z, s, _ = oracle.quantize(W, G)
    perm = np.concatenate([rng.permutation(G), G + rng.permutation(G)])
    q2, z2, s2, _ = oracle.quantize(np.ascontiguousarray(W[:, perm]), G)
    assert (q2 == q[:, perm]).all() and (z2 == z).all() and (s2.view(np.uint16) == s.view(np.uint16)).all()


@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan])
def test_non_finite_weight_is_reported(bad):
    W = awq_synth.matrix_f16(awq_synth.key(0, 99, "pins/nf"), 16, 2 * G, 0.02).copy()
    W[5, 200] = bad
    _, _, _, rc = oracle.quantize(W, G, allow_nonfinite=True)
    assert rc == oracle.ERR_NONFINITE
    with pytest.raises(oracle.OracleError):
        oracle.quantize(W, G)


@pytest.mark.parametrize("N,K", [(16, 100), (15, 128), (0, 128), (16, 192)])
def test_bad_shapes_are_rejected(N, K):
    W = np.zeros((max(N, 1), K), np.float16)
    lib = oracle._load()
    q = np.zeros(W.shape, np.uint8)
    z = np.zeros((max(N, 1), max(K // G, 1)), np.uint8)
    s = np.zeros((max(N, 1), max(K // G, 1)), np.uint16)
    assert lib.orc_quantize(W.ctypes.data, N, K, G, q.ctypes.data, z.ctypes.data, s.ctypes.data) == oracle.ERR_SHAPE
