"""Pins of the oracle's W4A8-FP8 functions against things other than itself.

- E4M3 decoding: all 256 codes against torch's float8_e4m3fn.
- E4M3 rounding: every finite value round-trips; every midpoint between
  neighbours goes to the even code (hand-derived rule); 200k random doubles
  within the finite range against torch's cast (which rounds to nearest, ties
  to even); saturation and NaN by hand.
- Per-token activation quantization: the largest |x| lands on +-448, the
  relative error of every element is within the E4M3 half-spacing, a row
  scaled by a power of two gives the same codes, and a zero row gives sx = 0.
- Row exponents: hand-derived cases at the 448 boundary.
- The layer: against the W4A16 oracle within the closed-form bound of the two
  quantizations, against numpy's fp64 matmul of torch-decoded operands, and
  one-hot activations.
"""
import numpy as np
import pytest
import torch

import awq_synth
import oracle


def _torch_e4m3(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _decode(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = _decode(codes)
    mine = np.array([oracle.e4m3_to_double(int(c)) for c in codes])
    assert np.all((ref == mine) | (np.isnan(ref) & np.isnan(mine)))
    assert oracle.e4m3_to_double(0x7E) == 448.0 and oracle.e4m3_to_double(0x01) == 2.0 ** -9


def test_e4m3_round_trip_and_ties_to_even():
    finite = [c for c in range(128) if c != 0x7F]
    vals = [oracle.e4m3_to_double(c) for c in finite]
    for c, v in zip(finite, vals):
        assert oracle.double_to_e4m3(v) == c
        assert oracle.double_to_e4m3(-v) == (c | 0x80 if c else 0x80)
    # the midpoint of neighbours c, c+1 rounds to the one with an even fraction
    for c in range(0x7D + 1):
        lo, hi = oracle.e4m3_to_double(c), oracle.e4m3_to_double(c + 1)
        mid = (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        assert oracle.double_to_e4m3(mid) == even, hex(c)
        assert oracle.double_to_e4m3(np.nextafter(mid, 0)) == c
        assert oracle.double_to_e4m3(np.nextafter(mid, 1e9)) == c + 1


def test_e4m3_rounding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-448, 448, 100000), 2.0 ** rng.uniform(-12, 8.8, 100000) *
                        np.sign(rng.standard_normal(100000))]).astype(np.float32)
    v = v[np.abs(v) < 448]
    mine = np.array([oracle.double_to_e4m3(float(a)) for a in v], np.uint8)
    assert (mine == _torch_e4m3(v)).all()


def test_e4m3_saturation_and_nan():
    for d in (448.0, 448.5, 464.0, 479.9, 480.0, 1e30, float("inf")):
        assert oracle.double_to_e4m3(d) == 0x7E
        assert oracle.double_to_e4m3(-d) == 0xFE
    assert oracle.double_to_e4m3(float("nan")) == 0x7F
    assert oracle.double_to_e4m3(2.0 ** -11) == 0x00       # below half the smallest subnormal
    assert oracle.double_to_e4m3(2.0 ** -10) == 0x00       # exact tie with 0 and 2^-9: even is 0
    assert oracle.double_to_e4m3(1.5 * 2.0 ** -10) == 0x01


def _x(M, K, seed=1, scale=1.0):
    return awq_synth.matrix_f16(awq_synth.key(0, 97, f"fp8x/{seed}"), M, K, scale)


def test_quantize_x_properties():
    x = _x(7, 512)
    x[3] = 0
    x[5, 17] = np.float16(-300.0)
    x8, sx = oracle.fp8_quantize_x(x)
    xd = x.astype(np.float64)
    assert sx[3] == 0 and (x8[3] == 0).all()
    for m in (0, 1, 2, 4, 5, 6):
        amax = np.abs(xd[m]).max()
        assert sx[m] == np.float32(np.float32(amax) / np.float32(448.0))
        k = int(np.abs(xd[m]).argmax())
        assert x8[m, k] & 0x7F == 0x7E                     # the largest |x| maps to +-448
        deq = _decode(x8[m]) * float(sx[m])
        # half the E4M3 spacing: 2^-4 relative for normal codes, 2^-10 sx below 2^-6
        bound = np.maximum(np.abs(xd[m]) * 2.0 ** -4, float(sx[m]) * 2.0 ** -10) * (1 + 2.0 ** -20)
        assert (np.abs(deq - xd[m]) <= bound).all()
    # every code, element by element, is torch's E4M3 rounding of the IEEE fp32
    # quotient x / sx (torch's float32 division and float8_e4m3fn cast, run
    # here as a library reference); rows with sx == 0 are all-zero codes
    live = sx > 0
    q_t = (torch.from_numpy(x[live].astype(np.float32)) / torch.from_numpy(sx[live])[:, None]).to(torch.float8_e4m3fn)
    assert np.array_equal(q_t.view(torch.uint8).numpy(), x8[live])
    # on 64 x 4096 activations, where a reciprocal-multiply stand-in for the
    # division already changes a few codes
    xb = _x(64, 4096)
    x8b, sxb = oracle.fp8_quantize_x(xb)
    q_b = (torch.from_numpy(xb.astype(np.float32)) / torch.from_numpy(sxb)[:, None]).to(torch.float8_e4m3fn)
    assert np.array_equal(q_b.view(torch.uint8).numpy(), x8b)
    # power-of-two scaling of a row changes sx by that power and no code
    x2 = (x.astype(np.float32) * 4.0).astype(np.float16)
    x8b, sxb = oracle.fp8_quantize_x(x2)
    assert (x8b == x8).all() and np.array_equal(sxb, sx * 4)


def test_row_exponents_at_the_boundary():
    # scales fp16 [K/G][N] with K/G = 2; row n's largest scale decides
    S = np.ones((2, 16), np.float16)   # rows 6..15: largest scale 1 -> e = 4
    S[:, :6] = [[1.0, 29.859375, 29.875, 0.25, 2.0 ** -20, 1000.0],
                [0.5, 1.0, 1.0, 0.0625, 2.0 ** -24, 7.0]]
    e = oracle.fp8_row_exponents(S, 16, 256)
    # 15*1*16 = 240 <= 448 < 480; 15*29.859375 = 447.9; 15*29.875 = 448.1 -> halve;
    # 15*0.25*64 = 240; 15*2^-20*2^24 = 240; 15*1000*2^-6 = 234.4 <= 448 < 468.75
    assert e.tolist() == [4, 0, -1, 6, 24, -6] + [4] * 10


def _layer(N, K, tag):
    W = awq_synth.matrix_f16(awq_synth.key(0, 97, f"fp8W/{tag}"), N, K, 0.02)
    return oracle.quantize_pack(W)


def test_layer_against_w4a16_within_the_quantization_bound():
    N, K, M = 48, 384, 5
    qw, sc, ze = _layer(N, K, "a")
    x = _x(M, K, seed=2)
    x8, sx = oracle.fp8_quantize_x(x)
    e = oracle.fp8_row_exponents(sc, N, K)
    y8, _ = oracle.fp8_linear(x8, sx, qw, sc, ze, e, N, K)
    y16, _ = oracle.linear(x, qw, sc, ze, N, K)
    q, z, s = oracle.unpack(qw, sc, ze, N, K)
    wh = np.abs(oracle.dequant(q, z, s).astype(np.float64))
    xa = np.abs(x.astype(np.float64))
    # |x8 sx - x| <= 2^-4 |x| + 2^-10 sx, |W8 2^-e - W^| <= 2^-4 |W^| + 2^-10 2^-e
    ex = xa * 2.0 ** -4 + sx[:, None].astype(np.float64) * 2.0 ** -10
    ew = wh * 2.0 ** -4 + (2.0 ** -10) * (2.0 ** -e.astype(np.float64))[:, None]
    bound = ex @ wh.T + xa @ ew.T + ex @ ew.T
    assert (np.abs(y8 - y16) <= bound * (1 + 1e-9)).all()
    assert np.abs(y8 - y16).max() > 0                       # it is a real quantization


def test_layer_against_numpy_matmul_of_torch_decoded_operands():
    N, K, M = 32, 256, 3
    qw, sc, ze = _layer(N, K, "b")
    x = _x(M, K, seed=3)
    x8, sx = oracle.fp8_quantize_x(x)
    e = oracle.fp8_row_exponents(sc, N, K)
    w8 = oracle.fp8_weights(qw, sc, ze, e, N, K)
    xv = _decode(x8) * sx[:, None].astype(np.float64)
    wv = _decode(w8) * (2.0 ** -e.astype(np.float64))[:, None]
    y, b = oracle.fp8_linear(x8, sx, qw, sc, ze, e, N, K)
    assert np.allclose(y, xv @ wv.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(b, np.abs(xv) @ np.abs(wv).T, rtol=1e-12)
    ye, be = oracle.fp8_linear_entries(x8, sx, qw, sc, ze, e, N, K, [0, 2, 1], [5, 31, 0])
    assert np.array_equal(ye, y[[0, 2, 1], [5, 31, 0]])


def test_weights_are_the_rounded_scaled_dequant_and_one_hot_reads_them():
    N, K = 32, 256
    qw, sc, ze = _layer(N, K, "c")
    e = oracle.fp8_row_exponents(sc, N, K)
    w8 = oracle.fp8_weights(qw, sc, ze, e, N, K)
    q, z, s = oracle.unpack(qw, sc, ze, N, K)
    wh = oracle.dequant(q, z, s).astype(np.float64)
    scaled = wh * (2.0 ** e.astype(np.float64))[:, None]
    assert np.abs(scaled).max() <= 448
    # where W^ is an fp16 normal number (here: all nonzero weights), W8 is
    # torch's E4M3 rounding of W^ 2^e
    assert (np.abs(wh[wh != 0]) >= 2.0 ** -14).all()
    assert (w8 == _torch_e4m3(scaled)).all()
    x = np.zeros((2, K), np.float16)
    x[0, 7], x[1, 200] = 448.0, -896.0     # sx = 1 and 2 exactly, x8 = +-448
    x8, sx = oracle.fp8_quantize_x(x)
    assert sx.tolist() == [1.0, 2.0]
    y, _ = oracle.fp8_linear(x8, sx, qw, sc, ze, e, N, K)
    assert np.array_equal(y[0], 448.0 * _decode(w8[:, 7]) * 2.0 ** -e.astype(np.float64))
    assert np.array_equal(y[1], -896.0 * _decode(w8[:, 200]) * 2.0 ** -e.astype(np.float64))


def test_weights_of_groups_with_fp16_subnormal_dequant_values():
    # scales below 2^-14 / 15 make W^ an fp16 subnormal; the scale is moved by
    # 2^e before the product is rounded, so W8 keeps full precision there
    N, K = 16, 256
    q = np.random.default_rng(5).integers(0, 16, (N, K)).astype(np.uint8)
    z = np.full((N, K // 128), 7, np.uint8)
    s = np.full((N, K // 128), 2.0 ** -20 * 1.3, np.float16)
    s[:, 1] = np.float16(2.0 ** -21 * 1.7)
    qw, sc, ze = oracle.pack(q, z, s)
    e = oracle.fp8_row_exponents(sc, N, K)
    w8 = oracle.fp8_weights(qw, sc, ze, e, N, K)
    for n in range(N):
        for k in (0, 5, 127, 128, 200, 255):
            g = k // 128
            s2 = np.float64(np.float16(np.float64(s[n, g]) * 2.0 ** int(e[n])))
            v = np.float64(np.float16((int(q[n, k]) - int(z[n, g])) * s2))
            assert w8[n, k] == _torch_e4m3(np.array([v]))[0]
