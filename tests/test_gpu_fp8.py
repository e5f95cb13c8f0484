"""GPU W4A8-FP8 variant against the oracle (the FP8 reading of the TensorRT-LLM
news item on INT4 AWQ on H200).

Bit-exact: the per-row exponents, the per-token E4M3 activation codes and
scales, and the E4M3 weight codes (awq_dequant_fp8, the same device code the
GEMM's dequant warps run). The GEMM's fp16 outputs are within
    |y_gpu - y_ref| <= 2e-3 * B8 + 1e-3,   B8 = sum_k |x8 sx W8 2^-e|
of the fp64 oracle on the same E4M3 operands: the method statement's tolerance
form, applied to the operands this variant multiplies (products of E4M3 values
are exact in fp32; only the fp32 accumulation and the final fp16 rounding
differ from the oracle).
"""
import numpy as np
import pytest
import torch

import awq_synth
import oracle
import weight_only_bit_awq_b200 as awq
from gpu_helpers import check_close, gpu_pack, host, packed_to_host, to_dev

pytestmark = pytest.mark.gpu


def _packed(N, K, tag, std=0.02, group=128):
    W = awq_synth.matrix_f16(awq_synth.key(0, 98, f"{tag}/W"), N, K, std)
    dev = gpu_pack(W, group=group)
    return dev, packed_to_host(*dev)


@pytest.mark.parametrize("group", [128, 64, 32])
def test_row_exponents_and_weight_codes_are_bit_exact(group):
    K, N = 1024, 592
    dev, hp = _packed(N, K, f"w8/{group}", group=group)
    e = awq.awq_fp8_row_exponents(dev[1], K, N, group)
    e_ref = oracle.fp8_row_exponents(hp[1], N, K, group)
    assert (host(e, np.int8) == e_ref).all()
    w8 = awq.awq_dequant_fp8(*dev, e, K, N, group)
    assert (host(w8, np.uint8) == oracle.fp8_weights(*hp, e_ref, N, K, group)).all()


def test_weight_codes_with_extreme_scales():
    # rows whose largest scale makes e negative (big weights) or large (tiny
    # ones, where (q - z) s is an fp16 subnormal)
    K, N = 256, 64
    W = awq_synth.matrix_f16(awq_synth.key(0, 98, "ext/W"), N, K, 1.0).astype(np.float64)
    W[:16] *= 300.0
    W[16:32] *= 1e-5
    W[32:48, :128] *= 1e-6
    W = W.astype(np.float16)
    dev = gpu_pack(W)
    hp = packed_to_host(*dev)
    e = awq.awq_fp8_row_exponents(dev[1], K, N, 128)
    e_ref = oracle.fp8_row_exponents(hp[1], N, K)
    assert (host(e, np.int8) == e_ref).all()
    assert e_ref.min() < 0 and e_ref.max() > 20
    w8 = awq.awq_dequant_fp8(*dev, e, K, N, 128)
    assert (host(w8, np.uint8) == oracle.fp8_weights(*hp, e_ref, N, K)).all()


def _edge_x(M, K, seed):
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, f"x/{seed}/{M}x{K}"), M, K, 1.0).astype(np.float64)
    if M > 1:
        x[1] = 0.0                                   # sx = 0
    if M > 2:
        x[2] *= 2.0 ** -16                           # fp16 subnormals
    if M > 3:
        x[3, 5] = -60000.0                           # one huge value
    if M > 4:
        x[4, :] = np.where(np.arange(K) % 2, 448.0, -448.0)   # ties of x / sx at the top
    return x.astype(np.float16)


@pytest.mark.parametrize("M,K", [(1, 128), (5, 4096), (37, 11008), (300, 1024)])
def test_activation_codes_and_scales_are_bit_exact(M, K):
    x = _edge_x(M, K, 1)
    x8, sx = awq.awq_fp8_quantize_x(to_dev(x.view(np.uint16), torch.float16))
    x8_ref, sx_ref = oracle.fp8_quantize_x(x)
    assert (host(x8, np.uint8) == x8_ref).all()
    assert np.array_equal(host(sx, np.uint32), sx_ref.view(np.uint32))


def _gemm(x, dev, N, group=128):
    M, K = x.shape
    x8, sx = awq.awq_fp8_quantize_x(to_dev(x.view(np.uint16), torch.float16))
    e = awq.awq_fp8_row_exponents(dev[1], K, N, group)
    ws = awq.new_workspace(0, K, N, x8.device, group)
    y = awq.awq_w4a8_gemm(x8, sx, *dev, e, N, ws, group)
    st = awq.awq_get_status(ws)
    assert st == awq.AWQ_OK, awq.awq_status_string(st)
    return host(y, np.float16), host(x8, np.uint8), host(sx, np.float32), host(e, np.int8)


SHAPES = [(128, 16), (256, 48), (384, 336), (1024, 592), (2048, 4096), (4096, 272), (11008, 160)]


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("M", [1, 7, 128, 129, 257, 513])
def test_w4a8_gemm_matches_oracle(K, N, M):
    dev, hp = _packed(N, K, f"g{K}x{N}")
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, f"g{K}x{N}/x{M}"), M, K, 1.0)
    y, x8, sx, e = _gemm(x, dev, N)
    if M * N * K <= 2e8:
        y_ref, b = oracle.fp8_linear(x8, sx, *hp, e, N, K)
        check_close(y, y_ref, b, f"w4a8 M={M} K={K} N={N}")
    else:
        rows = np.unique(np.concatenate([np.arange(16), np.arange(N - 16, N),
                                         np.random.default_rng(M).choice(N, 48, replace=False)]))
        y_ref, b = _rows(x8, sx, hp, e, N, K, rows)
        check_close(y[:, rows], y_ref, b, f"w4a8 M={M} K={K} N={N}")


def _rows(x8, sx, hp, e, N, K, rows):
    ys, bs = [], []
    for n in rows:
        y1, b1 = oracle.fp8_linear(x8, sx, *hp, e, N, K, rows=(int(n), int(n) + 1))
        ys.append(y1)
        bs.append(b1)
    return np.concatenate(ys, 1), np.concatenate(bs, 1)


@pytest.mark.parametrize("group", [64, 32])
def test_w4a8_gemm_group_sizes(group):
    K, N, M = 1024, 592, 200
    dev, hp = _packed(N, K, f"gg{group}", group=group)
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, f"gg{group}/x"), M, K, 1.0)
    y, x8, sx, e = _gemm(x, dev, N, group)
    y_ref, b = oracle.fp8_linear(x8, sx, *hp, e, N, K, group)
    check_close(y, y_ref, b, f"w4a8 group {group}")


def test_w4a8_gemm_with_edge_activations_and_extreme_rows():
    K, N, M = 1024, 336, 9
    W = awq_synth.matrix_f16(awq_synth.key(0, 98, "edge/W"), N, K, 0.02).astype(np.float64)
    W[:16] *= 2000.0
    W[16:32] *= 1e-4
    dev = gpu_pack(W.astype(np.float16))
    hp = packed_to_host(*dev)
    x = _edge_x(M, K, 2)
    y, x8, sx, e = _gemm(x, dev, N)
    y_ref, b = oracle.fp8_linear(x8, sx, *hp, e, N, K)
    # outputs beyond the fp16 range (the -60000 input times the x2000 rows)
    # must be infinities of the right sign; the rest within tolerance
    over = np.abs(y_ref) >= 65520.0
    assert over.any() and (~over).sum() > 0.9 * over.size
    assert np.isinf(y[over]).all() and (np.sign(y[over]) == np.sign(y_ref[over])).all()
    check_close(np.where(over, 0, y), np.where(over, 0, y_ref), np.where(over, 0, b), "w4a8 edge")
    assert (y[1] == 0).all()                         # a zero row of x gives zero outputs


def test_w4a8_stays_within_the_quantization_bound_of_w4a16():
    # the closed-form bound the oracle is pinned to, on the GPU outputs of both paths
    K, N, M = 2048, 256, 64
    dev, hp = _packed(N, K, "bound")
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, "bound/x"), M, K, 1.0)
    y8, x8, sx, e = _gemm(x, dev, N)
    ws = awq.new_workspace(M, K, N, "cuda")
    y16 = host(awq.awq_w4a16_gemm(to_dev(x.view(np.uint16), torch.float16), *dev, N, ws), np.float16)
    _, b = oracle.linear(x, *hp, N, K)
    err = np.abs(y8.astype(np.float64) - y16.astype(np.float64))
    assert (err <= 2.0 ** -3 * b * 1.05 + 2e-3).all()


PREFILL = [(l.name, M) for l in awq_synth.WORKLOADS["prefill"].layers for M in (512, 2048)]


@pytest.mark.parametrize("layer,M", PREFILL)
def test_w4a8_prefill_full_size_sampled(layer, M):
    wl = awq_synth.WORKLOADS["prefill"]
    L = wl.layer(layer)
    W = awq_synth.layer_weight(0, wl, L)
    dev = gpu_pack(W)
    hp = packed_to_host(*dev)
    x = awq_synth.layer_input(0, wl, L, M)
    y, x8, sx, e = _gemm(x, dev, L.N)
    rng = np.random.default_rng(M)
    ms = np.concatenate([rng.integers(0, M, 2048), [0, M - 1, 0, M - 1]])
    ns = np.concatenate([rng.integers(0, L.N, 2048), [0, 0, L.N - 1, L.N - 1]])
    order = np.argsort(ns, kind="stable")
    y_ref, b = oracle.fp8_linear_entries(x8, sx, *hp, e, L.N, L.K, ms[order], ns[order])
    check_close(y[ms[order], ns[order]], y_ref, b, f"w4a8 prefill/{layer} M={M}")
