"""GPU W4A16 GEMV / GEMM / linear against the fp64 oracle, element by element
within |y - y_ref| <= 2e-3 * sum|x w| + 1e-3, on the same seeded inputs."""
import numpy as np
import pytest
import torch

import awq_synth
import oracle
import weight_only_bit_awq_b200 as awq
from gpu_helpers import (check_close, gpu_pack, host, layer_inputs, oracle_rows, packed_to_host, sample_rows,
                         to_dev)

pytestmark = pytest.mark.gpu
G = 128


def _packed(N, K, tag, std=0.02, group=G):
    W = awq_synth.matrix_f16(awq_synth.key(0, 96, f"{tag}/W"), N, K, std)
    dev = gpu_pack(W, group=group)
    return W, dev, packed_to_host(*dev)


def _run(fn, x, dev, N, M=None, group=G):
    xd = to_dev(x.view(np.uint16), torch.float16)
    M = x.shape[0]
    K = x.shape[1]
    ws = awq.new_workspace(M, K, N, xd.device, group)
    y = fn(xd, *dev, N, ws, group)
    st = awq.awq_get_status(ws)
    assert st == awq.AWQ_OK, awq.awq_status_string(st)
    return host(y, np.float16)


def _check_against_oracle(y, x, hp, N, K, what, group=G):
    """Every output when the oracle's work is small, else all tokens on
    sampled output channels (first and last row block plus random rows)."""
    M = x.shape[0]
    if M * N * K <= 2e8:
        y_ref, b = oracle.linear(x, *hp, N, K, group)
        return check_close(y, y_ref, b, what)
    rows = sample_rows(N, 64, seed=M)
    y_ref, b = oracle_rows(x, *hp, N, K, rows, group)
    return check_close(y[:, rows], y_ref, b, what)


# small and ragged shapes: several row blocks and k-blocks, N not a multiple
# of the 128-row GEMM tile, single-k-block K, split-K on and off
SHAPES = [(128, 16), (256, 48), (384, 336), (1024, 592), (2048, 4096), (4096, 272), (11008, 160)]


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 16, 17, 31, 32])
def test_gemv_matches_oracle(K, N, M):
    W, dev, hp = _packed(N, K, f"gemv{K}x{N}")
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"gemv{K}x{N}/x{M}"), M, K, 1.0)
    y = _run(awq.awq_w4a16_gemv, x, dev, N)
    _check_against_oracle(y, x, hp, N, K, f"gemv M={M} K={K} N={N}")


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("M", [1, 7, 64, 128, 129, 200, 256, 257, 513])
def test_gemm_matches_oracle(K, N, M):
    W, dev, hp = _packed(N, K, f"gemm{K}x{N}")
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"gemm{K}x{N}/x{M}"), M, K, 1.0)
    y = _run(awq.awq_w4a16_gemm, x, dev, N)
    _check_against_oracle(y, x, hp, N, K, f"gemm M={M} K={K} N={N}")


@pytest.mark.parametrize("fn", [awq.awq_w4a16_gemv, awq.awq_w4a16_gemm])
def test_one_hot_activations_give_the_dequantized_weight_exactly(fn):
    K, N = 512, 336
    W, dev, hp = _packed(N, K, "onehot")
    ks = [0, 1, 7, 127, 128, 300, 511, 64]
    x = np.zeros((len(ks), K), np.float16)
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    y = _run(fn, x, dev, N)
    q, z, s = oracle.unpack(*hp, N, K)
    wh = oracle.dequant(q, z, s)
    for m, k in enumerate(ks):
        assert (y[m].view(np.uint16) == wh[:, k].view(np.uint16)).all(), (fn.__name__, k)


def test_linear_dispatch_and_empty_batch():
    K, N = 1024, 256
    W, dev, hp = _packed(N, K, "disp")
    lim = awq.awq_linear_gemv_limit()
    for M in (1, lim, lim + 1, 300):
        x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"disp/x{M}"), M, K, 1.0)
        y = _run(awq.awq_linear, x, dev, N)
        y_ref, b = oracle.linear(x, *hp, N, K)
        check_close(y, y_ref, b, f"linear M={M}")
    x0 = torch.empty((0, K), dtype=torch.float16, device="cuda")
    ws = awq.new_workspace(0, K, N, x0.device)
    for fn in (awq.awq_linear, awq.awq_w4a16_gemv, awq.awq_w4a16_gemm):
        assert fn(x0, *dev, N, ws).shape == (0, N)


def test_split_k_is_deterministic_and_the_workspace_reusable():
    K, N = 11008, 4096
    W, dev, hp = _packed(N, K, "det")
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, "det/x"), 3, K, 1.0)
    xd = to_dev(x.view(np.uint16), torch.float16)
    ws = awq.new_workspace(3, K, N, xd.device)
    ys = [host(awq.awq_w4a16_gemv(xd, *dev, N, ws), np.uint16) for _ in range(3)]
    assert (ys[0] == ys[1]).all() and (ys[1] == ys[2]).all()
    assert awq.awq_get_status(ws) == awq.AWQ_OK


def test_one_workspace_serves_gemv_and_stream_k_gemm_calls_of_any_size():
    # Partial sums and stream-K parts are written before they are read, so a
    # workspace sized for the largest call serves calls of every size and
    # either kernel, in any order.
    cases = [(1, 4096, 4096), (40, 1024, 38400), (3, 11008, 4096), (40, 24576, 1024), (8, 1024, 25600),
             (1, 4096, 4096)]
    nbytes = max(awq.awq_workspace_bytes(M, K, N) for M, K, N in cases)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    for M, K, N in cases:
        W, dev, hp = _packed(N, K, f"share{K}x{N}")
        x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"share{K}x{N}/x{M}"), M, K, 1.0)
        xd = to_dev(x.view(np.uint16), torch.float16)
        fn = awq.awq_w4a16_gemv if M <= 16 else awq.awq_w4a16_gemm
        y = host(fn(xd, *dev, N, ws), np.float16)
        assert awq.awq_get_status(ws) == awq.AWQ_OK
        _check_against_oracle(y, x, hp, N, K, f"shared workspace {fn.__name__} M={M} K={K} N={N}")


def test_gemv_and_gemm_agree_closely():
    K, N, M = 4096, 1024, 16
    W, dev, hp = _packed(N, K, "agree")
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, "agree/x"), M, K, 1.0)
    y1 = _run(awq.awq_w4a16_gemv, x, dev, N).astype(np.float64)
    y2 = _run(awq.awq_w4a16_gemm, x, dev, N).astype(np.float64)
    y_ref, b = oracle.linear(x, *hp, N, K)
    check_close(y1, y_ref, b)
    check_close(y2, y_ref, b)


# ---- prefill GEMM with the stream-K schedule --------------------------------
# When whole 128-channel x BN-token tiles would leave the last wave of SMs
# short, the k-blocks of the last tiles are split evenly between the CTAs and
# a fixup kernel adds the fp32 parts in CTA order. Shapes (M, K, N, group):
# every tile split many ways (8 tiles on all SMs); whole data-parallel tiles
# followed by split ones; 256-token tiles with a ragged last token tile
# (M = 300, 513); groups of 64 and 32.
STREAM_K_CASES = [(40, 24576, 1024, 128), (40, 1024, 38400, 128), (300, 1024, 9600, 128), (513, 2048, 6400, 128),
                  (40, 2048, 19200, 64), (40, 2048, 19200, 32)]


@pytest.mark.parametrize("M,K,N,group", STREAM_K_CASES)
def test_gemm_stream_k_matches_oracle(M, K, N, group):
    assert awq.awq_linear_launches(M, K, N, group) == 2  # the schedule is stream-K here
    W, dev, hp = _packed(N, K, f"sk{K}x{N}", group=group)
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"sk{K}x{N}/x{M}"), M, K, 1.0)
    xd = to_dev(x.view(np.uint16), torch.float16)
    ws = awq.new_workspace(M, K, N, xd.device, group)
    ys = [host(awq.awq_w4a16_gemm(xd, *dev, N, ws, group), np.float16) for _ in range(2)]
    st = awq.awq_get_status(ws)
    assert st == awq.AWQ_OK, awq.awq_status_string(st)
    assert (ys[0].view(np.uint16) == ys[1].view(np.uint16)).all()  # deterministic
    # all tokens on rows of every 128-channel tile (its first and last row and
    # random ones), about 8e7 oracle multiply-adds
    rng = np.random.default_rng(M + N)
    per_tile = max(2, int(8e7 / (M * K * ((N + 127) // 128))))
    rows = set()
    for n0 in range(0, N, 128):
        hi = min(N, n0 + 128)
        rows |= {n0, hi - 1} | set(rng.integers(n0, hi, per_tile - 2).tolist())
    rows = np.array(sorted(rows), dtype=np.int64)
    y_ref, b = oracle_rows(x, *hp, N, K, rows, group)
    check_close(ys[0][:, rows], y_ref, b, f"stream-K gemm M={M} K={K} N={N} g={group}")


def test_gemm_stream_k_one_hot_gives_the_dequantized_weight_exactly():
    # one nonzero input per token: each output is one dequantized weight, and
    # the fp32 parts of the split tiles (all but one exactly zero) add up to it
    M, K, N = 40, 24576, 1024
    W, dev, hp = _packed(N, K, "sk_onehot")
    q, z, s = oracle.unpack(*hp, N, K)
    wh = oracle.dequant(q, z, s)
    ks = np.random.default_rng(7).integers(0, K, M)
    x = np.zeros((M, K), np.float16)
    x[np.arange(M), ks] = 1.0
    y = _run(awq.awq_w4a16_gemm, x, dev, N)
    assert (y.view(np.uint16) == wh[:, ks].T.view(np.uint16)).all()


# ---- full-size workloads, sampled against the oracle ----------------------

DECODE_CASES = [("single_4096", "linear", 1)]
DECODE_CASES += [("llama2_7b_decode", l.name, 1) for l in awq_synth.WORKLOADS["llama2_7b_decode"].layers]
DECODE_CASES += [("llama3_8b_decode", l.name, M) for l in awq_synth.WORKLOADS["llama3_8b_decode"].layers
                 for M in (1, 4, 8, 16, 32)]
DECODE_CASES += [("llama2_70b_decode", l.name, M) for l in awq_synth.WORKLOADS["llama2_70b_decode"].layers
                 for M in (1, 8, 32)]


_cache = {}


def _full_layer(wl, layer):
    key = (wl, layer)
    if key not in _cache:
        _cache.clear()
        w = awq_synth.WORKLOADS[wl]
        L = w.layer(layer)
        W = awq_synth.layer_weight(0, w, L)
        dev = gpu_pack(W)
        _cache[key] = (L, dev, packed_to_host(*dev))
    return _cache[key]


@pytest.mark.parametrize("wl,layer,M", DECODE_CASES)
def test_decode_full_size(wl, layer, M):
    L, dev, hp = _full_layer(wl, layer)
    x = awq_synth.layer_input(0, awq_synth.WORKLOADS[wl], L, M)
    y = _run(awq.awq_linear, x, dev, L.N)
    rows = sample_rows(L.N, 96, seed=M)
    y_ref, b = oracle_rows(x, *hp, L.N, L.K, rows)
    check_close(y[:, rows], y_ref, b, f"{wl}/{layer} M={M}")


# Shapes whose streamed GEMV unit spans several k-blocks: 4 k-blocks with
# K/128 = 122 (the last unit of each group has 2) and a last group of 3 row
# blocks; K/128 = 149 with 4 k-blocks (M <= 3; the last unit has 1) and with
# 2 k-blocks (M = 8 and 16, where bigger units leave too few ring stages);
# 4 k-blocks with only 6 k-blocks per group. The checked rows include every
# row of the first two and the last two groups, where CTA ranges split groups.
UNIT_CASES = [(15616, 5168, 1), (15616, 5168, 24), (19072, 2048, 1), (19072, 2048, 3), (19072, 2048, 8),
              (19072, 2048, 16), (768, 75776, 1)]


@pytest.mark.parametrize("K,N,M", UNIT_CASES)
def test_gemv_multi_kblock_units(K, N, M):
    W, dev, hp = _packed(N, K, f"unit{K}x{N}")
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"unit{K}x{N}/x{M}"), M, K, 1.0)
    y = _run(awq.awq_w4a16_gemv, x, dev, N)
    rows = set(sample_rows(N, 64, seed=M).tolist()) | set(range(min(256, N))) | set(range(max(0, N - 256), N))
    rows = np.array(sorted(rows), dtype=np.int64)
    y_ref, b = oracle_rows(x, *hp, N, K, rows)
    check_close(y[:, rows], y_ref, b, f"unit K={K} N={N} M={M}")


# Group sizes 64 and 32 (TinyChat README, Usage step 3: Falcon-7B is quantized
# with groups of 64). Small shapes (one-k-block units), a ragged one, and a
# decode-sized layer whose units span 4 k-blocks, for the GEMV (M = 1, 5, 8,
# 16, 32) and the GEMM.
GROUP_SHAPES = [(256, 48), (1024, 592), (4096, 4096)]


@pytest.mark.parametrize("group", [64, 32])
@pytest.mark.parametrize("K,N", GROUP_SHAPES)
@pytest.mark.parametrize("M", [1, 5, 8, 16, 32])
def test_gemv_group_sizes(group, K, N, M):
    W, dev, hp = _packed(N, K, f"g{group}/{K}x{N}", group=group)
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"g{group}/{K}x{N}/x{M}"), M, K, 1.0)
    y = _run(awq.awq_w4a16_gemv, x, dev, N, group=group)
    _check_against_oracle(y, x, hp, N, K, f"gemv g={group} M={M} K={K} N={N}", group)


@pytest.mark.parametrize("group", [64, 32])
@pytest.mark.parametrize("K,N", GROUP_SHAPES)
@pytest.mark.parametrize("M", [7, 200, 513])
def test_gemm_group_sizes(group, K, N, M):
    W, dev, hp = _packed(N, K, f"g{group}/{K}x{N}", group=group)
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"g{group}m/{K}x{N}/x{M}"), M, K, 1.0)
    y = _run(awq.awq_w4a16_gemm, x, dev, N, group=group)
    _check_against_oracle(y, x, hp, N, K, f"gemm g={group} M={M} K={K} N={N}", group)


@pytest.mark.parametrize("group", [64, 32])
def test_group_sizes_multi_kblock_units(group):
    K, N, M = 15616, 5168, 1   # 4 k-blocks per unit, K/128 = 122 (ragged), last group of 3 row blocks
    W, dev, hp = _packed(N, K, f"g{group}unit", group=group)
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"g{group}unit/x"), M, K, 1.0)
    y = _run(awq.awq_w4a16_gemv, x, dev, N, group=group)
    rows = set(sample_rows(N, 64, seed=3).tolist()) | set(range(256)) | set(range(N - 256, N))
    rows = np.array(sorted(rows), dtype=np.int64)
    y_ref, b = oracle_rows(x, *hp, N, K, rows, group)
    check_close(y[:, rows], y_ref, b, f"unit g={group}")


PREFILL_CASES = [(l.name, M) for l in awq_synth.WORKLOADS["prefill"].layers for M in (512, 2048, 8192)]


@pytest.mark.parametrize("layer,M", PREFILL_CASES)
def test_prefill_full_size(layer, M):
    """4096 random outputs, the corners of the first and last output tiles,
    one row of y (every (N/2048)-th output channel) and one full column,
    against the oracle computed one by one."""
    L, dev, hp = _full_layer("prefill", layer)
    x = awq_synth.layer_input(0, awq_synth.WORKLOADS["prefill"], L, M)
    y = _run(awq.awq_linear, x, dev, L.N)
    rng = np.random.default_rng(M)
    ms = [rng.integers(0, M, 4096)]
    ns = [rng.integers(0, L.N, 4096)]
    for m0, n0 in ((0, 0), (M - 1, L.N - 1)):        # first / last 128 x 128 corner tiles, 8x8 subsampled
        mm = np.arange(max(0, m0 - 127), min(M, m0 + 128))[::16]
        nn = np.arange(max(0, n0 - 127), min(L.N, n0 + 128))[::16]
        ms.append(np.repeat(mm, len(nn)))
        ns.append(np.tile(nn, len(mm)))
    mr = rng.integers(0, M)
    row_ns = np.arange(0, L.N, max(1, L.N // 2048))
    ms.append(np.full(len(row_ns), mr)), ns.append(row_ns)                  # a row of y, strided
    nc = rng.integers(0, L.N)
    ms.append(np.arange(M)), ns.append(np.full(M, nc))                     # a full column of y
    ms, ns = np.concatenate(ms), np.concatenate(ns)
    order = np.argsort(ns, kind="stable")
    y_ref, b = oracle.linear_entries(x, *hp, L.N, L.K, ms[order], ns[order])
    check_close(y[ms[order], ns[order]], y_ref, b, f"prefill/{layer} M={M}")


# ---- decode at M <= 2, groups of 128: x as a block fixed-point integer -----
# Each 128-input block of x is scaled by a power of two fixed by its largest
# value and rounded to an integer below 2^30; these cases stress that step.

@pytest.mark.parametrize("M", [1, 2])
def test_decode_one_hot_gives_the_dequantized_weight_exactly(M):
    K, N = 1024, 336
    W, dev, hp = _packed(N, K, "onehot12")
    q, z, s = oracle.unpack(*hp, N, K)
    wh = oracle.dequant(q, z, s)
    for ks in ([0, 1], [127, 128], [300, 1023], [64, 65]):
        x = np.zeros((M, K), np.float16)
        for m in range(M):
            x[m, ks[m]] = 1.0
        y = _run(awq.awq_w4a16_gemv, x, dev, N)
        for m in range(M):
            assert (y[m].view(np.uint16) == wh[:, ks[m]].view(np.uint16)).all(), (M, ks[m])


def _edge_x(kind, M, K, rng):
    x = rng.standard_normal((M, K))
    if kind == "outlier":      # one value per block 2^16 times the rest
        x *= 1e-3
        x[:, ::128] = 65.0 * np.sign(rng.standard_normal((M, K // 128)))
    elif kind == "subnormal":  # only fp16 subnormals
        x = rng.integers(-1023, 1024, (M, K)) * 2.0 ** -24
    elif kind == "mixed_zero":  # whole zero blocks between normal ones
        x[:, 128:384] = 0.0
    elif kind == "wide":       # magnitudes from 2^-14 to 2^4 in every block (y stays finite)
        x = np.sign(x) * 2.0 ** rng.uniform(-14, 4, (M, K))
    return x.astype(np.float16)


@pytest.mark.parametrize("kind", ["outlier", "subnormal", "mixed_zero", "wide"])
@pytest.mark.parametrize("M", [1, 2])
def test_decode_block_fixed_point_edge_cases(kind, M):
    K, N = 2048, 592
    W, dev, hp = _packed(N, K, "edge")
    x = _edge_x(kind, M, K, np.random.default_rng(M))
    y = _run(awq.awq_w4a16_gemv, x, dev, N)
    y_ref, b = oracle.linear(x, *hp, N, K)
    check_close(y, y_ref, b, f"{kind} M={M}")


def test_decode_zero_activations_give_zero():
    K, N = 2048, 592
    W, dev, hp = _packed(N, K, "edge")
    for M in (1, 2, 5):
        y = _run(awq.awq_w4a16_gemv, np.zeros((M, K), np.float16), dev, N)
        assert (y.view(np.uint16) & 0x7FFF == 0).all()


@pytest.mark.parametrize("M", [1, 2, 5])
@pytest.mark.parametrize("bad", [np.inf, np.nan])
def test_decode_non_finite_activation_gives_non_finite_outputs(M, bad):
    K, N = 1024, 336
    W, dev, hp = _packed(N, K, "nonfin")
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, "nonfin/x"), M, K, 1.0)
    x[M - 1, 200] = bad
    y = _run(awq.awq_w4a16_gemv, x, dev, N).astype(np.float64)
    assert not np.isfinite(y[M - 1]).any()
    assert np.isfinite(y[:M - 1]).all()


# ---- decode at M = 1: more layer shapes ----------------------------------------
# K of one k-block, a ragged 9, 32 and 86 k-blocks; a last group of 4 row
# blocks; last groups of a single row block; 172 and 80 groups; K = 8192. Every
# output against the oracle, and two calls bit for bit equal.
ROWS_CASES = [(128, 4096), (1152, 4096), (4096, 4096), (11008, 4096), (4096, 2368), (2048, 6160), (4096, 12304),
              (1024, 22016), (8192, 10240)]


@pytest.mark.parametrize("K,N", ROWS_CASES)
def test_decode_m1_shapes_match_oracle(K, N):
    W, dev, hp = _packed(N, K, f"rows{K}x{N}")
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"rows{K}x{N}/x"), 1, K, 1.0)
    y = _run(awq.awq_w4a16_gemv, x, dev, N)
    y_ref, b = oracle.linear(x, *hp, N, K)
    check_close(y, y_ref, b, f"rows K={K} N={N}")
    y2 = _run(awq.awq_w4a16_gemv, x, dev, N)
    assert (y2.view(np.uint16) == y.view(np.uint16)).all()        # deterministic


def test_decode_m1_one_hot_wide_layer_gives_the_dequantized_weight_exactly():
    K, N = 1024, 4096
    W, dev, hp = _packed(N, K, "rows_onehot")
    q, z, s = oracle.unpack(*hp, N, K)
    wh = oracle.dequant(q, z, s)
    for k in (0, 127, 128, 555, 1023):
        x = np.zeros((1, K), np.float16)
        x[0, k] = 1.0
        y = _run(awq.awq_w4a16_gemv, x, dev, N)
        assert (y[0].view(np.uint16) == wh[:, k].view(np.uint16)).all(), k


# ---- decode at M <= 2: large K and odd row-block counts ----------------------
# K = 28672 at M = 1 and 2 (224 k-blocks per row); N/16 = 149 row blocks on
# 148 SMs; N/16 = 1041 (CTA ranges straddling groups, a last group of one row
# block); K = 14336 at M = 2. Every output against the oracle, and two calls
# bit for bit equal.
DECODE_ODD_CASES = [(28672, 512, 1), (28672, 256, 2), (1024, 2384, 1), (1024, 2384, 2), (256, 16656, 1),
                    (256, 16656, 2), (14336, 1040, 2)]


@pytest.mark.parametrize("K,N,M", DECODE_ODD_CASES)
def test_decode_odd_shapes_match_oracle(K, N, M):
    W, dev, hp = _packed(N, K, f"rowsk{K}x{N}")
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"rowsk{K}x{N}/x{M}"), M, K, 1.0)
    y = _run(awq.awq_w4a16_gemv, x, dev, N)
    y_ref, b = oracle.linear(x, *hp, N, K)
    check_close(y, y_ref, b, f"decode K={K} N={N} M={M}")
    y2 = _run(awq.awq_w4a16_gemv, x, dev, N)
    assert (y2.view(np.uint16) == y.view(np.uint16)).all()        # deterministic


# ---- the GEMM at small M on layers with more 128-channel tiles than SMs ----
# (some CTAs then walk two tiles: the regime where the dequant groups'
# alternating use of the code stages raced before the previous-phase wait).
# Against the oracle, and repeated calls bit for bit equal.
SMALL_M_MANY_TILES = [(4, 1024, 25600, 128), (4, 4096, 28672, 128), (32, 2048, 38400, 128), (16, 1024, 25600, 64)]


@pytest.mark.parametrize("M,K,N,group", SMALL_M_MANY_TILES)
def test_gemm_small_m_many_tiles(M, K, N, group):
    W, dev, hp = _packed(N, K, f"smt{K}x{N}", group=group)
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"smt{K}x{N}/x{M}"), M, K, 1.0)
    ys = [_run(awq.awq_w4a16_gemm, x, dev, N, group=group) for _ in range(5)]
    for y in ys[1:]:
        assert (y.view(np.uint16) == ys[0].view(np.uint16)).all()
    rows = sample_rows(N, 256, seed=M)
    y_ref, b = oracle_rows(x, *hp, N, K, rows, group)
    check_close(ys[0][:, rows], y_ref, b, f"gemm M={M} K={K} N={N} group={group}")


# ---- prefill GEMM on CTA pairs (tcgen05 cta_group::2) ------------------------
# The data-parallel schedule at 256-token tiles runs on clusters of two CTAs
# that share one MMA stream: 256 channels x 256 tokens per tile, each CTA
# dequantizing its 128 channels and loading its 128 tokens. Shapes (M, K, N,
# group): an even number of channel tiles; an odd one (the last pair has one
# CTA without channels) with a ragged last token tile; groups of 64 and 32.
PAIR_CASES = [(512, 256, 16384, 128), (500, 256, 16512, 128), (512, 256, 16384, 64), (512, 256, 16384, 32)]


@pytest.mark.parametrize("M,K,N,group", PAIR_CASES)
def test_gemm_cta_pairs_match_oracle(M, K, N, group):
    assert awq.awq_linear_path(M, K, N, group) == 3  # these shapes run on CTA pairs
    W, dev, hp = _packed(N, K, f"pair{K}x{N}", group=group)
    x = awq_synth.matrix_f16(awq_synth.key(0, 96, f"pair{K}x{N}/x{M}"), M, K, 1.0)
    xd = to_dev(x.view(np.uint16), torch.float16)
    ws = awq.new_workspace(M, K, N, xd.device, group)
    ys = [host(awq.awq_w4a16_gemm(xd, *dev, N, ws, group), np.float16) for _ in range(2)]
    assert awq.awq_get_status(ws) == awq.AWQ_OK
    assert (ys[0].view(np.uint16) == ys[1].view(np.uint16)).all()  # deterministic
    _check_against_oracle(ys[0], x, hp, N, K, f"pair gemm M={M} K={K} N={N} G={group}", group=group)


def test_gemm_cta_pairs_one_hot_gives_every_dequantized_weight():
    # every output channel of both CTAs of every pair, bit for bit
    M, K, N = 512, 256, 16512
    W, dev, hp = _packed(N, K, "pair1hot")
    x = np.zeros((M, K), np.float16)
    ks = [(37 * m + 11) % K for m in range(M)]
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    y = _run(awq.awq_w4a16_gemm, x, dev, N)
    q, z, s = oracle.unpack(*hp, N, K)
    wh = oracle.dequant(q, z, s)
    for m, k in enumerate(ks):
        assert (y[m].view(np.uint16) == wh[:, k].view(np.uint16)).all(), (m, k)
