"""GPU quantize+pack and dequant, bit for bit against the CPU oracle."""
import numpy as np
import pytest
import torch

import awq_synth
import oracle
import weight_only_bit_awq_b200 as awq
from gpu_helpers import block_of, gpu_pack, host, packed_to_host, to_dev

pytestmark = pytest.mark.gpu
G = 128


def _adversarial(N=64, K=1024):
    """Groups that stress the rounding and clamping rules: exact ties for
    rint(v/s) with odd zero points, all-positive / all-negative groups,
    subnormal scales, constant and all-zero groups, outlier channels."""
    rng = np.random.default_rng(21)
    W = awq_synth.matrix_f16(awq_synth.key(0, 97, "adv/W"), N, K, 0.02).astype(np.float64)
    W[:, rng.choice(K, 10, replace=False)] *= 20.0
    W[0:4, 0:G] = np.abs(W[0:4, 0:G]) + 0.01
    W[4:8, G:2 * G] = -np.abs(W[4:8, G:2 * G]) - 0.01
    W[8:12, 2 * G:3 * G] *= 1e-3
    W[12:16, 3 * G:4 * G] = 0.25
    W[16:20, 4 * G:5 * G] = 0.0
    # exact ties: s = 2^-6 with lo = -3s, hi = 12s and values at (k + 1/2) s
    s = 2.0 ** -6
    tie = np.full(G, 0.0)
    tie[0], tie[1] = -3 * s, 12 * s
    tie[2:30] = (rng.integers(-3, 12, 28) + 0.5) * s
    W[20:24, 5 * G:6 * G] = tie
    # exactly representable groups (zero error)
    z = rng.integers(0, 16)
    q = rng.integers(0, 16, G)
    q[:2] = [0, 15]
    W[24:28, 6 * G:7 * G] = (q - z) * 2.0 ** -8
    return W.astype(np.float16)


def _check_pack(W, group=G):
    N, K = W.shape
    qw, sc, ze = packed_to_host(*gpu_pack(W, group=group))
    oq, osc, oze = oracle.quantize_pack(W, group)
    assert (qw == oq.reshape(qw.shape)).all(), "qweight differs"
    assert (sc.view(np.uint16) == osc.view(np.uint16)).all(), "scales differ"
    assert (ze == oze).all(), "zeros differ"


@pytest.mark.parametrize("N,K", [(16, 128), (32, 256), (48, 384), (64, 1024), (272, 640)])
def test_pack_bit_exact_small(N, K):
    W = awq_synth.matrix_f16(awq_synth.key(0, 97, f"pack/{N}x{K}"), N, K, 0.02)
    _check_pack(W)


def test_pack_bit_exact_adversarial_groups():
    _check_pack(_adversarial())


@pytest.mark.parametrize("group", [64, 32])
@pytest.mark.parametrize("N,K", [(16, 128), (48, 384), (272, 640)])
def test_pack_bit_exact_group_sizes(group, N, K):
    W = awq_synth.matrix_f16(awq_synth.key(0, 97, f"pack{group}/{N}x{K}"), N, K, 0.02)
    _check_pack(W, group)


@pytest.mark.parametrize("group", [64, 32])
def test_pack_and_dequant_bit_exact_adversarial_group_sizes(group):
    W = _adversarial()
    N, K = W.shape
    _check_pack(W, group)
    qw, sc, ze = gpu_pack(W, group=group)
    wh = host(awq.awq_dequant(qw, sc, ze, K, N, group), np.float16)
    q, z, s, _ = oracle.quantize(W, group)
    assert (wh.view(np.uint16) == oracle.dequant(q, z, s, group).view(np.uint16)).all()


def test_dequant_bit_exact():
    W = _adversarial()
    N, K = W.shape
    qw, sc, ze = gpu_pack(W)
    wh = host(awq.awq_dequant(qw, sc, ze, K, N), np.float16)
    q, z, s, _ = oracle.quantize(W)
    ref = oracle.dequant(q, z, s)
    assert (wh.view(np.uint16) == ref.view(np.uint16)).all()
    # exactly representable groups come back unchanged
    assert (wh[24:28, 6 * G:7 * G].view(np.uint16) == W[24:28, 6 * G:7 * G].view(np.uint16)).all()


def test_dequant_of_oracle_packed_buffers():
    # the GPU dequant reads the oracle's packing (layout agreement both ways)
    W = awq_synth.matrix_f16(awq_synth.key(0, 97, "deq/W"), 96, 512, 0.02)
    oq, osc, oze = oracle.quantize_pack(W)
    wh = host(awq.awq_dequant(to_dev(oq.view(np.int32)), to_dev(osc.view(np.uint16), torch.float16),
                              to_dev(oze), 512, 96), np.float16)
    q, z, s, _ = oracle.quantize(W)
    assert (wh.view(np.uint16) == oracle.dequant(q, z, s).view(np.uint16)).all()


@pytest.mark.parametrize("bad", [np.inf, np.nan])
def test_non_finite_weight_sets_the_status_word(bad):
    W = awq_synth.matrix_f16(awq_synth.key(0, 97, "nf/W"), 32, 256, 0.02).copy()
    W[17, 140] = bad
    w = to_dev(W.view(np.uint16), torch.float16)
    ws = awq.new_workspace(0, 256, 32, w.device)
    qw, sc, ze = awq.awq_pack(w, ws)
    assert awq.awq_get_status(ws) == awq.AWQ_ERR_NONFINITE
    assert awq.awq_get_status(ws) == awq.AWQ_OK      # reading clears it
    # every other group is still exact
    oq, osc, oze = oracle.quantize_pack(np.where(np.isfinite(W), W, 0).astype(np.float16))
    sch = host(sc, np.uint16)
    mask = np.ones_like(sch, bool)
    mask[1, 17] = False
    assert (sch[mask] == osc.view(np.uint16)[mask]).all()


@pytest.mark.parametrize("wl,layer", [("llama2_7b_decode", "down"), ("llama2_70b_decode", "gate_up"),
                                      ("prefill", "falcon180b")])
def test_pack_bit_exact_full_size_sampled(wl, layer):
    """Full-size layer packed on the GPU; the oracle re-quantizes sampled row
    blocks (quantization is independent per row) and must match them bit for bit."""
    w = awq_synth.WORKLOADS[wl]
    L = w.layer(layer)
    W = awq_synth.layer_weight(0, w, L)
    qw, sc, ze = packed_to_host(*gpu_pack(W))
    KB = L.K // 128
    rng = np.random.default_rng(1)
    blocks = sorted(set([0, L.N // 16 - 1]) | set(rng.choice(L.N // 16, 6, replace=False).tolist()))
    for nb in blocks:
        rows = slice(16 * nb, 16 * nb + 16)
        oq, osc, oze = oracle.quantize_pack(np.ascontiguousarray(W[rows]))
        blocks_gpu = qw.reshape(-1, 16, 16)[[block_of(nb, kb, KB, L.N // 16) for kb in range(KB)]]
        assert (blocks_gpu == oq.reshape(KB, 16, 16)).all(), nb
        assert (sc[:, rows].view(np.uint16) == osc.view(np.uint16)).all(), nb
        assert (ze[:, 8 * nb:8 * nb + 8] == oze).all(), nb
