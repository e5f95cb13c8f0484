"""The seeded input generator: splitmix64 stream, normal draws, channel picks."""
import numpy as np

import awq_synth


def test_splitmix64_published_sequence():
    # splitmix64 seeded with 0 (S. Vigna's reference generator) starts with
    # these three outputs.
    w = awq_synth.words(0, 0, 3)
    assert [int(v) for v in w] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_based_and_deterministic():
    k = awq_synth.key(0, 1, "qkv/W")
    a = awq_synth.normal_f16(k, 1000)
    b = awq_synth.normal_f16(k, 500, start=500)
    assert (a[500:].view(np.uint16) == b.view(np.uint16)).all()
    m = awq_synth.matrix_f16(k, 3, 128, 1.0, row0=2)
    full = awq_synth.matrix_f16(k, 5, 128, 1.0)
    assert (m.view(np.uint16) == full[2:].view(np.uint16)).all()
    assert awq_synth.key(0, 1, "qkv/W") != awq_synth.key(0, 2, "qkv/W")


def test_normal_moments():
    a = awq_synth.normal_f16(awq_synth.key(0, 0, "moments"), 1 << 20, 0.02).astype(np.float64)
    assert abs(a.mean()) < 1e-4 and abs(a.std() - 0.02) < 2e-4


def test_outlier_channels():
    wl = awq_synth.WORKLOADS["llama2_70b_decode"]
    assert awq_synth.outlier_count(8192, wl.outlier_frac) == 82
    assert awq_synth.outlier_count(28672, wl.outlier_frac) == 287
    ch = awq_synth.pick_channels(awq_synth.key(0, 3, "x"), 8192, 82)
    assert len(set(ch.tolist())) == 82 and ch.min() >= 0 and ch.max() < 8192
    layer = wl.layer("o_proj")
    W = awq_synth.layer_weight(0, wl, layer, rows=slice(0, 64)).astype(np.float64)
    col_std = W.std(axis=0)
    big = np.sort(np.argsort(col_std)[-82:])
    chosen = np.sort(awq_synth.pick_channels(awq_synth.key(0, wl.config_id, "o_proj/outliers"), 8192, 82))
    assert (big == chosen).all()
