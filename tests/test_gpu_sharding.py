"""N-sharded layer on one GPU: a world of one is the full layer bit for bit;
two shards built in one process pack exactly the column slices of the full GPU
packing and their outputs, side by side, match the oracle. (The all-gather
itself is exercised on CPU ranks with gloo in test_sharding.py; this run has
one GPU, so no NCCL collective spans GPUs here.)"""
import numpy as np
import pytest
import torch

import awq_synth
import oracle
import weight_only_bit_awq_b200 as awq
from gpu_helpers import check_close, gpu_pack, host, packed_to_host, to_dev
from weight_only_bit_awq_b200.sharding import ShardedLinear, shard_range

pytestmark = pytest.mark.gpu


def _W(N, K):
    return awq_synth.matrix_f16(awq_synth.key(0, 99, f"gshard/{N}x{K}"), N, K, 0.02)


@pytest.mark.parametrize("M", [1, 8, 300])
def test_world_of_one_is_the_full_layer(M):
    N, K = 592, 1024
    W = _W(N, K)
    Wd = to_dev(W.view(np.uint16), torch.float16)
    sl = ShardedLinear(Wd, 1, 0)
    x = to_dev(awq_synth.matrix_f16(awq_synth.key(0, 99, f"gshard/x{M}"), M, K, 1.0).view(np.uint16), torch.float16)
    full = gpu_pack(W)
    ws = awq.new_workspace(M, K, N, x.device)
    y_ref = host(awq.awq_linear(x, *full, N, ws), np.uint16)
    assert (host(sl.forward_full(x), np.uint16) == y_ref).all()


@pytest.mark.parametrize("N,world", [(592, 2), (4096, 3)])
def test_shards_in_one_process(N, world):
    K, M = 2048, 5
    W = _W(N, K)
    Wd = to_dev(W.view(np.uint16), torch.float16)
    full = packed_to_host(*gpu_pack(W))
    x = awq_synth.matrix_f16(awq_synth.key(0, 99, f"gshard/x{N}"), M, K, 1.0)
    xd = to_dev(x.view(np.uint16), torch.float16)
    ys = []
    KB = K // 128
    for r in range(world):
        sl = ShardedLinear(Wd, world, r)
        n0, n1 = shard_range(N, world, r)
        sq, ss, sz = packed_to_host(*sl.packed)
        b0 = (n0 // 16) * KB
        assert np.array_equal(sq.reshape(-1, 256), full[0].reshape(-1, 256)[b0:b0 + (n1 - n0) // 16 * KB])
        assert np.array_equal(ss.view(np.uint16), full[1][:, n0:n1].view(np.uint16))
        assert np.array_equal(sz, full[2][:, n0 // 2:n1 // 2])
        ys.append(host(sl.forward(xd), np.float16))
    y = np.concatenate(ys, 1)
    y_ref, b = oracle.linear(x, *full, N, K)
    check_close(y, y_ref, b, f"sharded N={N} world={world}")
