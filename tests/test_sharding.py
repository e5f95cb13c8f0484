"""N-sharded (column-parallel) layer: host logic on CPU.

- shard_range: contiguous whole groups of 128 output channels covering N
  once, balanced to one group, empty ranges allowed.
- A shard's packed buffers (the oracle packing W[n0:n1]) are exactly the
  matching block range and column slices of the full packing, so each rank can
  pack its own slice.
- all_gather_columns over gloo ranks (world sizes 2 and 3): each rank computes
  its slice with the oracle from its own shard's packing; the assembled y
  equals the oracle's full y bit for bit (every output depends only on its own
  row of W).
"""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import awq_synth
import oracle
from weight_only_bit_awq_b200.sharding import all_gather_columns, max_shard, shard_range

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N", [16, 128, 336, 4096, 12288, 22016, 59392])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_ranges_cover_n_in_whole_groups(N, world):
    rs = [shard_range(N, world, r) for r in range(world)]
    assert rs[0][0] == 0 and rs[-1][1] == N
    for (a0, a1), (b0, b1) in zip(rs, rs[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in rs]
    assert all(a % 128 == 0 for a, b in rs if b > a)   # empty ranges sit at N
    groups = [-(-s // 128) for s in sizes]
    assert max(groups) - min(groups) <= 1
    assert max_shard(N, world) == max(sizes)


def _W(N, K, tag):
    return awq_synth.matrix_f16(awq_synth.key(0, 99, f"shard/{tag}"), N, K, 0.02)


@pytest.mark.parametrize("N,world", [(336, 2), (640, 3), (4096, 8)])
def test_a_shards_packing_is_a_slice_of_the_full_packing(N, world):
    K = 512
    W = _W(N, K, f"{N}")
    qw, sc, ze = oracle.quantize_pack(W)
    KB = K // 128
    flat = qw.reshape(-1, 16, 16)
    for r in range(world):
        n0, n1 = shard_range(N, world, r)
        if n0 == n1:
            continue
        sq, ss, sz = oracle.quantize_pack(W[n0:n1])
        b0 = (n0 // 16) * KB                      # whole groups: the shard's blocks are contiguous
        assert np.array_equal(sq.reshape(-1, 16, 16), flat[b0:b0 + (n1 - n0) // 16 * KB])
        assert np.array_equal(ss.view(np.uint16), sc[:, n0:n1].view(np.uint16))
        assert np.array_equal(sz, ze[:, n0 // 2:n1 // 2])


def _rank(rank, world, port, N, K, M, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W = _W(N, K, f"ag{N}")
        x = awq_synth.matrix_f16(awq_synth.key(0, 99, f"shard/x{M}"), M, K, 1.0)
        n0, n1 = shard_range(N, world, rank)
        if n1 > n0:
            y_local, _ = oracle.linear(x, *oracle.quantize_pack(W[n0:n1]), n1 - n0, K)
        else:
            y_local = np.zeros((M, 0))
        y = all_gather_columns(torch.from_numpy(np.ascontiguousarray(y_local)), N, world, rank)
        out.put((rank, y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N", [(2, 336), (3, 640)])
def test_all_gather_assembles_the_full_output(world, N):
    K, M = 256, 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() + world) % 2000
    procs = [ctx.Process(target=_rank, args=(r, world, port, N, K, M, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W = _W(N, K, f"ag{N}")
    x = awq_synth.matrix_f16(awq_synth.key(0, 99, f"shard/x{M}"), M, K, 1.0)
    y_ref, _ = oracle.linear(x, *oracle.quantize_pack(W), N, K)
    for r in range(world):
        assert np.array_equal(res[r], y_ref)
