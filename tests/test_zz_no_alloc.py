"""awq_w4a16_gemv_no_alloc: the decode GEMV for callers that cannot allocate
device memory (e.g. code confined to a fixed memory pool, or a plug-in whose
host process owns every device allocation).

It is called here through the C ABI (ctypes) on two calls in a row and must
give the same y, bit for bit, as the workspace entry point awq_w4a16_gemv (the
same kernels run in the same order), and y within the tolerance of the other
parity tests of the fp64 oracle (|y - y_ref| <= 2e-3 * sum|x w| + 1e-3). Its
status word, read back with awq_get_status_no_alloc, must stay AWQ_OK. Sizes
whose scratch would exceed AWQ_GEMV_NO_ALLOC_SCRATCH_BYTES must be rejected
with AWQ_ERR_WORKSPACE, and a y that overlaps an input with
AWQ_ERR_INVALID_ARG, before anything runs. This file is collected last so that
a run stopping at the first failure has run every other test before it.
"""
import numpy as np
import pytest
import torch

import awq_synth
import oracle
import weight_only_bit_awq_b200 as awq
from gpu_helpers import check_close, gpu_pack, host, packed_to_host, to_dev

pytestmark = pytest.mark.gpu

SCRATCH_MAX = 1 << 20   # AWQ_GEMV_NO_ALLOC_SCRATCH_BYTES in include/awq.h


def _no_alloc(x, qw, sc, ze, y, N):
    M, K = x.shape
    return awq.lib.awq_w4a16_gemv_no_alloc(x.data_ptr(), qw.data_ptr(), sc.data_ptr(), ze.data_ptr(),
                                           y.data_ptr(), M, K, N, 128, torch.cuda.current_stream().cuda_stream)


# (K, N, M): split-K on (down-projection shape) and off, one and many tokens
CASES = [(11008, 4096, 1), (11008, 4096, 5), (4096, 12288, 1), (1024, 272, 32), (4096, 4096, 32)]


@pytest.mark.parametrize("K,N,M", CASES)
def test_matches_the_workspace_entry_point_on_two_calls_in_a_row(K, N, M):
    W = awq_synth.matrix_f16(awq_synth.key(0, 95, f"noalloc/{K}x{N}/W"), N, K, 0.02)
    dev = gpu_pack(W)
    hp = packed_to_host(*dev)
    x = awq_synth.matrix_f16(awq_synth.key(0, 95, f"noalloc/{K}x{N}/x{M}"), M, K, 1.0)
    xd = to_dev(x.view(np.uint16), torch.float16)
    need = awq.awq_workspace_bytes(M, K, N)
    y = torch.zeros((M, N), dtype=torch.float16, device="cuda")
    if need > SCRATCH_MAX:
        assert _no_alloc(xd, *dev, y, N) == awq.AWQ_ERR_WORKSPACE
        torch.cuda.synchronize()
        assert (y == 0).all()          # rejected before anything ran
        return
    ws = awq.new_workspace(M, K, N, xd.device)
    y_ws = host(awq.awq_w4a16_gemv(xd, *dev, N, ws), np.uint16)
    assert awq.awq_get_status(ws) == awq.AWQ_OK
    y_ref, bound = oracle.linear(x, *hp, N, K)
    for call in range(2):
        y.fill_(float("nan"))
        assert _no_alloc(xd, *dev, y, N) == awq.AWQ_OK
        assert awq.awq_get_status_no_alloc() == awq.AWQ_OK
        y_na = host(y, np.uint16)
        assert np.array_equal(y_na, y_ws), (call, int((y_na != y_ws).sum()))
        check_close(y_na.view(np.float16), y_ref, bound, f"no-alloc call {call}, M={M} K={K} N={N}")


def test_sizes_beyond_the_scratch_are_rejected():
    # the largest decode plans of this library need more than the 1 MiB array
    rejected = [(M, K, N) for (M, K, N) in [(32, 4096, 4096), (32, 14336, 4096), (16, 4096, 4096)]
                if awq.awq_workspace_bytes(M, K, N) > SCRATCH_MAX]
    assert rejected, "no candidate exceeds the scratch size"
    M, K, N = rejected[0]
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    qw = torch.zeros((N // 16, K // 128, 16, 16), dtype=torch.int32, device="cuda")
    sc = torch.zeros((K // 128, N), dtype=torch.float16, device="cuda")
    ze = torch.zeros((K // 128, N // 2), dtype=torch.uint8, device="cuda")
    y = torch.zeros((M, N), dtype=torch.float16, device="cuda")
    assert _no_alloc(x, qw, sc, ze, y, N) == awq.AWQ_ERR_WORKSPACE


def test_argument_errors():
    x = torch.zeros((1, 128), dtype=torch.float16, device="cuda")
    qw = torch.zeros((1, 1, 16, 16), dtype=torch.int32, device="cuda")
    sc = torch.zeros((1, 16), dtype=torch.float16, device="cuda")
    ze = torch.zeros((1, 8), dtype=torch.uint8, device="cuda")
    y = torch.zeros((1, 16), dtype=torch.float16, device="cuda")
    L = awq.lib
    s = torch.cuda.current_stream().cuda_stream
    args = [x.data_ptr(), qw.data_ptr(), sc.data_ptr(), ze.data_ptr(), y.data_ptr()]
    assert L.awq_w4a16_gemv_no_alloc(*args, 33, 128, 16, 128, s) == awq.AWQ_ERR_UNSUPPORTED
    assert L.awq_w4a16_gemv_no_alloc(*args, 1, 100, 16, 128, s) == awq.AWQ_ERR_SHAPE
    assert L.awq_w4a16_gemv_no_alloc(*args, 1, 128, 16, 96, s) == awq.AWQ_ERR_UNSUPPORTED
    assert L.awq_w4a16_gemv_no_alloc(None, *args[1:], 1, 128, 16, 128, s) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_w4a16_gemv_no_alloc(*args, 0, 128, 16, 128, s) == awq.AWQ_OK
    # y overlapping x, the codes, the scales or the zeros
    for alias in (x, qw, sc, ze):
        bad = [x.data_ptr(), qw.data_ptr(), sc.data_ptr(), ze.data_ptr(), alias.data_ptr()]
        assert L.awq_w4a16_gemv_no_alloc(*bad, 1, 128, 16, 128, s) == awq.AWQ_ERR_INVALID_ARG
    assert awq.awq_get_status_no_alloc() == awq.AWQ_OK
