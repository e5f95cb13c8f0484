"""Shared helpers of the GPU parity tests: seeded inputs, GPU packing through
the C ABI, oracle references on sampled rows, and the output tolerance.

Tolerance (fp16 outputs of the W4A16 matmul):
    |y_gpu - y_ref| <= 2e-3 * B + 1e-3,   B = sum_k |x[m,k] * W^[n,k]|
with y_ref and B computed by the fp64 oracle from the same packed buffers.
"""
from __future__ import annotations

import numpy as np
import torch

import awq_synth
import oracle
import weight_only_bit_awq_b200 as awq

REL_TOL = 2e-3
ABS_TOL = 1e-3
G = 128


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def host(t: torch.Tensor, np_dtype) -> np.ndarray:
    return t.cpu().numpy().view(np_dtype)


def gpu_pack(W: np.ndarray, ws: torch.Tensor | None = None, group: int = G):
    """fp16 W [N][K] -> GPU packed (qweight int32, scales fp16, zeros uint8); checks the status word."""
    N, K = W.shape
    w = to_dev(W.view(np.uint16), torch.float16)
    if ws is None:
        ws = awq.new_workspace(0, K, N, w.device, group)
    qw, sc, ze = awq.awq_pack(w, ws, group)
    st = awq.awq_get_status(ws)
    assert st == awq.AWQ_OK, awq.awq_status_string(st)
    return qw, sc, ze


def block_of(nb: int, kb: int, KB: int, NB: int) -> int:
    """Block number of row block nb, k-block kb in the packed layout of
    include/awq.h (groups of 8 row blocks, k-block-major inside a group)."""
    gi = nb // 8
    R = min(8, NB - 8 * gi)
    return 8 * gi * KB + kb * R + nb % 8


def packed_to_host(qw, sc, ze):
    return host(qw, np.uint32), host(sc, np.float16), host(ze, np.uint8)


def check_close(y_gpu: np.ndarray, y_ref: np.ndarray, bound: np.ndarray, what: str = ""):
    y_gpu = y_gpu.astype(np.float64)
    err = np.abs(y_gpu - y_ref)
    lim = REL_TOL * bound + ABS_TOL
    bad = ~(err <= lim)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} outputs outside tolerance, e.g. "
                             + ", ".join(f"{tuple(i)}: gpu {y_gpu[tuple(i)]:.6g} ref {y_ref[tuple(i)]:.6g} "
                                         f"bound {bound[tuple(i)]:.3g}" for i in idx))
    return float((err / lim).max()) if err.size else 0.0


def layer_inputs(wl_name: str, layer_name: str, M: int, seed: int = 0):
    wl = awq_synth.WORKLOADS[wl_name]
    layer = wl.layer(layer_name)
    W = awq_synth.layer_weight(seed, wl, layer)
    x = awq_synth.layer_input(seed, wl, layer, M)
    return W, x


def sample_rows(N: int, count: int, seed: int = 0) -> np.ndarray:
    """First and last 16-row block, plus random rows."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(16, N))) | set(range(max(0, N - 16), N))
    rows |= set(rng.choice(N, size=min(count, N), replace=False).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def oracle_rows(x: np.ndarray, qw, sc, ze, N: int, K: int, rows: np.ndarray, group: int = G):
    """Oracle y, B [M][len(rows)] at the given output channels."""
    M = x.shape[0]
    ms = np.repeat(np.arange(M), len(rows))
    ns = np.tile(rows, M)
    # group by row so the oracle unpacks each row once
    order = np.lexsort((ms, ns))
    y = np.empty(len(ms))
    b = np.empty(len(ms))
    yo, bo = oracle.linear_entries(x, qw, sc, ze, N, K, ms[order], ns[order], group)
    y[order] = yo
    b[order] = bo
    return y.reshape(M, len(rows)), b.reshape(M, len(rows))
