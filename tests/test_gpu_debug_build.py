"""The debug build (libawq_b200_debug.so, compiled with -DAWQ_DEBUG): every
guarded global and shared access of the pack, dequant, GEMV and GEMM kernels
checks its index range before it happens and records AWQ_ERR_BOUNDS (and
skips the access) instead of faulting. Here it runs the small, ragged and
multi-tile shapes of the parity tests through the C ABI and must report
AWQ_OK, pack bit for bit like the oracle, and match the oracle's outputs
within the usual tolerance. No case here provokes an out-of-range access."""
import ctypes
import os

import numpy as np
import pytest
import torch

import awq_synth
import oracle
from gpu_helpers import check_close, host, to_dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _debug_lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_awq_b200_build_dbg", os.path.join(ROOT, "weight_only_bit_awq_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    lib = ctypes.CDLL(b.build(debug=True))
    vp, i64, ci, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.awq_workspace_bytes.argtypes = [i64, i64, i64, ci]
    lib.awq_workspace_bytes.restype = sz
    lib.awq_pack.argtypes = [vp, i64, i64, ci, vp, vp, vp, vp, sz, vp]
    lib.awq_dequant.argtypes = [vp, vp, vp, i64, i64, ci, vp, vp]
    for f in ("awq_w4a16_gemv", "awq_w4a16_gemm", "awq_linear"):
        getattr(lib, f).argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, ci, vp, sz, vp]
    lib.awq_get_status.argtypes = [vp, vp]
    return lib


_LIB = {}


def lib():
    if "l" not in _LIB:
        _LIB["l"] = _debug_lib()
    return _LIB["l"]


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _pack(W, group):
    L = lib()
    N, K = W.shape
    w = to_dev(W.view(np.uint16), torch.float16)
    qw = torch.empty(((N // 16) * (K // 128), 16, 16), dtype=torch.int32, device="cuda")
    sc = torch.empty((K // group, N), dtype=torch.float16, device="cuda")
    ze = torch.empty((K // group, N // 2), dtype=torch.uint8, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert L.awq_pack(w.data_ptr(), K, N, group, qw.data_ptr(), sc.data_ptr(), ze.data_ptr(), ws.data_ptr(), 256,
                      _stream()) == 0
    assert L.awq_get_status(ws.data_ptr(), _stream()) == 0
    return qw, sc, ze


# (entry point, M, K, N, group): GEMV at M = 1, 2 (integer path), 5, 17 and
# 32; ragged N and single-k-block K; the GEMM data-parallel with a ragged
# channel tile, at small M over more tiles than SMs, stream-K, and on CTA
# pairs (an odd number of channel tiles and a ragged token tile).
CASES = [("awq_w4a16_gemv", 1, 128, 16, 128), ("awq_w4a16_gemv", 2, 1152, 4096, 128),
         ("awq_w4a16_gemv", 5, 384, 336, 128), ("awq_w4a16_gemv", 17, 4096, 272, 128),
         ("awq_w4a16_gemv", 32, 1024, 592, 64), ("awq_w4a16_gemv", 1, 256, 16656, 32),
         ("awq_w4a16_gemm", 130, 1024, 592, 128), ("awq_w4a16_gemm", 4, 1024, 25600, 128),
         ("awq_w4a16_gemm", 300, 1024, 9600, 128), ("awq_linear", 40, 1024, 38400, 128),
         ("awq_w4a16_gemm", 500, 256, 15232, 128)]


@pytest.mark.parametrize("fn,M,K,N,group", CASES)
def test_debug_build_reports_no_bounds_error_and_matches_the_oracle(fn, M, K, N, group):
    L = lib()
    W = awq_synth.matrix_f16(awq_synth.key(0, 98, f"dbg{K}x{N}/W"), N, K, 0.02)
    qw, sc, ze = _pack(W, group)
    oq, osc, oze = oracle.quantize_pack(W, group)
    assert (host(qw, np.uint32).reshape(-1) == oq.reshape(-1)).all()
    assert (host(sc, np.uint16) == osc.view(np.uint16)).all() and (host(ze, np.uint8) == oze).all()
    x = awq_synth.matrix_f16(awq_synth.key(0, 98, f"dbg{K}x{N}/x{M}"), M, K, 1.0)
    xd = to_dev(x.view(np.uint16), torch.float16)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    nbytes = max(L.awq_workspace_bytes(M, K, N, group), 256)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        assert getattr(L, fn)(xd.data_ptr(), qw.data_ptr(), sc.data_ptr(), ze.data_ptr(), y.data_ptr(), M, K, N,
                              group, ws.data_ptr(), nbytes, _stream()) == 0
        assert L.awq_get_status(ws.data_ptr(), _stream()) == 0   # AWQ_OK: no bounds error
    y_ref, b = oracle.linear(x, oq, osc, oze, N, K, group)
    check_close(host(y, np.float16), y_ref, b, f"debug {fn} M={M} K={K} N={N} G={group}")
    wd = torch.empty((N, K), dtype=torch.float16, device="cuda")
    assert L.awq_dequant(qw.data_ptr(), sc.data_ptr(), ze.data_ptr(), K, N, group, wd.data_ptr(), _stream()) == 0
    q, z, s = oracle.unpack(oq, osc, oze, N, K, group)
    assert (host(wd, np.uint16) == oracle.dequant(q, z, s, group).view(np.uint16)).all()
