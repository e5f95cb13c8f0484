"""CPU oracle for the W4A16 group-quantized linear layer (fp64, plain C).

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The CUDA library
never loads it; the two share no code (the only common inputs come from the
seeded generator in ``awq_synth``, which holds none of the method's
arithmetic).

The arithmetic lives in ``awq_oracle.c`` (see its header for every step and
the passage it follows). This module only compiles it with gcc and marshals
numpy arrays through ctypes. fp16 tensors cross the boundary as their uint16
bit patterns.

Pins (tests/test_oracle_*.py) check it against things other than itself:
exhaustive fp16 conversion against numpy/torch, exactly representable groups
(zero error, original q/z/s recovered), the per-element error bound, nearest-
grid-point brute force over all 16 codes, hand-derived tie cases
(tests/golden/), pack/unpack round trips and a hand-derived packed word, one-
hot activations, a second factored matmul route, numpy's fp64 matmul and
exact rational arithmetic on tiny shapes. The W4A8-FP8 functions
(tests/test_oracle_fp8.py) are pinned to torch's float8_e4m3fn decoding and
in-range rounding, hand-derived ties, saturation and exponent cases, and a
closed-form bound against the W4A16 layer.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "awq_oracle.c")
_SO = os.path.join(_HERE, "liborc.so")
_lock = threading.Lock()
_lib = None

OK = 0
ERR_SHAPE = 2
ERR_NONFINITE = 8


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile awq_oracle.c into an in-tree shared library (plain -O2, no
    fast-math, no FMA contraction, so every fp64 operation rounds once)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                               "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
            lib.orc_half_to_double.restype = ctypes.c_double
            lib.orc_half_to_double.argtypes = [ctypes.c_uint16]
            lib.orc_double_to_half.restype = ctypes.c_uint16
            lib.orc_double_to_half.argtypes = [ctypes.c_double]
            lib.orc_quantize.argtypes = [vp, i64, i64, ci, vp, vp, vp]
            lib.orc_dequant.argtypes = [vp, vp, vp, i64, i64, ci, vp]
            lib.orc_pack.argtypes = [vp, vp, vp, i64, i64, ci, vp, vp, vp]
            lib.orc_unpack.argtypes = [vp, vp, vp, i64, i64, ci, vp, vp, vp]
            lib.orc_matmul.argtypes = [vp, i64, vp, i64, i64, vp, vp]
            lib.orc_matmul_factored.argtypes = [vp, i64, vp, vp, vp, i64, i64, ci, vp]
            lib.orc_linear_rows.argtypes = [vp, i64, vp, vp, vp, i64, i64, ci, i64, i64, vp, vp]
            lib.orc_linear.argtypes = [vp, i64, vp, vp, vp, i64, i64, ci, vp, vp]
            lib.orc_linear_entries.argtypes = [vp, i64, vp, vp, vp, i64, i64, ci, vp, vp, i64, vp, vp]
            lib.orc_e4m3_to_double.restype = ctypes.c_double
            lib.orc_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.orc_double_to_e4m3.restype = ctypes.c_uint8
            lib.orc_double_to_e4m3.argtypes = [ctypes.c_double]
            lib.orc_fp8_quantize_x.argtypes = [vp, i64, i64, vp, vp]
            lib.orc_fp8_row_exponents.argtypes = [vp, i64, i64, ci, vp]
            lib.orc_fp8_weights.argtypes = [vp, vp, vp, vp, i64, i64, ci, vp]
            lib.orc_fp8_linear_rows.argtypes = [vp, vp, i64, vp, vp, vp, vp, i64, i64, ci, i64, i64, vp, vp]
            lib.orc_fp8_linear_entries.argtypes = [vp, vp, i64, vp, vp, vp, vp, i64, i64, ci, vp, vp, i64, vp, vp]
            for f in ("orc_quantize", "orc_dequant", "orc_pack", "orc_unpack", "orc_matmul",
                      "orc_matmul_factored", "orc_linear_rows", "orc_linear", "orc_linear_entries",
                      "orc_fp8_quantize_x", "orc_fp8_row_exponents", "orc_fp8_weights", "orc_fp8_linear_rows",
                      "orc_fp8_linear_entries"):
                getattr(lib, f).restype = ci
            _lib = lib
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _bits(a: np.ndarray) -> np.ndarray:
    """fp16 array -> contiguous uint16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


def _check(rc: int, what: str):
    if rc == ERR_NONFINITE:
        raise OracleError(f"{what}: non-finite weight")
    if rc != OK:
        raise OracleError(f"{what}: error {rc}")


# -- binary16 ---------------------------------------------------------------

def half_to_double(bits: int) -> float:
    return float(_load().orc_half_to_double(int(bits)))


def double_to_half(d: float) -> int:
    return int(_load().orc_double_to_half(float(d)))


# -- quantization -----------------------------------------------------------

def quantize(W: np.ndarray, group: int = 128, allow_nonfinite: bool = False):
    """W fp16 [N][K] -> (q uint8 [N][K], z uint8 [N][K/G], s fp16 [N][K/G])."""
    Wb = _bits(W)
    N, K = Wb.shape
    q = np.zeros((N, K), np.uint8)
    z = np.zeros((N, K // group), np.uint8)
    s = np.zeros((N, K // group), np.uint16)
    rc = _load().orc_quantize(_p(Wb), N, K, group, _p(q), _p(z), _p(s))
    if not (allow_nonfinite and rc == ERR_NONFINITE):
        _check(rc, "quantize")
    return q, z, s.view(np.float16), rc


def dequant(q, z, s, group: int = 128) -> np.ndarray:
    N, K = q.shape
    out = np.empty((N, K), np.uint16)
    _check(_load().orc_dequant(_p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(z)), _p(_bits(s)),
                               N, K, group, _p(out)), "dequant")
    return out.view(np.float16)


# -- packed layout ----------------------------------------------------------

def pack(q, z, s, group: int = 128):
    """-> (qweight uint32 [N/16][K/128][16][16], scales fp16 [K/G][N], zeros uint8 [K/G][N/2])."""
    N, K = q.shape
    qw = np.empty((N // 16, K // 128, 16, 16), np.uint32)
    sc = np.empty((K // group, N), np.uint16)
    ze = np.empty((K // group, N // 2), np.uint8)
    _check(_load().orc_pack(_p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(z)), _p(_bits(s)),
                            N, K, group, _p(qw), _p(sc), _p(ze)), "pack")
    return qw, sc.view(np.float16), ze


def unpack(qweight, scales, zeros, N: int, K: int, group: int = 128):
    q = np.empty((N, K), np.uint8)
    z = np.empty((N, K // group), np.uint8)
    s = np.empty((N, K // group), np.uint16)
    _check(_load().orc_unpack(_p(np.ascontiguousarray(qweight)), _p(_bits(scales)),
                              _p(np.ascontiguousarray(zeros)), N, K, group, _p(q), _p(z), _p(s)), "unpack")
    return q, z, s.view(np.float16)


def quantize_pack(W, group: int = 128):
    q, z, s, _ = quantize(W, group)
    return pack(q, z, s, group)


# -- matmul -----------------------------------------------------------------

def matmul(x, What):
    """y, B [M][N] (fp64) for x fp16 [M][K] and W^ fp16 [N][K]."""
    xb, wb = _bits(x), _bits(What)
    M, K = xb.shape
    N = wb.shape[0]
    y = np.empty((M, N), np.float64)
    b = np.empty((M, N), np.float64)
    _check(_load().orc_matmul(_p(xb), M, _p(wb), N, K, _p(y), _p(b)), "matmul")
    return y, b


def matmul_factored(x, q, z, s, group: int = 128):
    xb = _bits(x)
    M, K = xb.shape
    N = q.shape[0]
    y = np.empty((M, N), np.float64)
    _check(_load().orc_matmul_factored(_p(xb), M, _p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(z)),
                                       _p(_bits(s)), N, K, group, _p(y)), "matmul_factored")
    return y


def linear(x, qweight, scales, zeros, N: int, K: int, group: int = 128, rows: tuple | None = None):
    """y, B for x . W^T computed from the packed buffers (all rows, or rows n0..n1-1)."""
    xb = _bits(x)
    M = xb.shape[0]
    n0, n1 = (0, N) if rows is None else rows
    y = np.empty((M, n1 - n0), np.float64)
    b = np.empty((M, n1 - n0), np.float64)
    _check(_load().orc_linear_rows(_p(xb), M, _p(np.ascontiguousarray(qweight)), _p(_bits(scales)),
                                   _p(np.ascontiguousarray(zeros)), N, K, group, n0, n1, _p(y), _p(b)),
           "linear")
    return y, b


def linear_entries(x, qweight, scales, zeros, N: int, K: int, ms, ns, group: int = 128):
    """y, B at the listed output coordinates (ms[i], ns[i])."""
    xb = _bits(x)
    M = xb.shape[0]
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    y = np.empty(len(ms), np.float64)
    b = np.empty(len(ms), np.float64)
    _check(_load().orc_linear_entries(_p(xb), M, _p(np.ascontiguousarray(qweight)), _p(_bits(scales)),
                                      _p(np.ascontiguousarray(zeros)), N, K, group, _p(ms), _p(ns), len(ms),
                                      _p(y), _p(b)), "linear_entries")
    return y, b


# -- W4A8-FP8 variant (E4M3 activations and weights) --------------------------

def e4m3_to_double(code: int) -> float:
    return float(_load().orc_e4m3_to_double(int(code)))


def double_to_e4m3(d: float) -> int:
    """Nearest E4M3 value (ties to even), saturating at +-448; NaN -> 0x7F."""
    return int(_load().orc_double_to_e4m3(float(d)))


def fp8_quantize_x(x):
    """x fp16 [M][K] -> (x8 uint8 E4M3 codes [M][K], sx float32 [M])."""
    xb = _bits(x)
    M, K = xb.shape
    x8 = np.empty((M, K), np.uint8)
    sx = np.empty(M, np.float32)
    _check(_load().orc_fp8_quantize_x(_p(xb), M, K, _p(x8), _p(sx)), "fp8_quantize_x")
    return x8, sx


def fp8_row_exponents(scales, N: int, K: int, group: int = 128) -> np.ndarray:
    """int8 [N]: the largest e with 15 * max_g s[n] * 2^e <= 448."""
    e = np.empty(N, np.int8)
    _check(_load().orc_fp8_row_exponents(_p(_bits(scales)), N, K, group, _p(e)), "fp8_row_exponents")
    return e


def fp8_weights(qweight, scales, zeros, e, N: int, K: int, group: int = 128) -> np.ndarray:
    """uint8 [N][K]: E4M3 codes of W^[n,k] * 2^e[n]."""
    w8 = np.empty((N, K), np.uint8)
    _check(_load().orc_fp8_weights(_p(np.ascontiguousarray(qweight)), _p(_bits(scales)),
                                   _p(np.ascontiguousarray(zeros)), _p(np.ascontiguousarray(e, dtype=np.int8)),
                                   N, K, group, _p(w8)), "fp8_weights")
    return w8


def fp8_linear(x8, sx, qweight, scales, zeros, e, N: int, K: int, group: int = 128, rows: tuple | None = None):
    """y, B (fp64) of the W4A8-FP8 layer for all rows, or rows n0..n1-1."""
    x8 = np.ascontiguousarray(x8, dtype=np.uint8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    M = x8.shape[0]
    n0, n1 = (0, N) if rows is None else rows
    y = np.empty((M, n1 - n0), np.float64)
    b = np.empty((M, n1 - n0), np.float64)
    _check(_load().orc_fp8_linear_rows(_p(x8), _p(sx), M, _p(np.ascontiguousarray(qweight)), _p(_bits(scales)),
                                       _p(np.ascontiguousarray(zeros)), _p(np.ascontiguousarray(e, dtype=np.int8)),
                                       N, K, group, n0, n1, _p(y), _p(b)), "fp8_linear")
    return y, b


def fp8_linear_entries(x8, sx, qweight, scales, zeros, e, N: int, K: int, ms, ns, group: int = 128):
    x8 = np.ascontiguousarray(x8, dtype=np.uint8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    M = x8.shape[0]
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    y = np.empty(len(ms), np.float64)
    b = np.empty(len(ms), np.float64)
    _check(_load().orc_fp8_linear_entries(_p(x8), _p(sx), M, _p(np.ascontiguousarray(qweight)), _p(_bits(scales)),
                                          _p(np.ascontiguousarray(zeros)),
                                          _p(np.ascontiguousarray(e, dtype=np.int8)), N, K, group, _p(ms), _p(ns),
                                          len(ms), _p(y), _p(b)), "fp8_linear_entries")
    return y, b
