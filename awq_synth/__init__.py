"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

Holds no quantization or matmul arithmetic: it draws fp16 weights W [N][K]
and fp16 activations x [M][K] from a counter-based splitmix64 + Box-Muller
generator (see ``synth.c``) and describes the workloads (layer shapes, batch
sizes, value distributions) of the W4A16 decode and prefill cases.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .workloads import WORKLOADS, Layer, Workload, outlier_count  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_SO = os.path.join(_HERE, "libawq_synth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile synth.c into an in-tree shared library (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=gnu11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            lib.synth_key.restype = u64
            lib.synth_key.argtypes = [u64, u64, u64]
            lib.synth_words.argtypes = [u64, i64, i64, vp]
            lib.synth_normal_f16.argtypes = [u64, i64, i64, dbl, vp]
            lib.synth_matrix_f16.argtypes = [u64, i64, i64, i64, dbl, vp, vp]
            lib.synth_pick_channels.restype = ctypes.c_int
            lib.synth_pick_channels.argtypes = [u64, i64, i64, vp, vp]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def name_id(name: str) -> int:
    """64-bit FNV-1a of a tensor name; the tensor id inside a workload."""
    h = 0xCBF29CE484222325
    for b in name.encode():
        h = ((h ^ b) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def key(seed: int, config_id: int, name: str) -> int:
    return int(_load().synth_key(seed, config_id, name_id(name)))


def words(k: int, start: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.uint64)
    _load().synth_words(k, start, count, _ptr(out))
    return out


def normal_f16(k: int, count: int, std: float = 1.0, start: int = 0) -> np.ndarray:
    out = np.empty(count, dtype=np.uint16)
    _load().synth_normal_f16(k, start, count, float(std), _ptr(out))
    return out.view(np.float16)


def pick_channels(k: int, K: int, count: int) -> np.ndarray:
    scratch = np.empty(K, dtype=np.int64)
    out = np.empty(count, dtype=np.int64)
    if _load().synth_pick_channels(k, K, count, _ptr(scratch), _ptr(out)) != 0:
        raise ValueError("bad channel count")
    return out


def matrix_f16(k: int, rows: int, K: int, std: float, chan_mult: np.ndarray | None = None,
               row0: int = 0) -> np.ndarray:
    """Rows [row0, row0+rows) of a seeded [*][K] fp16 matrix (element (n,k) uses
    normal number n*K+k of the stream, times chan_mult[k] if given)."""
    out = np.empty((rows, K), dtype=np.uint16)
    cm = None
    if chan_mult is not None:
        cm = np.ascontiguousarray(chan_mult, dtype=np.float64)
        assert cm.shape == (K,)
    _load().synth_matrix_f16(k, row0, rows, K, float(std), None if cm is None else _ptr(cm), _ptr(out))
    return out.view(np.float16)


def layer_weight(seed: int, wl: Workload, layer: Layer, rows: slice | None = None) -> np.ndarray:
    """fp16 W [N][K] of one layer of a workload (or a slice of its rows)."""
    kw = key(seed, wl.config_id, f"{layer.name}/W")
    mult = None
    if wl.outlier_frac > 0:
        cnt = outlier_count(layer.K, wl.outlier_frac)
        ch = pick_channels(key(seed, wl.config_id, f"{layer.name}/outliers"), layer.K, cnt)
        mult = np.ones(layer.K, dtype=np.float64)
        mult[ch] = wl.outlier_mult
    r0, r1 = (0, layer.N) if rows is None else (rows.start or 0, rows.stop if rows.stop is not None else layer.N)
    return matrix_f16(kw, r1 - r0, layer.K, wl.w_std, mult, row0=r0)


def layer_input(seed: int, wl: Workload, layer: Layer, M: int, tag: str = "") -> np.ndarray:
    """fp16 x [M][K] fed to one layer at batch M."""
    kx = key(seed, wl.config_id, f"{layer.name}/x/M={M}{tag}")
    return matrix_f16(kx, M, layer.K, wl.x_std)
