"""W4A16 group-quantized linear layer for NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libawq_b200.so`` (C ABI: ``include/awq.h``).
Every step of the computation runs in the library's CUDA kernels; this
module only checks tensors, allocates output buffers with PyTorch and passes
raw device pointers and the current CUDA stream. There is no CPU fallback:
importing the binding fails loudly if the shared library cannot be loaded.

Functions (same names as the C entry points):
  awq_packed_size, awq_workspace_bytes, awq_workspace_init, awq_pack,
  awq_dequant, awq_w4a16_gemv, awq_w4a16_gemm, awq_linear,
  awq_linear_gemv_limit, awq_linear_launches, awq_linear_path, awq_check_bounded_wait,
  awq_get_status, awq_status_string, awq_w4a16_gemv_no_alloc,
  awq_get_status_no_alloc, and the W4A8-FP8
  variant awq_fp8_row_exponents, awq_fp8_quantize_x, awq_dequant_fp8,
  awq_w4a8_gemm.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# AWQ_B200_DEBUG=1 loads the debug build (every guarded device access checks
# its index range and records AWQ_ERR_BOUNDS instead of faulting).
DEBUG = os.environ.get("AWQ_B200_DEBUG", "") == "1"
LIB_PATH = os.path.join(_PKG, "libawq_b200_debug.so" if DEBUG else "libawq_b200.so")

GROUP = 128
GEMV_MAX_M = 32

STATUS_NAMES = {
    0: "AWQ_OK", 1: "AWQ_ERR_INVALID_ARG", 2: "AWQ_ERR_SHAPE", 3: "AWQ_ERR_ALIGNMENT", 4: "AWQ_ERR_WORKSPACE",
    5: "AWQ_ERR_UNSUPPORTED", 6: "AWQ_ERR_CUDA", 7: "AWQ_ERR_TIMEOUT", 8: "AWQ_ERR_NONFINITE", 9: "AWQ_ERR_BOUNDS",
}
globals().update({name: code for code, name in STATUS_NAMES.items()})

# Every symbol include/awq.h declares.
EXPORTS = ("awq_packed_size", "awq_workspace_bytes", "awq_workspace_init", "awq_pack", "awq_dequant",
           "awq_w4a16_gemv", "awq_w4a16_gemm", "awq_linear", "awq_linear_gemv_limit", "awq_get_status",
           "awq_status_string", "awq_w4a16_gemv_no_alloc", "awq_get_status_no_alloc", "awq_linear_launches",
           "awq_linear_path",
           "awq_check_bounded_wait",
           "awq_fp8_row_exponents", "awq_fp8_quantize_x", "awq_dequant_fp8", "awq_w4a8_gemm")


class AwqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {awq_status_string(status)}")


class _PackedSizes(ctypes.Structure):
    _fields_ = [("qweight_bytes", ctypes.c_size_t), ("scales_bytes", ctypes.c_size_t),
                ("zeros_bytes", ctypes.c_size_t)]


def _build_module():
    """build.py loaded by path (importing it must not load the library)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("_awq_b200_build", os.path.join(_PKG, "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _load() -> ctypes.CDLL:
    # (Re)compile in-tree with nvcc when the library is missing or older than
    # its sources; a failed build raises, there is no fallback.
    _build_module().build(debug=DEBUG)
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, ci, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.awq_packed_size.argtypes = [i64, i64, ci, ctypes.POINTER(_PackedSizes)]
    lib.awq_workspace_bytes.argtypes = [i64, i64, i64, ci]
    lib.awq_workspace_bytes.restype = sz
    lib.awq_workspace_init.argtypes = [vp, sz, vp]
    lib.awq_pack.argtypes = [vp, i64, i64, ci, vp, vp, vp, vp, sz, vp]
    lib.awq_dequant.argtypes = [vp, vp, vp, i64, i64, ci, vp, vp]
    for f in ("awq_w4a16_gemv", "awq_w4a16_gemm", "awq_linear"):
        getattr(lib, f).argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, ci, vp, sz, vp]
    lib.awq_w4a16_gemv_no_alloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, ci, vp]
    lib.awq_get_status_no_alloc.argtypes = [vp]
    lib.awq_linear_gemv_limit.argtypes = []
    lib.awq_linear_launches.argtypes = [i64, i64, i64, ci]
    lib.awq_linear_path.argtypes = [i64, i64, i64, ci]
    lib.awq_check_bounded_wait.argtypes = [vp, sz, ctypes.c_uint32, vp]
    lib.awq_get_status.argtypes = [vp, vp]
    lib.awq_fp8_row_exponents.argtypes = [vp, i64, i64, ci, vp, vp]
    lib.awq_fp8_quantize_x.argtypes = [vp, i64, i64, vp, vp, vp]
    lib.awq_dequant_fp8.argtypes = [vp, vp, vp, vp, i64, i64, ci, vp, vp]
    lib.awq_w4a8_gemm.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, ci, vp, sz, vp]
    lib.awq_status_string.argtypes = [ci]
    lib.awq_status_string.restype = ctypes.c_char_p
    for f in EXPORTS:
        if f not in ("awq_workspace_bytes", "awq_status_string"):
            getattr(lib, f).restype = ci
    return lib


lib = _load()


def awq_status_string(status: int) -> str:
    return lib.awq_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != 0:
        raise AwqError(status, where)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _dev(t: torch.Tensor, dtype, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def awq_packed_size(K: int, N: int, group: int = GROUP) -> tuple[int, int, int]:
    out = _PackedSizes()
    _check(lib.awq_packed_size(K, N, group, ctypes.byref(out)), "awq_packed_size")
    return out.qweight_bytes, out.scales_bytes, out.zeros_bytes


def awq_workspace_bytes(M: int, K: int, N: int, group: int = GROUP) -> int:
    return int(lib.awq_workspace_bytes(M, K, N, group))


def awq_workspace_init(workspace: torch.Tensor):
    _check(lib.awq_workspace_init(_dev(workspace, torch.uint8, "workspace"), workspace.numel(),
                                  _stream(workspace)), "awq_workspace_init")


def new_workspace(M: int, K: int, N: int, device, group: int = GROUP) -> torch.Tensor:
    """Allocate (with torch) and zero a workspace large enough for (M, K, N)."""
    nbytes = awq_workspace_bytes(M, K, N, group)
    if nbytes == 0:
        raise AwqError(AWQ_ERR_SHAPE, "awq_workspace_bytes")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    awq_workspace_init(ws)
    return ws


def awq_pack(w: torch.Tensor, workspace: torch.Tensor, group: int = GROUP):
    """w fp16 [N][K] -> (qweight int32 [(N/16)*(K/128)][16][16] packed blocks in the order
    include/awq.h documents, scales fp16 [K/G][N], zeros uint8 [K/G][N/2])."""
    N, K = w.shape
    qweight = torch.empty(((N // 16) * (K // 128), 16, 16), dtype=torch.int32, device=w.device)
    scales = torch.empty((K // group, N), dtype=torch.float16, device=w.device)
    zeros = torch.empty((K // group, N // 2), dtype=torch.uint8, device=w.device)
    _check(lib.awq_pack(_dev(w, torch.float16, "w"), K, N, group, qweight.data_ptr(), scales.data_ptr(),
                        zeros.data_ptr(), _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(w)),
           "awq_pack")
    return qweight, scales, zeros


def awq_dequant(qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, K: int, N: int,
                group: int = GROUP) -> torch.Tensor:
    w = torch.empty((N, K), dtype=torch.float16, device=qweight.device)
    _check(lib.awq_dequant(_dev(qweight, torch.int32, "qweight"), _dev(scales, torch.float16, "scales"),
                           _dev(zeros, torch.uint8, "zeros"), K, N, group, w.data_ptr(), _stream(qweight)),
           "awq_dequant")
    return w


def _linear_call(fn, name, x, qweight, scales, zeros, N, workspace, group, y):
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    elif y.shape != (M, N):
        raise ValueError(f"y must be [{M}, {N}]")
    _check(fn(_dev(x, torch.float16, "x"), _dev(qweight, torch.int32, "qweight"),
              _dev(scales, torch.float16, "scales"), _dev(zeros, torch.uint8, "zeros"),
              _dev(y, torch.float16, "y"), M, K, N, group, _dev(workspace, torch.uint8, "workspace"),
              workspace.numel(), _stream(x)), name)
    return y


def awq_w4a16_gemv(x, qweight, scales, zeros, N, workspace, group: int = GROUP, y=None):
    """Decode GEMV (1 <= M <= 32): y fp16 [M][N] = x fp16 [M][K] . W^T."""
    return _linear_call(lib.awq_w4a16_gemv, "awq_w4a16_gemv", x, qweight, scales, zeros, N, workspace, group, y)


def awq_w4a16_gemm(x, qweight, scales, zeros, N, workspace, group: int = GROUP, y=None):
    """Prefill GEMM on tcgen05 tensor cores (any M)."""
    return _linear_call(lib.awq_w4a16_gemm, "awq_w4a16_gemm", x, qweight, scales, zeros, N, workspace, group, y)


def awq_linear(x, qweight, scales, zeros, N, workspace, group: int = GROUP, y=None):
    """The linear layer: the GEMV for M <= awq_linear_gemv_limit() (and up to
    M = 32 on layers with fewer 128-channel tiles than SMs), the GEMM otherwise."""
    return _linear_call(lib.awq_linear, "awq_linear", x, qweight, scales, zeros, N, workspace, group, y)


def awq_w4a16_gemv_no_alloc(x, qweight, scales, zeros, N, group: int = GROUP, y=None):
    """Decode GEMV for callers that cannot allocate device memory: no
    workspace argument; the library's own static scratch array is used (see
    include/awq.h). Here torch allocates y only when the caller passes none."""
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    _check(lib.awq_w4a16_gemv_no_alloc(_dev(x, torch.float16, "x"), _dev(qweight, torch.int32, "qweight"),
                                       _dev(scales, torch.float16, "scales"), _dev(zeros, torch.uint8, "zeros"),
                                       _dev(y, torch.float16, "y"), M, K, N, group, _stream(x)),
           "awq_w4a16_gemv_no_alloc")
    return y


def awq_get_status_no_alloc(device=None) -> int:
    """Synchronize the current stream; return (and clear) the status word of
    the no-alloc GEMV's scratch array on the current device."""
    return int(lib.awq_get_status_no_alloc(torch.cuda.current_stream(device).cuda_stream))


def awq_fp8_row_exponents(scales: torch.Tensor, K: int, N: int, group: int = GROUP) -> torch.Tensor:
    """int8 [N]: per output channel, the power of two that moves its weights into
    the E4M3 range (W4A8-FP8 variant; once per weight, like awq_pack)."""
    e = torch.empty(N, dtype=torch.int8, device=scales.device)
    _check(lib.awq_fp8_row_exponents(_dev(scales, torch.float16, "scales"), K, N, group, e.data_ptr(),
                                     _stream(scales)), "awq_fp8_row_exponents")
    return e


def awq_fp8_quantize_x(x: torch.Tensor):
    """x fp16 [M][K] -> (x8 uint8 E4M3 codes [M][K], sx float32 [M])."""
    M, K = x.shape
    x8 = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    sx = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib.awq_fp8_quantize_x(_dev(x, torch.float16, "x"), M, K, x8.data_ptr(), sx.data_ptr(), _stream(x)),
           "awq_fp8_quantize_x")
    return x8, sx


def awq_dequant_fp8(qweight, scales, zeros, row_exp, K: int, N: int, group: int = GROUP) -> torch.Tensor:
    """uint8 [N][K]: the E4M3 weight codes the W4A8 GEMM multiplies (test surface)."""
    w8 = torch.empty((N, K), dtype=torch.uint8, device=qweight.device)
    _check(lib.awq_dequant_fp8(_dev(qweight, torch.int32, "qweight"), _dev(scales, torch.float16, "scales"),
                               _dev(zeros, torch.uint8, "zeros"), _dev(row_exp, torch.int8, "row_exp"), K, N, group,
                               w8.data_ptr(), _stream(qweight)), "awq_dequant_fp8")
    return w8


def awq_w4a8_gemm(x8, sx, qweight, scales, zeros, row_exp, N, workspace, group: int = GROUP, y=None):
    """W4A8-FP8 prefill GEMM (tcgen05 kind::f8f6f4): y fp16 [M][N] from the
    outputs of awq_fp8_quantize_x and awq_fp8_row_exponents."""
    M, K = x8.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x8.device)
    elif y.shape != (M, N):
        raise ValueError(f"y must be [{M}, {N}]")
    _check(lib.awq_w4a8_gemm(_dev(x8, torch.uint8, "x8"), _dev(sx, torch.float32, "sx"),
                             _dev(qweight, torch.int32, "qweight"), _dev(scales, torch.float16, "scales"),
                             _dev(zeros, torch.uint8, "zeros"), _dev(row_exp, torch.int8, "row_exp"),
                             _dev(y, torch.float16, "y"), M, K, N, group, _dev(workspace, torch.uint8, "workspace"),
                             workspace.numel(), _stream(x8)), "awq_w4a8_gemm")
    return y


def awq_linear_gemv_limit() -> int:
    return int(lib.awq_linear_gemv_limit())


def awq_linear_launches(M: int, K: int, N: int, group: int = GROUP) -> int:
    """Kernels awq_linear launches for these sizes on the current device."""
    return int(lib.awq_linear_launches(M, K, N, group))


def awq_linear_path(M: int, K: int, N: int, group: int = GROUP) -> int:
    """Kernel awq_linear runs for these sizes: 1 = the GEMV, 2 = the GEMM, 3 = the
    GEMM on CTA pairs, 0 = none."""
    return int(lib.awq_linear_path(M, K, N, group))


def awq_check_bounded_wait(workspace: torch.Tensor, limit_us: int = 1000):
    """Run the kernels' bounded wait on a barrier nothing completes (self-test);
    afterwards awq_get_status(workspace) reports AWQ_ERR_TIMEOUT."""
    _check(lib.awq_check_bounded_wait(_dev(workspace, torch.uint8, "workspace"), workspace.numel(), limit_us,
                                      _stream(workspace)), "awq_check_bounded_wait")


def awq_get_status(workspace: torch.Tensor) -> int:
    """Synchronize the current stream; return (and clear) the device-side status word."""
    return int(lib.awq_get_status(_dev(workspace, torch.uint8, "workspace"), _stream(workspace)))
