"""The C ABI library on the host: it loads, exports every symbol include/awq.h
declares, and rejects bad arguments with the documented codes before anything
is launched. No test here launches a kernel: the pointers are fake, and the
only call that gets past the argument checks runs only when no GPU exists
(it must then stop at the device check)."""
import ctypes
import os
import re

import pytest
import torch

import weight_only_bit_awq_b200 as awq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq.h")
L = awq.lib

FAKE = 0x7F0000000000          # 16-byte aligned, never dereferenced
FAKE2 = FAKE + (1 << 32)
FAKE3 = FAKE + (2 << 32)
FAKE4 = FAKE + (3 << 32)
FAKE5 = FAKE + (4 << 32)
FAKE6 = FAKE + (5 << 32)


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:awq_status|size_t|int|const char\*)\s+(awq_\w+)\(", text, re.M)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(awq.EXPORTS)


def test_every_declaration_names_its_source():
    # each entry point's comment ends with "Source:" and the page section that
    # defines the operation, or says that the pages have none
    text = open(HEADER).read()
    for name in declared_functions():
        m = re.search(r"/\*((?:(?!\*/).)*)\*/\s*(?:awq_status|size_t|int|const char\*)\s+" + name + r"\(", text, re.S)
        assert m, f"{name}: no comment right before the declaration"
        src = m.group(1).split("Source:")
        assert len(src) == 2, f"{name}: no Source line"
        assert ("TinyChat README" in src[1] or "TensorRT-LLM news item" in src[1]
                or "none on the pages" in src[1]), name


def test_library_exports_every_declared_symbol():
    for name in declared_functions():
        assert hasattr(L, name), name
        ctypes.cast(getattr(L, name), ctypes.c_void_p)


def test_status_strings():
    for code, name in awq.STATUS_NAMES.items():
        assert awq.awq_status_string(code).startswith(name)
    assert "unknown" in awq.awq_status_string(99)


def test_packed_sizes():
    assert awq.awq_packed_size(4096, 4096) == (4096 * 4096 // 2, 4096 // 128 * 4096 * 2, 4096 // 128 * 4096 // 2)
    for g in (64, 32):  # TinyChat README, Usage step 3: Falcon-7B uses groups of 64
        assert awq.awq_packed_size(4096, 4096, g) == (4096 * 4096 // 2, 4096 // g * 4096 * 2, 4096 // g * 4096 // 2)
    assert awq.awq_packed_size(11008, 4096)[0] == 11008 * 4096 // 2


@pytest.mark.parametrize("K,N,group,code", [
    (100, 16, 128, awq.AWQ_ERR_SHAPE), (128, 15, 128, awq.AWQ_ERR_SHAPE), (0, 16, 128, awq.AWQ_ERR_SHAPE),
    (128, 0, 128, awq.AWQ_ERR_SHAPE), (-128, 16, 128, awq.AWQ_ERR_SHAPE), (192, 16, 128, awq.AWQ_ERR_SHAPE),
    (128, 16, 256, awq.AWQ_ERR_UNSUPPORTED), (128, 16, 96, awq.AWQ_ERR_UNSUPPORTED), (128, 16, 16, awq.AWQ_ERR_UNSUPPORTED),
    (1 << 23, 16, 128, awq.AWQ_ERR_UNSUPPORTED),
])
def test_packed_size_rejects(K, N, group, code):
    with pytest.raises(awq.AwqError) as e:
        awq.awq_packed_size(K, N, group)
    assert e.value.status == code


def test_workspace_bytes():
    assert awq.awq_workspace_bytes(1, 100, 16) == 0
    assert awq.awq_workspace_bytes(-1, 128, 16) == 0
    assert awq.awq_workspace_bytes(0, 4096, 4096) >= 256
    assert awq.awq_workspace_bytes(2048, 4096, 4096) >= 256
    # the decode path's split-K partials grow with M * N
    assert awq.awq_workspace_bytes(32, 4096, 4096) >= awq.awq_workspace_bytes(1, 4096, 4096)


def test_gemm_schedule_on_148_sms():
    # Without a device the library plans for 148 SMs. Tiles are 128 channels x
    # 256 tokens here. Stream-K (a second, fixup kernel, and two fp32 slots of
    # 128 x 256 per SM in the workspace) when whole tiles fill under 80 % of the
    # SM-tile slots: 448 tiles = 3.03 waves at M = 512 (76 %), but not 1792 =
    # 12.1 waves at M = 2048 (93 %) or 7168 = 48.4 at M = 8192.
    slots = 256 + 148 * 2 * 256 * 128 * 4
    for M, launches in ((512, 2), (2048, 1), (8192, 1)):
        assert awq.awq_linear_launches(M, 4096, 28672, 128) == launches
        assert (awq.awq_workspace_bytes(M, 4096, 28672) >= slots) == (launches == 2)
    # never for decode sizes: those workspaces stay what the GEMV needs
    assert awq.awq_linear_launches(32, 14336, 4096, 128) in (1, 2)
    assert awq.awq_workspace_bytes(32, 14336, 4096) < slots
    # at least 8 k-blocks per SM: K = 128 with 8 tiles stays data-parallel
    assert awq.awq_linear_launches(40, 128, 1024, 128) == 1


def test_gemv_launches_no_fixup_when_every_cta_range_ends_on_a_group():
    # 148 SMs, M = 1: at K = 512 a group of 128 channels is one unit of 4
    # k-blocks, so N = 148 x 128 (148 units on 148 CTAs) and N = 296 x 128
    # (296 on 296) give every CTA whole groups: no split row, no fixup kernel
    assert awq.awq_linear_launches(1, 512, 148 * 128) == 1
    assert awq.awq_linear_launches(1, 512, 296 * 128) == 1
    # K = 1024 (2 units per group over 296 CTAs) and K = 4096 (8 per group
    # over 256 CTAs) put CTA boundaries inside groups: the GEMV and its fixup
    assert awq.awq_linear_launches(1, 1024, 148 * 128) == 2
    assert awq.awq_linear_launches(1, 4096, 4096) == 2


def _linear(fn, x=FAKE, q=FAKE2, s=FAKE3, z=FAKE4, y=FAKE5, M=1, K=4096, N=4096, group=128, ws=FAKE6,
            ws_bytes=1 << 30):
    return getattr(L, fn)(x, q, s, z, y, M, K, N, group, ws, ws_bytes, None)


ENTRIES = ["awq_w4a16_gemv", "awq_w4a16_gemm", "awq_linear"]


@pytest.mark.parametrize("fn", ENTRIES)
def test_linear_argument_errors(fn):
    assert _linear(fn, M=-1) == awq.AWQ_ERR_SHAPE
    assert _linear(fn, K=4000) == awq.AWQ_ERR_SHAPE
    assert _linear(fn, N=4104) == awq.AWQ_ERR_SHAPE
    assert _linear(fn, group=256) == awq.AWQ_ERR_UNSUPPORTED
    assert _linear(fn, group=96) == awq.AWQ_ERR_UNSUPPORTED
    assert _linear(fn, K=1 << 23) == awq.AWQ_ERR_UNSUPPORTED              # K, N <= 2^22
    assert _linear(fn, N=1 << 23) == awq.AWQ_ERR_UNSUPPORTED
    assert _linear(fn, x=None) == awq.AWQ_ERR_INVALID_ARG
    assert _linear(fn, y=None) == awq.AWQ_ERR_INVALID_ARG
    assert _linear(fn, ws=None) == awq.AWQ_ERR_INVALID_ARG
    assert _linear(fn, x=FAKE + 8) == awq.AWQ_ERR_ALIGNMENT
    assert _linear(fn, z=FAKE4 + 2) == awq.AWQ_ERR_ALIGNMENT
    assert _linear(fn, y=FAKE + 16) == awq.AWQ_ERR_INVALID_ARG          # y overlaps x
    assert _linear(fn, ws_bytes=16) == awq.AWQ_ERR_WORKSPACE
    assert _linear(fn, M=0) == awq.AWQ_OK                                  # empty batch: nothing to do
    assert _linear(fn, M=0, x=None, y=None) == awq.AWQ_OK                  # ... and x, y may be null


def test_gemv_rejects_large_batches():
    assert _linear("awq_w4a16_gemv", M=33) == awq.AWQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("fn", ["awq_w4a16_gemm", "awq_linear"])
def test_batches_above_the_limit_are_rejected(fn):
    assert _linear(fn, M=(1 << 24) + 1) == awq.AWQ_ERR_UNSUPPORTED         # M <= 2^24


def test_pack_and_dequant_argument_errors():
    assert L.awq_pack(FAKE, 100, 4096, 128, FAKE2, FAKE3, FAKE4, FAKE5, 1 << 20, None) == awq.AWQ_ERR_SHAPE
    assert L.awq_pack(None, 4096, 4096, 128, FAKE2, FAKE3, FAKE4, FAKE5, 1 << 20, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_pack(FAKE + 2, 4096, 4096, 128, FAKE2, FAKE3, FAKE4, FAKE5, 1 << 20, None) == awq.AWQ_ERR_ALIGNMENT
    assert L.awq_pack(FAKE, 4096, 4096, 128, FAKE, FAKE3, FAKE4, FAKE5, 1 << 20, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_pack(FAKE, 4096, 4096, 128, FAKE2, FAKE3, FAKE4, FAKE5, 8, None) == awq.AWQ_ERR_WORKSPACE
    assert L.awq_pack(FAKE, 4096, 4096, 64, FAKE2, FAKE3, FAKE4, FAKE5, 1 << 20, None) == awq.AWQ_ERR_UNSUPPORTED
    assert L.awq_dequant(FAKE2, FAKE3, FAKE4, 4096, 4096, 128, None, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_dequant(FAKE2, FAKE3, FAKE4, 4096, 4095, 128, FAKE, None) == awq.AWQ_ERR_SHAPE
    assert L.awq_dequant(FAKE2, FAKE3, FAKE4 + 1, 4096, 4096, 128, FAKE, None) == awq.AWQ_ERR_ALIGNMENT
    assert L.awq_workspace_init(None, 256, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_get_status(None, None) == awq.AWQ_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="would launch with fake pointers on a GPU")
def test_valid_arguments_without_a_device_stop_at_the_device_check():
    for fn in ENTRIES:
        assert _linear(fn) == awq.AWQ_ERR_UNSUPPORTED
    assert L.awq_pack(FAKE, 4096, 4096, 128, FAKE2, FAKE3, FAKE4, FAKE5, 1 << 20, None) == awq.AWQ_ERR_UNSUPPORTED
    assert L.awq_dequant(FAKE2, FAKE3, FAKE4, 4096, 4096, 128, FAKE, None) == awq.AWQ_ERR_UNSUPPORTED


def test_linear_launch_counts():
    assert awq.awq_linear_launches(0, 4096, 4096) == 0
    assert awq.awq_linear_launches(1, 4000, 4096) == 0
    assert awq.awq_linear_launches(8192, 4096, 4096) == 1          # the GEMM, data-parallel: one kernel
    assert awq.awq_linear_launches(300, 1024, 9600) == 2           # stream-K: the GEMM and its fixup
    assert awq.awq_linear_launches(1, 4096, 4096) in (1, 2)        # the GEMV, plus its fixup when rows are split


def test_bounded_wait_self_test_argument_errors():
    assert L.awq_check_bounded_wait(None, 256, 1000, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_check_bounded_wait(FAKE, 256, 0, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_check_bounded_wait(FAKE, 256, 2000000, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_check_bounded_wait(FAKE + 4, 256, 1000, None) == awq.AWQ_ERR_ALIGNMENT
    assert L.awq_check_bounded_wait(FAKE, 16, 1000, None) == awq.AWQ_ERR_WORKSPACE


def test_fp8_entry_points_reject_bad_arguments():
    # awq_fp8_row_exponents(scales, K, N, group, e_out, stream)
    assert L.awq_fp8_row_exponents(FAKE, 100, 16, 128, FAKE2, None) == awq.AWQ_ERR_SHAPE
    assert L.awq_fp8_row_exponents(FAKE, 128, 16, 96, FAKE2, None) == awq.AWQ_ERR_UNSUPPORTED
    assert L.awq_fp8_row_exponents(None, 128, 16, 128, FAKE2, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_fp8_row_exponents(FAKE + 2, 128, 16, 128, FAKE2, None) == awq.AWQ_ERR_ALIGNMENT
    assert L.awq_fp8_row_exponents(FAKE, 128, 16, 128, FAKE + 4, None) == awq.AWQ_ERR_INVALID_ARG  # overlap
    # awq_fp8_quantize_x(x, M, K, x8, sx, stream)
    assert L.awq_fp8_quantize_x(FAKE, 4, 100, FAKE2, FAKE3, None) == awq.AWQ_ERR_SHAPE
    assert L.awq_fp8_quantize_x(FAKE, -1, 128, FAKE2, FAKE3, None) == awq.AWQ_ERR_SHAPE
    assert L.awq_fp8_quantize_x(None, 0, 128, None, None, None) == awq.AWQ_OK          # empty batch
    assert L.awq_fp8_quantize_x(FAKE, 4, 128, None, FAKE3, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_fp8_quantize_x(FAKE, 4, 128, FAKE2 + 8, FAKE3, None) == awq.AWQ_ERR_ALIGNMENT
    assert L.awq_fp8_quantize_x(FAKE, 4, 128, FAKE + 256, FAKE3, None) == awq.AWQ_ERR_INVALID_ARG  # x8 inside x
    # awq_dequant_fp8(qweight, scales, zeros, row_exp, K, N, group, w8_out, stream)
    assert L.awq_dequant_fp8(FAKE, FAKE2, FAKE3, FAKE4, 128, 15, 128, FAKE5, None) == awq.AWQ_ERR_SHAPE
    assert L.awq_dequant_fp8(FAKE, FAKE2, FAKE3, None, 128, 16, 128, FAKE5, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_dequant_fp8(FAKE, FAKE2, FAKE3, FAKE4, 128, 16, 128, FAKE5 + 1, None) == awq.AWQ_ERR_ALIGNMENT
    # awq_w4a8_gemm(x8, sx, qweight, scales, zeros, row_exp, y, M, K, N, group, ws, ws_bytes, stream)
    args = [FAKE, FAKE2, FAKE3, FAKE4, FAKE5, FAKE6, FAKE6 + (1 << 20)]
    assert L.awq_w4a8_gemm(*args, 8, 128, 16, 128, FAKE6 + (1 << 24), 16, None) == awq.AWQ_ERR_WORKSPACE
    assert L.awq_w4a8_gemm(*args, -1, 128, 16, 128, FAKE6 + (1 << 24), 256, None) == awq.AWQ_ERR_SHAPE
    assert L.awq_w4a8_gemm(*args, 8, 128, 16, 256, FAKE6 + (1 << 24), 256, None) == awq.AWQ_ERR_UNSUPPORTED
    bad = list(args)
    bad[5] = None
    assert L.awq_w4a8_gemm(*bad, 8, 128, 16, 128, FAKE6 + (1 << 24), 256, None) == awq.AWQ_ERR_INVALID_ARG
    bad = list(args)
    bad[1] = FAKE2 + 4
    assert L.awq_w4a8_gemm(*bad, 8, 128, 16, 128, FAKE6 + (1 << 24), 256, None) == awq.AWQ_ERR_ALIGNMENT
    bad = list(args)
    bad[6] = FAKE                                    # y on top of x8
    assert L.awq_w4a8_gemm(*bad, 8, 128, 16, 128, FAKE6 + (1 << 24), 256, None) == awq.AWQ_ERR_INVALID_ARG
    assert L.awq_w4a8_gemm(*args, 0, 128, 16, 128, FAKE6 + (1 << 24), 256, None) == awq.AWQ_OK  # empty batch


def test_linear_dispatch_follows_the_measured_split():
    # GEMV up to M = 16 on every layer; from M = 17 to 32 the GEMM on layers
    # with at least as many 128-channel tiles as SMs (148 here), the GEMV on
    # narrower ones. The GEMV's split-row plans launch its fixup kernel too;
    # the GEMM at M <= 32 is data-parallel (one kernel).
    assert awq.awq_linear_gemv_limit() == 16
    assert awq.awq_linear_path(16, 4096, 28672) == 1   # GEMV
    assert awq.awq_linear_path(24, 4096, 28672) == 2   # GEMM: 224 tiles >= 148 SMs
    assert awq.awq_linear_path(24, 4096, 4096) == 1    # GEMV: 32 tiles
    assert awq.awq_linear_path(32, 8192, 57344) == 2   # GEMM
    assert awq.awq_linear_path(0, 4096, 4096) == 0
    assert awq.awq_linear_path(1, 4000, 4096) == 0


def test_gemm_runs_on_cta_pairs_for_data_parallel_256_token_tiles():
    # without a device the library plans for 148 SMs: 256-token tiles without
    # the stream-K split, and at least two channel tiles, run on CTA pairs
    assert awq.awq_linear_path(2048, 4096, 28672) == 3   # 1792 tiles, 12.1 waves
    assert awq.awq_linear_path(8192, 14848, 59392) == 3
    assert awq.awq_linear_path(500, 256, 15232) == 3     # 119 channel tiles: the last pair has one
    assert awq.awq_linear_path(512, 4096, 28672) == 2    # stream-K (3.03 waves): one CTA per tile
    assert awq.awq_linear_path(512, 14336, 4096) == 2    # 128-token tiles
    assert awq.awq_linear_path(200, 1024, 256) == 2
    for M, K, N in ((2048, 4096, 28672), (500, 256, 15232)):
        assert awq.awq_linear_launches(M, K, N) == 1
    assert awq.awq_linear_launches(16, 4096, 28672) == 2   # GEMV + fixup
    assert awq.awq_linear_launches(24, 4096, 28672) == 1   # GEMM, data-parallel
