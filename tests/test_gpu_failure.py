"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes expires into AWQ_ERR_TIMEOUT in the workspace status word, the host
reads it, and the context keeps working."""
import time

import numpy as np
import pytest
import torch

import awq_synth
import oracle
import weight_only_bit_awq_b200 as awq
from gpu_helpers import check_close, gpu_pack, host, packed_to_host, to_dev

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_context_survives():
    ws = awq.new_workspace(1, 1024, 256, torch.device("cuda"))
    t0 = time.perf_counter()
    awq.awq_check_bounded_wait(ws, limit_us=20000)
    assert awq.awq_get_status(ws) == awq.AWQ_ERR_TIMEOUT
    assert time.perf_counter() - t0 >= 0.015          # it waited about its limit, then gave up
    assert awq.awq_get_status(ws) == awq.AWQ_OK       # reading cleared the word
    # the same context still computes correctly
    W = awq_synth.matrix_f16(awq_synth.key(0, 94, "fail/W"), 256, 1024, 0.02)
    dev = gpu_pack(W)
    x = awq_synth.matrix_f16(awq_synth.key(0, 94, "fail/x"), 1, 1024, 1.0)
    y = host(awq.awq_w4a16_gemv(to_dev(x.view(np.uint16), torch.float16), *dev, 256, ws), np.float16)
    assert awq.awq_get_status(ws) == awq.AWQ_OK
    y_ref, b = oracle.linear(x, *packed_to_host(*dev), 256, 1024)
    check_close(y, y_ref, b, "after the expired wait")


def test_status_word_keeps_the_first_error():
    ws = awq.new_workspace(1, 1024, 256, torch.device("cuda"))
    awq.awq_check_bounded_wait(ws, limit_us=1000)
    W = np.zeros((16, 128), np.float16)
    W[3, 5] = np.inf
    awq.awq_pack(to_dev(W.view(np.uint16), torch.float16), ws)   # a second, different device error
    assert awq.awq_get_status(ws) == awq.AWQ_ERR_TIMEOUT
