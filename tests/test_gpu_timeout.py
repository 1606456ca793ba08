"""Failure path of the bounded waits, made to happen without a GPU fault: the
GEMM's pipeline waits are given a poll bound of zero (svq_debug_set_wait_polls),
so the first wait gives up at once.  The kernel must return (no hang, no trap),
report SVQ_ERR_TIMEOUT through the device status word, and leave the context
usable: the next call with the default bound succeeds and is correct."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, rel_err, torch, x_bf16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu


def test_gemm_wait_timeout_is_reported_and_recoverable():
    need_gpu()
    m = synth.make_matrix(98, 0, 256, 512, 8)
    W = svq.SvqWeight.from_synth(m)
    M = 64
    x_bits = synth.make_x(98, 1, M, m.K, dtype="bf16")
    x = x_bf16(x_bits)
    y = torch.empty((M, m.N), dtype=torch.float32, device="cuda")
    nb = svq.svq_linear_gemm_workspace_size(W, M)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    assert svq.svq_get_device_status() == svq.SVQ_OK
    prev = svq.svq_debug_set_wait_polls(0)
    try:
        svq.svq_linear_gemm(W, x, y, ws)
        torch.cuda.synchronize()                  # the kernel returned
        assert svq.svq_get_device_status() == svq.SVQ_ERR_TIMEOUT
    finally:
        svq.svq_debug_set_wait_polls(prev)
    assert prev > 0
    svq.svq_linear_gemm(W, x, y, ws)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_OK
    y_ref, den = oracle.linear(m, x_bits, "bf16")
    assert rel_err(y.cpu().numpy(), y_ref, den) <= 1e-2
