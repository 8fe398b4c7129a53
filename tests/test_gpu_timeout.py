"""The failure path of the bounded device-side waits, on a GPU, without a
fault: the test switch makes the GEMM's MMA warp wait on a barrier that
nothing arrives on, so the wait runs out after a short limit. The kernel must
return, record QLIN_ERR_TIMEOUT in the device status word (read on the
host), leave the context usable, free its TMEM and leave its barriers in a
state from which the next launches run normally: the forwards that follow are
checked against the oracle, three different GEMM launches in a row.
"""
import numpy as np
import pytest
import torch

import oracle
from tests._parity import assert_rows_close

pytestmark = pytest.mark.gpu


def _case(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn((M, K), generator=g)
    X[1, 3] = 11.0
    W = torch.randn((N, K), generator=g) * 0.02
    return X.to(torch.bfloat16), W.to(torch.bfloat16)


def test_wait_runs_out_and_the_device_recovers():
    import quantized_w8a8_linear_b200 as q
    torch.cuda.init()
    assert q.qlin_get_device_status(reset=True) == q.QLIN_OK
    X, W = _case(300, 520, 1024, 3)
    Wq, s_w = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_INT8_ROW)
    q.qlin_set_wait_timeout_ns(1_000_000)          # 1 ms
    q.qlin_debug_inject_wait_timeout(True)
    try:
        q.qlin_int8_outlier_forward(X.cuda(), Wq, s_w, 6.0)
        status = q.qlin_get_device_status(reset=True)   # synchronises: the kernel returned
    finally:
        q.qlin_debug_inject_wait_timeout(False)
        q.qlin_set_wait_timeout_ns(2_000_000_000)
    assert status == q.QLIN_ERR_TIMEOUT
    torch.cuda.synchronize()                       # no sticky CUDA error
    assert q.qlin_get_device_status() == q.QLIN_OK
    # the next launches find TMEM free and run normally
    for (M, N, K, seed) in ((300, 520, 1024, 3), (129, 257, 512, 4), (2048, 1024, 256, 5)):
        X, W = _case(M, N, K, seed)
        Wq, s_w = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_INT8_ROW)
        Y = q.qlin_int8_outlier_forward(X.cuda(), Wq, s_w, 6.0)
        r = oracle.int8_outlier_forward(X, Wq.cpu().numpy(), s_w.cpu().numpy(), 6.0)
        assert_rows_close(Y, r, what=f"after timeout {M}x{N}x{K}")
    assert q.qlin_get_device_status() == q.QLIN_OK
