"""The LLM.int8 forward with built-in scratch (qlin_int8_outlier_forward_noalloc).

This entry point serves callers that cannot allocate device memory where
they run the layer (a plugin whose host framework owns all allocations, a
latency-critical path that must not call cudaMalloc): it takes no workspace
and keeps its scratch in a device array inside the library. The test calls
it through the C ABI twice in a row, with different shapes, dtypes and
outlier sets, so the second call starts from the first call's leftovers in
the shared array, and compares each result with the regular entry point
qlin_int8_outlier_forward (which has a workspace of its own) within the
parity tolerance of the other GPU tests. The file is named to be collected
last; it does not depend on any other test having run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import ROW_REL_TOL, assert_rows_close

pytestmark = pytest.mark.gpu


def _row_rel(a: torch.Tensor, b: torch.Tensor) -> float:
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    den = np.linalg.norm(b, axis=1)
    num = np.linalg.norm(a - b, axis=1)
    return float(np.max(np.where(den > 0, num / np.where(den > 0, den, 1.0), num)))


def _noalloc(q, X, Wq, s_w, thr, bias=None):
    M, K = X.shape
    N = Wq.shape[0]
    Y = torch.full((M, N), float("nan"), dtype=X.dtype, device=X.device)
    st = q.lib.qlin_int8_outlier_forward_noalloc(
        ctypes.c_void_p(X.data_ptr()), q._dt(X), M, K, ctypes.c_void_p(Wq.data_ptr()),
        ctypes.c_void_p(s_w.data_ptr()), N, ctypes.c_float(thr),
        None if bias is None else ctypes.c_void_p(bias.data_ptr()), ctypes.c_void_p(Y.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == q.QLIN_OK, q.lib.qlin_last_error_string()
    return Y


def _case_a():
    g = torch.Generator().manual_seed(11)
    X = torch.randn((300, 1024), generator=g)
    for i in range(0, 300, 9):
        X[i, (i * 13) % 1024] = 9.0 + i / 50          # ~34 outlier columns (> 32: general path)
    W = torch.randn((520, 1024), generator=g) * 0.02
    bias = torch.randn(520, generator=g) * 0.1
    return X.to(torch.bfloat16), W.to(torch.bfloat16), bias.to(torch.bfloat16)


def _case_b():
    wl = workloads.get_workload("tiny_int8")            # fp16, 2 outlier columns
    X, W, bias = workloads.make_linear(wl, wl.linears[0])
    return X, W, bias


def test_noalloc_matches_regular_forward_twice():
    import quantized_w8a8_linear_b200 as q
    for X, W, bias in (_case_a(), _case_b()):
        Xc, Wc, bc = X.cuda(), W.cuda(), bias.cuda()
        Wq, s_w = q.qlin_quantize_weight(Wc, q.QLIN_W_INT8_ROW)
        ref = q.qlin_int8_outlier_forward(Xc, Wq, s_w, 6.0, bias=bc)
        got = _noalloc(q, Xc, Wq, s_w, 6.0, bias=bc)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        assert _row_rel(got, ref) <= ROW_REL_TOL
        # and directly against the CPU oracle, as the other parity tests do
        r = oracle.int8_outlier_forward(X, Wq.cpu().numpy(), s_w.cpu().numpy(), 6.0, bias=bias)
        assert_rows_close(got, r, what="no-alloc forward")
    assert q.qlin_get_device_status() == 0


def test_noalloc_accepts_the_documented_example_shape():
    """M = 2048, K = N = 4096 needs about 56 MiB of the 64 MiB array (the
    workspace layout without stream-K slots): accepted, and equal to the
    regular forward within the parity tolerance."""
    import quantized_w8a8_linear_b200 as q
    g = torch.Generator().manual_seed(12)
    M, K, N = 2048, 4096, 4096
    X = torch.randn((M, K), generator=g)
    X[5, 100] = 20.0
    X[1000, 4000] = -7.5
    X = X.to(torch.bfloat16).cuda()
    W = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16).cuda()
    Wq, s_w = q.qlin_quantize_weight(W, q.QLIN_W_INT8_ROW)
    ref = q.qlin_int8_outlier_forward(X, Wq, s_w, 6.0)
    got = _noalloc(q, X, Wq, s_w, 6.0)
    torch.cuda.synchronize()
    assert torch.isfinite(got.float()).all()
    assert _row_rel(got, ref) <= ROW_REL_TOL
    assert q.qlin_get_device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import quantized_w8a8_linear_b200 as q
    M, K, N = 4352, 12288, 12288                        # needs far more than 64 MiB of scratch
    assert q.qlin_workspace_bytes(q.QLIN_OP_INT8_OUTLIER, M, N, K) > (64 << 20)
    st = q.lib.qlin_int8_outlier_forward_noalloc(
        ctypes.c_void_p(4096), q.QLIN_BF16, M, K, ctypes.c_void_p(4096), ctypes.c_void_p(4096), N,
        ctypes.c_float(6.0), None, ctypes.c_void_p(4096), None)
    assert st == q.QLIN_ERR_UNSUPPORTED
    assert b"scratch" in q.lib.qlin_last_error_string()
