"""GPU parity of the unquantised 16-bit linear (the layers a model keeps in
floating point: Image21-Turbo-OrbitQuant-W4A4, "What 4-bit breaks here and
what stays in fp16") against the CPU oracle: Y = dtype(X W^T + bias), the
tcgen05 kind::f16 GEMM with fp32 accumulation.

Per output row the normwise error against the oracle's rounded output is
<= 2e-3, and the output is no farther from the oracle's fp64 value than
correct rounding plus the fp32 accumulation (EXTRA_F16 of the row norm).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import assert_rows_close, sample_rows

pytestmark = pytest.mark.gpu

EXTRA_F16 = 5e-4


@pytest.fixture(scope="module")
def q():
    import quantized_w8a8_linear_b200 as q
    torch.cuda.init()
    assert q.qlin_get_device_status(reset=True) == 0
    yield q
    assert q.qlin_get_device_status() == 0


def _draw(M, N, K, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn((M, K), generator=g)
    if M > 3 and K > 40:
        X[3, 40] = 900.0                    # a massive activation: kept exactly by the 16-bit path
    W = torch.randn((N, K), generator=g) * 0.02
    b = torch.randn(N, generator=g) * 0.1
    return X.to(dtype), W.to(dtype), b.to(dtype)


@pytest.mark.parametrize("M,N,K", [(64, 512, 256), (200, 300, 208), (333, 520, 1024), (1, 1, 16),
                                   (257, 129, 64), (130, 4096, 3072), (70, 264, 32768)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_fp_linear_ragged(q, M, N, K, dtype):
    X, W, b = _draw(M, N, K, M * 31 + N + K, dtype)
    Y = q.qlin_fp_linear_forward(X.cuda(), W.cuda(), bias=b.cuda())
    r = oracle.fp_linear_forward(X, W, bias=b)
    assert Y.dtype == dtype
    assert_rows_close(Y, r, extra=EXTRA_F16, what=f"fp linear {M}x{N}x{K}")


def test_fp_linear_no_bias_and_empty(q):
    X, W, _ = _draw(100, 200, 512, 5, torch.bfloat16)
    Y = q.qlin_fp_linear_forward(X.cuda(), W.cuda())
    assert_rows_close(Y, oracle.fp_linear_forward(X, W), extra=EXTRA_F16, what="no bias")
    E = q.qlin_fp_linear_forward(torch.zeros((0, 512), dtype=torch.bfloat16, device="cuda"), W.cuda())
    assert E.shape == (0, 200)


def test_fp_linear_small_integers_exact(q):
    """Small-integer operands: every product and partial sum is an integer the
    fp32 accumulator holds exactly, so the output equals the integer matmul."""
    g = torch.Generator().manual_seed(9)
    M, N, K = 130, 260, 256
    xi = torch.randint(-1, 2, (M, K), generator=g)
    wi = torch.randint(-1, 2, (N, K), generator=g)
    Y = q.qlin_fp_linear_forward(xi.to(torch.bfloat16).cuda(), wi.to(torch.bfloat16).cuda())
    ref = (xi.double() @ wi.double().T)
    assert torch.all(ref.abs() <= 256)      # every result is a bf16 integer
    assert torch.equal(Y.cpu().double(), ref)


@pytest.mark.parametrize("wl_name,li", [("te_fp8_dynamic_mlp", 2), ("dit1024_int8_mlp", 0)])
def test_fp_linear_full_size(q, wl_name, li):
    """The text-encoder down projection (its activations carry the 9000/13000
    massive values) and the DiT up projection at full size, in bf16, outputs
    on 512 sampled rows."""
    wl = workloads.get_workload(wl_name)
    lin = wl.linears[li]
    X, W, bias = workloads.make_linear(wl, lin, index=li)
    Y = q.qlin_fp_linear_forward(X.cuda(), W.cuda(), bias=bias.cuda())
    rows = sample_rows(lin.M, n=512, seed=li, must=[0, 5])
    r = oracle.fp_linear_forward(X, W, bias=bias, rows=rows)
    assert_rows_close(Y, r, rows=rows, extra=EXTRA_F16, what=f"fp linear {lin.name}")
