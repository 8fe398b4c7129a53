"""GPU parity at full size: one DiT block at 2048^2 (16640 tokens = 16384 image
+ 256 text, hidden 3072: fused QKV 9216, out 3072, MLP up 12288, MLP down
back to 3072), in LLM.int8 mode and in W4A8 mode, in the launch
configuration the bench times.

Per linear: the activation prep is compared in full (outlier set, count,
row scales and every int8 code, bit for bit); the int32 accumulators and the
outputs on 512 seeded rows x all columns (the CPU oracle is too slow for all
16640 rows of a 12288 x 3072 contraction in a test). W4A8 adds ragged shapes
at K = 12288 (96 groups), where the per-group promotion runs longest.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import assert_rows_close, sample_rows

pytestmark = pytest.mark.gpu

THR = 6.0
EXTRA_W4A8 = 1e-3   # fp32 group sums in the kernel's order
N_ROWS = 512


@pytest.fixture(scope="module")
def q():
    import quantized_w8a8_linear_b200 as q
    torch.cuda.init()
    assert q.qlin_get_device_status(reset=True) == 0
    yield q
    assert q.qlin_get_device_status() == 0, "a device-side wait timed out"


@pytest.mark.parametrize("li", [0, 1, 2, 3], ids=["qkv", "out", "mlp_up", "mlp_down"])
def test_int8_dit2048_block_full_size(q, li):
    wl = workloads.get_workload("dit2048_block_int8")
    lin = wl.linears[li]
    X, W, bias = workloads.make_linear(wl, lin, index=li)
    Xc = X.cuda()
    # prep in full: outlier set, scales, codes
    p = q.qlin_int8_prep(Xc, THR)
    r = oracle.int8_outlier_prep(X, THR)
    n = int(p["count"].item())
    assert n == r["count"] and n > 0
    assert np.array_equal(p["O"].cpu().numpy()[:n], r["O"])
    assert np.array_equal(p["s_x"].cpu().numpy(), r["s_x"])
    assert np.array_equal(p["Xq"].cpu().numpy(), r["Xq"])
    del p
    Wq, s_w = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_INT8_ROW)
    rq, rs = oracle.quantize_weight(W, "int8_row")
    assert np.array_equal(Wq.cpu().numpy(), rq) and np.array_equal(s_w.cpu().numpy(), rs)
    # the fused forward's own int32 accumulator (the path the bench times)
    ws = q.workspace(q.QLIN_OP_INT8_OUTLIER, lin.M, lin.N, lin.K, "cuda")
    q.qlin_int8_outlier_prepare(Xc, Wq, s_w, THR, ws)
    rows = sample_rows(lin.M, n=N_ROWS, seed=20 + li, must=[0, 255, 256, lin.M - 1])
    C = q.qlin_int8_outlier_gemm_i32(lin.M, lin.K, Wq, ws)[rows].cpu().numpy()
    Y = q.qlin_int8_outlier_forward(Xc, Wq, s_w, THR, ws=ws)
    ro = oracle.int8_outlier_forward(X, rq, rs, THR, rows=rows)
    assert np.array_equal(C, ro["C"])
    assert_rows_close(Y, ro, rows=rows, what=f"int8 2048^2 {lin.name}")


@pytest.mark.parametrize("li", [0, 1, 2, 3], ids=["qkv", "out", "mlp_up", "mlp_down"])
def test_w4a8_dit2048_block_full_size(q, li):
    wl = workloads.get_workload("dit2048_block_w4a8")
    lin = wl.linears[li]
    X, W, bias = workloads.make_linear(wl, lin, index=li)
    Xc = X.cuda()
    Xq, s_x = q.qlin_w4a8_prep(Xc)
    r = oracle.int8_outlier_prep(X, float("inf"))
    assert np.array_equal(Xq.cpu().numpy(), r["Xq"]) and np.array_equal(s_x.cpu().numpy(), r["s_x"])
    Wq4, sw = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_INT4_G128)
    rq, rs = oracle.quantize_weight(W, "int4_g128")
    assert np.array_equal(Wq4.cpu().numpy(), rq) and np.array_equal(sw.cpu().numpy(), rs)
    Y = q.qlin_w4a8_forward(Xc, Wq4, sw)
    rows = sample_rows(lin.M, n=N_ROWS, seed=30 + li, must=[0, lin.M - 1])
    ro = oracle.w4a8_forward(X, rq, rs, group=128, rows=rows, want_cg=True)
    # int32 group partials of the first, a middle and the last group, on the sampled rows
    G = lin.K // 128
    for g in sorted({0, G // 2, G - 1}):
        Cg = q.qlin_w4a8_group_i32(Xq, Wq4, g)[rows].cpu().numpy()
        assert np.array_equal(Cg, ro["Cg"][:, :, g]), g
    assert_rows_close(Y, ro, rows=rows, extra=EXTRA_W4A8, what=f"w4a8 2048^2 {lin.name}")


@pytest.mark.parametrize("M,N", [(129, 257), (300, 520), (1, 128)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_w4a8_forward_k12288_ragged(q, M, N, dtype):
    """96 groups per row: ragged tiles at the longest per-group promotion."""
    K = 12288
    g = torch.Generator().manual_seed(M * 3 + N)
    X = torch.randn((M, K), generator=g)
    X[0, 17] = 30.0
    X = X.to(dtype)
    W = (torch.randn((N, K), generator=g) * 0.02)
    W[:, 128 * 40:128 * 41] *= 25.0                     # one group with a much larger scale
    W = W.to(dtype)
    bias = (torch.randn(N, generator=g) * 0.1).to(dtype)
    Wq4, sw = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_INT4_G128)
    rq, rs = oracle.quantize_weight(W, "int4_g128")
    assert np.array_equal(Wq4.cpu().numpy(), rq) and np.array_equal(sw.cpu().numpy(), rs)
    Y = q.qlin_w4a8_forward(X.cuda(), Wq4, sw, bias=bias.cuda())
    ro = oracle.w4a8_forward(X, rq, rs, group=128, bias=bias, want_cg=True)
    Xq, _ = q.qlin_w4a8_prep(X.cuda())
    for gi in (0, 40, 95):
        Cg = q.qlin_w4a8_group_i32(Xq, Wq4, gi).cpu().numpy()
        assert np.array_equal(Cg, ro["Cg"][:, :, gi]), gi
    assert_rows_close(Y, ro, extra=EXTRA_W4A8, what=f"w4a8 {M}x{N}x{K}")
