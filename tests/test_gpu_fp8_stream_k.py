"""GPU parity of the FP8 GEMM when tiles are cut along K between CTAs
(stream-K, kind::f8f6f4 with fp32 partial sums).

The FP8 linears' definition (Text-Encoder-FP8 page, "Format"; Darkstar
ModelOpt-FP8 page, static per-tensor) fixes the products and the scales, not
the order of the fp32 sum over K, so a cut tile is held to the same oracle
tolerance as a whole one. What the schedule must not change is determinism:
the parties' partials are added in a fixed order, so two runs give the same
bits whatever CTA finishes a tile, and the call clears the scratch's arrival
counters itself (a scratch full of garbage works).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import as_bits, assert_rows_close, sample_rows

pytestmark = pytest.mark.gpu

EXTRA_FP8 = 1e-3


@pytest.fixture(scope="module")
def q():
    import quantized_w8a8_linear_b200 as q
    torch.cuda.init()
    assert q.qlin_get_device_status(reset=True) == 0
    yield q
    q.qlin_set_gemm_schedule(0)
    assert q.qlin_get_device_status() == 0, "a device-side wait timed out"


@pytest.fixture
def schedule(q):
    yield q.qlin_set_gemm_schedule
    q.qlin_set_gemm_schedule(0)


def _x(M, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((M, K), generator=g)
    x[0, 1] = 700.0   # one large row, so per-token scales differ
    return x.to(torch.bfloat16)


def _w(N, K, seed):
    g = torch.Generator().manual_seed(seed + 1000)
    return (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16)


# Forced stream-K (schedule 2) cuts the work down to about one k-block per
# CTA: (300, 520, 512) has 9 tiles of 4 k-blocks (each tile in 4 CTAs);
# (130, 260, 3072) 4 tiles of 24 (each in 24 CTAs); (1000, 1100, 2048) 40 tiles
# of 16 over 148 CTAs (ranges that start and end inside tiles); (512, 4096,
# 12288) is the text-encoder down projection's shape (64 tiles of 96).
CASES = [(300, 520, 512), (130, 260, 3072), (1000, 1100, 2048), (512, 4096, 12288)]


@pytest.mark.parametrize("M,N,K", CASES)
@pytest.mark.parametrize("wmode", ["dynamic", "static"])
def test_fp8_stream_k_matches_oracle_and_is_deterministic(q, schedule, M, N, K, wmode):
    X, W = _x(M, K, M + N), _w(N, K, M + N)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(3)) * 0.1).to(torch.bfloat16)
    Xc = X.cuda()
    if wmode == "dynamic":
        mode, xs = q.QLIN_W_FP8_CHANNEL, None
    else:
        mode = q.QLIN_W_FP8_TENSOR
        xs = q.qlin_calibrate_input_scale(Xc)
    Wq, sw = q.qlin_quantize_weight(W.cuda(), mode)
    codes, s_x = q.qlin_fp8_prep(Xc, xs)
    n = q.qlin_workspace_bytes(q.QLIN_OP_FP8_GEMM, M, N, K)
    ws = torch.full((n,), 0xA5, dtype=torch.uint8, device="cuda")   # garbage counters: the call clears them
    schedule(2)
    Y1 = q.qlin_fp8_gemm(codes, s_x, Wq, sw, mode, torch.bfloat16, x_scale=xs, bias=bias.cuda(), ws=ws)
    Y2 = q.qlin_fp8_gemm(codes, s_x, Wq, sw, mode, torch.bfloat16, x_scale=xs, bias=bias.cuda(), ws=ws)
    torch.cuda.synchronize()
    assert np.array_equal(as_bits(Y1), as_bits(Y2)), "fp32 partials must be added in a fixed order"
    if wmode == "dynamic":
        r = oracle.fp8_forward(X, Wq.cpu().numpy(), as_bits(sw).reshape(-1), x_scale=None, bias=bias)
    else:
        r = oracle.fp8_forward(X, Wq.cpu().numpy(), sw.cpu().numpy(), x_scale=xs.item(), bias=bias)
    assert np.array_equal(codes.cpu().numpy(), r["Xq"])
    assert_rows_close(Y1, r, extra=EXTRA_FP8, what=f"fp8 {wmode} stream-K {M}x{N}x{K}")
    # whole tiles (no scratch) agree with the oracle too; the two schedules
    # add the same products in a different order, so only to that tolerance
    schedule(1)
    Y0 = q.qlin_fp8_gemm(codes, s_x, Wq, sw, mode, torch.bfloat16, x_scale=xs, bias=bias.cuda())
    assert_rows_close(Y0, r, extra=EXTRA_FP8, what=f"fp8 {wmode} whole tiles {M}x{N}x{K}")


@pytest.mark.parametrize("li", [0, 2], ids=["gate", "down"])
def test_fp8_text_encoder_automatic_schedule_full_size(q, li):
    """The te MLP linears at full size through the one-call forward (its
    workspace carries the GEMM scratch), in the automatic schedule the bench
    times; sampled rows against the oracle, and run-to-run determinism."""
    wl = workloads.get_workload("te_fp8_dynamic_mlp")
    lin = wl.linears[li]
    X, W, bias = workloads.make_linear(wl, lin, index=li)
    Xc = X.cuda()
    Wq, sb = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_FP8_CHANNEL)
    Y1 = q.qlin_fp8_forward(Xc, Wq, sb, q.QLIN_W_FP8_CHANNEL)
    Y2 = q.qlin_fp8_forward(Xc, Wq, sb, q.QLIN_W_FP8_CHANNEL)
    assert np.array_equal(as_bits(Y1), as_bits(Y2))
    rows = sample_rows(lin.M, n=12, seed=li, must=[0, lin.M - 1])
    r = oracle.fp8_forward(X, Wq.cpu().numpy(), as_bits(sb).reshape(-1), x_scale=None, rows=rows)
    assert_rows_close(Y1, r, rows=rows, extra=EXTRA_FP8, what=lin.name)
