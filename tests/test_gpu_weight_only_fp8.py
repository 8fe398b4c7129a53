"""GPU parity of the weight-only FP8 linear (Qwen-Image-2.1-Text-Encoder-FP8,
"Format": E4M3 weights with bf16 [out,1] scales consumed as
weight.to(bf16) * weight_scale, bf16 activations) against the CPU oracle.

The dequantised weight W_deq = bf16(decode(Wq) * s_w) exists only in shared
memory, so it is checked through the output: with one-hot activation rows
every output is a single product 1 * W_deq[j,k], which the fp32 accumulator
and the bf16 output hold exactly, so Y equals W_deq^T (bit for bit, except
that a -0 weight comes out as +0). Outputs of
general inputs: normwise per-row error <= 2e-3 against the oracle's rounded
output and within rounding plus fp32 accumulation of its fp64 value.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import as_bits, assert_rows_close, sample_rows

pytestmark = pytest.mark.gpu

EXTRA_WO8 = 5e-4


@pytest.fixture(scope="module")
def q():
    import quantized_w8a8_linear_b200 as q
    torch.cuda.init()
    assert q.qlin_get_device_status(reset=True) == 0
    yield q
    assert q.qlin_get_device_status() == 0


def _weights(q, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn((N, K), generator=g) * 0.02)
    if K > 7:
        W[:, 7] *= 40.0                              # a column of large weights
    if N > 3:
        W[3] = 0.0                                   # a zero row: scale 0, W_deq 0
    W = W.to(torch.bfloat16)
    Wq, sb = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_FP8_CHANNEL)
    return W, Wq, sb


@pytest.mark.parametrize("N,K", [(300, 256), (257, 512), (40, 4096)])
def test_weight_only_dequant_bit_exact_through_one_hot_rows(q, N, K):
    W, Wq, sb = _weights(q, N, K, N + K)
    Y = q.qlin_fp8_weight_only_forward(torch.eye(K, dtype=torch.bfloat16, device="cuda"), Wq, sb)
    ref = oracle.fp8_weight_only_dequant(Wq.cpu().numpy(), as_bits(sb).reshape(-1))   # [N,K] bf16 bits
    # values, not bit patterns: a negative weight that rounds to the e4m3 zero
    # (code 0x80) dequantises to -0, and the accumulator's 1 * (-0) + 0 + ... is +0
    got = Y.float().cpu().numpy()
    want = oracle.bits_to_torch(np.ascontiguousarray(ref.T), oracle.BF16).float().numpy()
    assert np.array_equal(got, want)
    nz = want != 0
    assert np.array_equal(as_bits(Y)[nz], np.ascontiguousarray(ref.T)[nz])


@pytest.mark.parametrize("M,N,K", [(64, 512, 256), (200, 300, 208), (333, 520, 1024), (1, 1, 16),
                                   (257, 129, 64), (130, 4096, 3072), (70, 264, 32768)])
def test_weight_only_forward_ragged(q, M, N, K):
    W, Wq, sb = _weights(q, N, K, M + N + K)
    g = torch.Generator().manual_seed(M)
    X = torch.randn((M, K), generator=g)
    if M > 5 and K > 2276:
        X[5, 2276] = 9000.0                          # a massive activation, unquantised here
    X = X.to(torch.bfloat16)
    bias = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16)
    Y = q.qlin_fp8_weight_only_forward(X.cuda(), Wq, sb, bias=bias.cuda())
    r = oracle.fp8_weight_only_forward(X, Wq.cpu().numpy(), as_bits(sb).reshape(-1), bias=bias)
    assert_rows_close(Y, r, extra=EXTRA_WO8, what=f"weight-only fp8 {M}x{N}x{K}")


def test_weight_only_rejects_fp16_activations(q):
    _, Wq, sb = _weights(q, 64, 128, 1)
    X = torch.randn((8, 128)).to(torch.float16).cuda()
    with pytest.raises(q.QlinError) as e:
        q.qlin_fp8_weight_only_forward(X, Wq, sb)
    assert e.value.status == q.QLIN_ERR_UNSUPPORTED


@pytest.mark.parametrize("li", [0, 2])
def test_weight_only_text_encoder_full_size(q, li):
    """The text-encoder MLP gate (K = 4096) and down (K = 12288) projections
    at full size, with the page's massive activations, outputs on 512 rows."""
    wl = workloads.get_workload("te_fp8_dynamic_mlp")
    lin = wl.linears[li]
    X, W, bias = workloads.make_linear(wl, lin, index=li)
    Wq, sb = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_FP8_CHANNEL)
    rq, rs = oracle.quantize_weight(W, "fp8_channel")
    assert np.array_equal(Wq.cpu().numpy(), rq) and np.array_equal(as_bits(sb).reshape(-1), rs)
    Y = q.qlin_fp8_weight_only_forward(X.cuda(), Wq, sb, bias=bias.cuda())
    rows = sample_rows(lin.M, n=512, seed=li, must=[0, 5])
    r = oracle.fp8_weight_only_forward(X, rq, rs, bias=bias, rows=rows)
    assert_rows_close(Y, r, rows=rows, extra=EXTRA_WO8, what=f"weight-only {lin.name}")
