"""GPU parity of the NVFP4 weight-only linear against the CPU oracle.

The format is a reading of the release format the Darkstar ModelOpt-FP8 page
names (E2M1 codes, one E4M3 scale per 16 weights of a row, one fp32 scale per
tensor; the page gives no layout). The quantiser is compared byte for byte:
packed codes, block scales and the tensor scale. The dequantised weight
exists only in shared memory; one-hot activation rows make every output a
single product s_t * 1 * W_deq[j,k] (exact in fp32: W_deq has at most 6
significant bits), so Y equals bf16(s_t * W_deq)^T, which checks every
code's decode, its block scale and its place in the swizzled tile. General
inputs: normwise per-row error against the oracle, on small shapes in full
and on the text-encoder MLP shapes at full size on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import assert_rows_close, sample_rows

pytestmark = pytest.mark.gpu

EXTRA_NVFP4 = 5e-4   # fp32 accumulation over K in the kernel's order


@pytest.fixture(scope="module")
def q():
    import quantized_w8a8_linear_b200 as q
    torch.cuda.init()
    assert q.qlin_get_device_status(reset=True) == 0
    yield q
    assert q.qlin_get_device_status() == 0


def _weights(N, K, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    W = torch.randn((N, K), generator=g) * 0.02
    if K > 7:
        W[:, 7] *= 40.0                 # a column of large weights: small codes elsewhere in its blocks
    if N > 3:
        W[3] = 0.0                      # a zero row: block scales 0, codes 0
    if N > 5 and K >= 32:
        W[5, 16:32] = 0.0               # one zero block in an otherwise normal row
    return W.to(dtype)


def _quantize(q, W):
    Wq, ws = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_NVFP4)
    N, K = W.shape
    sb, st = q.nvfp4_scales(ws, N, K)
    return Wq, ws, sb, st


@pytest.mark.parametrize("N,K", [(8, 64), (300, 1024), (257, 128), (4096, 12288), (12288, 4096)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_nvfp4_quantiser_bit_exact(q, N, K, dtype):
    W = _weights(N, K, N + K, dtype)
    Wq, ws, sb, st = _quantize(q, W)
    rq, rsb, rst = oracle.quantize_weight_nvfp4(W)
    assert st.item() == rst
    assert np.array_equal(sb.cpu().numpy(), rsb)
    assert np.array_equal(Wq.cpu().numpy(), rq)


@pytest.mark.parametrize("N,K", [(300, 256), (257, 512), (40, 4096)])
def test_nvfp4_dequant_bit_exact_through_one_hot_rows(q, N, K):
    W = _weights(N, K, 3 * N + K)
    Wq, ws, sb, st = _quantize(q, W)
    Y = q.qlin_nvfp4_weight_only_forward(torch.eye(K, dtype=torch.bfloat16, device="cuda"), Wq, ws)
    rq, rsb, rst = oracle.quantize_weight_nvfp4(W)
    b = rq.reshape(N, K // 32, 16)                   # the packed layout, unpacked here
    codes = np.concatenate([b & 0x0F, b >> 4], axis=2).reshape(N, K)
    assert all(oracle.nvfp4_code(rq, K, j, k) == codes[j, k] for j, k in [(0, 0), (N - 1, K - 1), (1, 17)])
    vals = np.array([oracle.e2m1_decode(c) for c in range(16)])[codes]
    scales = torch.from_numpy(rsb.copy()).view(torch.float8_e4m3fn).float().numpy()
    wd = (vals.astype(np.float32) * np.repeat(scales, 16, axis=1)).astype(np.float32)   # exact
    want = torch.from_numpy(np.ascontiguousarray((wd * np.float32(rst)).T)).to(torch.bfloat16).float().numpy()
    got = Y.float().cpu().numpy()
    assert np.array_equal(got, want)


@pytest.mark.parametrize("M,N,K", [(64, 256, 256), (200, 300, 1024), (129, 520, 4096), (7, 264, 12288)])
def test_nvfp4_forward(q, M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    X = torch.randn((M, K), generator=g).to(torch.bfloat16)
    W = _weights(N, K, M * 7 + K)
    bias = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16)
    Wq, ws, sb, st = _quantize(q, W)
    Y = q.qlin_nvfp4_weight_only_forward(X.cuda(), Wq, ws, bias=bias.cuda())
    r = oracle.nvfp4_weight_only_forward(X, Wq.cpu().numpy(), sb.cpu().numpy(), st.item(), bias=bias)
    assert_rows_close(Y, r, extra=EXTRA_NVFP4, what=f"nvfp4 {M}x{N}x{K}")


@pytest.mark.parametrize("li", [0, 1, 2], ids=["gate", "up", "down"])
def test_nvfp4_text_encoder_full_size(q, li):
    wl = workloads.get_workload("te_fp8_weight_only_mlp")
    lin = wl.linears[li]
    X, W, bias = workloads.make_linear(wl, lin, index=li)
    Wq, ws, sb, st = _quantize(q, W)
    Y = q.qlin_nvfp4_weight_only_forward(X.cuda(), Wq, ws)
    rows = sample_rows(lin.M, n=12, seed=li, must=[0, lin.M - 1])
    r = oracle.nvfp4_weight_only_forward(X, Wq.cpu().numpy(), sb.cpu().numpy(), st.item(), rows=rows)
    assert_rows_close(Y, r, rows=rows, extra=EXTRA_NVFP4, what=lin.name)
