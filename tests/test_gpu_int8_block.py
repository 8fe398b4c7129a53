"""GPU parity of the block-scaled int8 linear (Qwen-Image-2.1-Text-Encoder-FP8,
"How it was tested": GGUF Q8_0, int8 weight codes with one scale per run of
32 weights of a row) against the CPU oracle.

Bit-exact: the weight codes and block scales, the per-token activation codes
(written as exact fp16 values) and their scales.

Outputs: the kernel applies each weight's block scale before the sum, as an
fp16 product q * s (relative error at most 2^-11 per weight), so it does not
reproduce the oracle's exact int32 block sums, and an output near a rounding
boundary of the output dtype may round the other way: the flat 2e-3 bar
against the oracle's rounded output does not hold for it in general. Each
output row is held to the bound the arithmetic gives instead,
    ||y_gpu - y64|| <= ||halfulp(y64)|| + 2^-11 ||S|| + 1e-6 ||y64||,
S[i,j] = s_x[i] * sum_k |Xq[i,k]| |Wq[j,k]| s_w[j,k/32] (the size of the
terms the dequantisation rounds), and to a relative error of 1e-2 against
the fp64 value.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import sample_rows

pytestmark = pytest.mark.gpu

DEQ_REL = 2.0 ** -11


def assert_rows_within_dequant_bound(y_gpu, r, Wq, s_w, rows=None, what=""):
    """The per-row bound of the module docstring; r: the oracle's result with Xq, s_x, Y64, dt."""
    yg = y_gpu.detach().cpu()
    if rows is not None:
        yg = yg[rows]
    yg = yg.double().numpy()
    assert np.all(np.isfinite(yg)), what
    y64 = r["Y64"]
    rr = np.arange(r["Xq"].shape[0]) if rows is None else np.asarray(rows)
    xa = np.abs(r["Xq"][rr].astype(np.float64)) * r["s_x"][rr].astype(np.float64)[:, None]
    wa = np.abs(Wq.astype(np.float64)) * np.repeat(s_w.astype(np.float64), 32, axis=1)
    S = xa @ wa.T
    sig = 8 if r["dt"] == oracle.BF16 else 11          # significant bits of the output dtype
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.abs(y64)))
    half_ulp = np.where(y64 != 0, np.exp2(e - sig), 0.0)
    d = np.linalg.norm(yg - y64, axis=1)
    bound = np.linalg.norm(half_ulp, axis=1) + DEQ_REL * np.linalg.norm(S, axis=1) + 1e-6 * np.linalg.norm(y64, axis=1)
    bad = np.nonzero(d > bound)[0]
    assert bad.size == 0, f"{what}: rows {bad[:5]} beyond the dequantisation bound ({d[bad[0]]:.3e} > {bound[bad[0]]:.3e})"
    nrm = np.linalg.norm(y64, axis=1)
    rel = np.where(nrm > 0, d / np.where(nrm > 0, nrm, 1.0), d)
    assert rel.max() <= 1e-2, f"{what}: row rel err {rel.max():.3e}"


@pytest.fixture(scope="module")
def q():
    import quantized_w8a8_linear_b200 as q
    torch.cuda.init()
    assert q.qlin_get_device_status(reset=True) == 0
    yield q
    assert q.qlin_get_device_status() == 0


def _w(N, K, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    W = torch.randn((N, K), generator=g) * 0.02
    if N > 3 and K >= 96:
        W[3, 64:96] = 0.0                        # an all-zero block: scale 0, codes 0
        W[2, 40] = 0.5                           # one large weight sets its own block's scale
    return W.to(dtype)


@pytest.mark.parametrize("N,K", [(300, 256), (37, 4096), (33, 32768), (5, 32)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_int8_block_weight_quantisation(q, N, K, dtype):
    W = _w(N, K, N + K, dtype)
    Wq, s = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_INT8_BLOCK32)
    rq, rs = oracle.quantize_weight(W, "int8_block", group=32)
    assert np.array_equal(Wq.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy(), rs)


@pytest.mark.parametrize("M,K", [(64, 128), (333, 3072), (7, 12288)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_int8_block_activation_codes(q, M, K, dtype):
    g = torch.Generator().manual_seed(M + K)
    X = torch.randn((M, K), generator=g)
    X[0, 5] = 40.0
    X = X.to(dtype)
    Xq16, s_x = q.qlin_int8_block_prep(X.cuda())
    r = oracle.int8_outlier_prep(X, float("inf"))    # per-token int8 over all columns
    assert np.array_equal(Xq16.cpu().float().numpy().astype(np.int8), r["Xq"])
    assert np.array_equal(Xq16.cpu().float().numpy(), r["Xq"].astype(np.float32))
    assert np.array_equal(s_x.cpu().numpy(), r["s_x"])


@pytest.mark.parametrize("M,N,K", [(64, 512, 256), (200, 300, 224), (333, 520, 1024), (1, 1, 32),
                                   (257, 129, 64), (130, 4096, 3072), (70, 264, 32768)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_int8_block_forward_ragged(q, M, N, K, dtype):
    g = torch.Generator().manual_seed(M * 7 + N)
    X = torch.randn((M, K), generator=g)
    X[0, K // 2] = 25.0
    X = X.to(dtype)
    W = _w(N, K, M + N + K, dtype)
    bias = (torch.randn(N, generator=g) * 0.1).to(dtype)
    Wq, s = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_INT8_BLOCK32)
    Y = q.qlin_int8_block_forward(X.cuda(), Wq, s, bias=bias.cuda())
    r = oracle.int8_block_forward(X, Wq.cpu().numpy(), s.cpu().numpy(), block=32, bias=bias)
    assert Y.dtype == dtype
    assert_rows_within_dequant_bound(Y, r, Wq.cpu().numpy(), s.cpu().numpy(), what=f"int8 block {M}x{N}x{K}")


@pytest.mark.parametrize("li", [0, 2])
def test_int8_block_text_encoder_full_size(q, li):
    """The text-encoder MLP gate and down projections at full size (the page's
    Q8_0 comparison is on the text encoder), outputs on 512 rows."""
    wl = workloads.get_workload("te_fp8_dynamic_mlp")
    lin = wl.linears[li]
    X, W, bias = workloads.make_linear(wl, lin, index=li)
    Wq, s = q.qlin_quantize_weight(W.cuda(), q.QLIN_W_INT8_BLOCK32)
    rq, rs = oracle.quantize_weight(W, "int8_block", group=32)
    assert np.array_equal(Wq.cpu().numpy(), rq) and np.array_equal(s.cpu().numpy(), rs)
    Y = q.qlin_int8_block_forward(X.cuda(), Wq, s, bias=bias.cuda())
    rows = sample_rows(lin.M, n=512, seed=li, must=[0, 5])
    r = oracle.int8_block_forward(X, rq, rs, block=32, bias=bias, rows=rows)
    assert_rows_within_dequant_bound(Y, r, rq, rs, rows=rows, what=f"int8 block {lin.name}")
