"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bit-exact: int8 / E4M3 codes, scales, outlier sets and X_O copies, W_O,
int32 accumulators and all weight-quantisation outputs. Floating-point
outputs: normwise relative error per output row <= 2e-3 against the oracle's
output in the same dtype, and no farther from the oracle's fp64 value than
correct rounding plus the kernels' fp32 arithmetic (tests/_parity.py).

Sizes: the tiny workload and ragged shapes spanning several 128x256 tiles
and partial tiles run whole; the 1024^2 DiT and text-encoder shapes run at
full size in the launch configuration the bench times, with the oracle on a
sample of rows (the outlier set and row scales are still compared in full).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import as_bits, assert_rows_close, sample_rows

# FP8: the tensor cores accumulate e4m3 products in fp32 in their own order
EXTRA_FP8 = 1e-3

pytestmark = pytest.mark.gpu

THR = 6.0


@pytest.fixture(scope="module")
def q():
    import quantized_w8a8_linear_b200 as q
    torch.cuda.init()
    assert q.qlin_get_device_status(reset=True) == 0
    yield q
    assert q.qlin_get_device_status() == 0, "a device-side wait timed out"


def dev(t):
    return t.cuda()


def rand_x(M, K, seed, dtype=torch.bfloat16, outliers=()):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((M, K), generator=g)
    for (i, k, v) in outliers:
        if i < M and k < K:
            x[i, k] = v
    return x.to(dtype)


def rand_w(N, K, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed + 1000)
    return (torch.randn((N, K), generator=g) * 0.02).to(dtype)


# ---------------------------------------------------------------------------
# E4M3 / int8 code parity on values that hit every rounding boundary
# ---------------------------------------------------------------------------

def test_e4m3_codes_every_boundary(q):
    # grid values, midpoints and their fp32 neighbours, scaled so that the
    # static scale is 1.0: X * (1/1) hits every tie of the e4m3 grid.
    pos = sorted(oracle.e4m3_decode(c) for c in range(0x7F)) + [480.0]
    pts = []
    for a, b in zip(pos[:-1], pos[1:]):
        m = np.float32((a + b) / 2)
        pts += [a, m, np.nextafter(m, np.float32(1e9)), np.nextafter(m, np.float32(-1e9))]
    v = np.array(pts + [600.0, 1e5, 0.0, -0.0, 2.0 ** -11], np.float32)
    v = np.concatenate([v, -v])
    # bf16 keeps only some of these exactly; use fp16 as well as bf16
    for dtype in (torch.float16, torch.bfloat16):
        x = torch.from_numpy(v).to(dtype)
        n = (x.numel() + 15) // 16 * 16
        X = torch.zeros((1, n), dtype=dtype)
        X[0, : x.numel()] = x
        one = torch.ones(1, dtype=torch.float32).cuda()
        codes, _ = q.qlin_fp8_prep(dev(X), one)
        ref = oracle.fp8_static_prep(X, 1.0)
        assert np.array_equal(codes.cpu().numpy(), ref), dtype


def test_e4m3_device_conversion_all_finite_fp32(q):
    """The conversion every FP8 kernel uses, on all 2^32 fp32 bit patterns,
    against the oracle's encoder. Non-finite inputs are outside the reading
    (the pages leave them unspecified), so NaN and infinity are skipped."""
    chunk = 1 << 26
    for lo in range(0, 1 << 32, chunk):
        bits = torch.arange(lo, lo + chunk, dtype=torch.int64, device="cuda").to(torch.int32)
        codes = q.qlin_e4m3_encode_f32(bits.view(torch.float32)).cpu().numpy()
        ref = oracle.e4m3_encode_range(lo, chunk)
        u = np.arange(lo, lo + chunk, dtype=np.uint64)
        finite = ((u >> 23) & 0xFF) != 0xFF
        assert np.array_equal(codes[finite], ref[finite]), hex(lo)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_all_16bit_values_int8_and_e4m3(q, dtype):
    # every finite 16-bit pattern, one row per block of 2048, dynamic scales
    bits = torch.arange(0, 65536, dtype=torch.int32).to(torch.int16).view(dtype).float()
    bits = bits[torch.isfinite(bits)]
    bits = bits[: (bits.numel() // 2048) * 2048]
    X = bits.reshape(-1, 2048).to(dtype)
    Xc = dev(X)
    codes, s_x = q.qlin_fp8_prep(Xc, None)
    ref_codes, ref_s = oracle.fp8_dynamic_prep(X)
    assert np.array_equal(s_x.cpu().numpy(), ref_s)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    p = q.qlin_int8_prep(Xc, 0.0)
    r = oracle.int8_outlier_prep(X, 0.0)
    assert np.array_equal(p["s_x"].cpu().numpy(), r["s_x"])
    assert np.array_equal(p["Xq"].cpu().numpy(), r["Xq"])


# ---------------------------------------------------------------------------
# weight quantisation (offline step)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(512, 256), (300, 208), (37, 4096), (33, 32768)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_quantize_weight_parity(q, N, K, dtype):
    W = rand_w(N, K, N + K, dtype)
    W[3, 5] = 0.0
    if N > 10:
        W[7] = 0.0                                        # an all-zero row: scale 0, codes 0
    Wc = dev(W)
    for mode, name in ((q.QLIN_W_INT8_ROW, "int8_row"), (q.QLIN_W_FP8_TENSOR, "fp8_tensor"),
                       (q.QLIN_W_FP8_CHANNEL, "fp8_channel")):
        Wq, s = q.qlin_quantize_weight(Wc, mode)
        rq, rs = oracle.quantize_weight(W, name)
        assert np.array_equal(Wq.cpu().numpy().view(rq.dtype), rq), name
        got_s = s.cpu()
        if name == "fp8_channel":
            got_s = got_s.view(torch.int16).numpy().view(np.uint16).reshape(-1)
        else:
            got_s = got_s.numpy().reshape(-1)
        assert np.array_equal(got_s, rs.reshape(-1)), name
    if K % 128 == 0:
        Wq, s = q.qlin_quantize_weight(Wc, q.QLIN_W_INT4_G128)
        rq, rs = oracle.quantize_weight(W, "int4_g128")
        assert np.array_equal(Wq.cpu().numpy(), rq)
        assert np.array_equal(s.cpu().numpy(), rs)


def test_calibrate_input_scale(q):
    wl = workloads.get_workload("dit1024_fp8_static_qkv")
    lin = wl.linears[0]
    Xc = workloads.make_calibration(wl, lin, M=512)
    s = q.qlin_calibrate_input_scale(dev(Xc))
    assert s.item() == oracle.absmax_scale(Xc, 448.0)


# ---------------------------------------------------------------------------
# LLM.int8 activation prep: outlier set, codes, scales, X_O, W_O
# ---------------------------------------------------------------------------

PREP_CASES = [
    ("tiny", 64, 256, [(3, 17, 9.5), (9, 200, -11.0)]),
    ("ragged", 333, 208, [(0, 5, 6.5), (332, 207, -7.0), (100, 5, 1.0)]),
    ("boundary", 40, 64, [(0, 3, 6.0), (1, 5, 6.03125), (2, 7, -6.03125), (3, 9, -6.0)]),
    ("many", 130, 1024, [(i % 130, (i * 37) % 1024, 7.0 + i) for i in range(150)]),
    ("none", 77, 512, []),
    # rows 1 and 2 have their largest sub-threshold value in outlier column 5
    ("recompute", 64, 128, [(0, 5, 9.0), (1, 5, 5.9), (2, 5, -5.95), (3, 9, 6.0), (4, 9, 3.5)]),
    ("wide", 96, 12288, [(0, 17, 40.0), (1, 17, 5.5), (50, 9000, -7.0), (95, 12287, 6.5)]),
    # the largest K the library takes (16 vectors per lane, rows of 64 KB)
    ("max_k", 40, 32768, [(0, 17, 40.0), (39, 32767, -6.5), (20, 16384, 7.0), (21, 16384, 5.0)]),
]


@pytest.mark.parametrize("name,M,K,outl", PREP_CASES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_int8_prep_parity(q, name, M, K, outl, dtype):
    X = rand_x(M, K, M * K, dtype, outl)
    p = q.qlin_int8_prep(dev(X), THR)
    r = oracle.int8_outlier_prep(X, THR)
    n = int(p["count"].item())
    assert n == r["count"]
    assert np.array_equal(p["O"].cpu().numpy()[:n], r["O"])
    flags = p["flags"].cpu().numpy().view(np.uint32)
    bits = np.unpackbits(flags.view(np.uint8), bitorder="little")[:K]
    assert np.array_equal(bits, r["is_outlier"])
    assert np.array_equal(p["s_x"].cpu().numpy(), r["s_x"])
    assert np.array_equal(p["Xq"].cpu().numpy(), r["Xq"])
    xo = as_bits(p["X_O"])
    assert np.array_equal(xo[:, :n], r["X_O"])
    pad = 16 if 1 <= n <= 16 else (n + 7) // 8 * 8   # zero padding the header documents
    assert np.all(xo[:, n:pad] == 0)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_outlier_weights_parity(q, dtype):
    N, K = 300, 512
    W = rand_w(N, K, 5, dtype)
    X = rand_x(16, K, 6, dtype, [(1, 0, 9.0), (2, 100, -8.0), (3, 511, 50.0), (4, 101, 7.0)])
    Wq, s = q.qlin_quantize_weight(dev(W), q.QLIN_W_INT8_ROW)
    p = q.qlin_int8_prep(dev(X), THR)
    W_O = q.qlin_outlier_weights(Wq, s, p["O"], p["count"], dtype)
    r = oracle.int8_outlier_prep(X, THR)
    ref = oracle.outlier_weights(Wq.cpu().numpy(), s.cpu().numpy(), r["O"], r["dt"])
    n = r["count"]
    got = as_bits(W_O)
    assert np.array_equal(got[:, :n], ref)
    assert np.all(got[:, n:(n + 7) // 8 * 8] == 0)


# ---------------------------------------------------------------------------
# int8 tcgen05 GEMM: int32 accumulators bit-exact
# ---------------------------------------------------------------------------

# (2500, 600, 128): 20 m-blocks in one round-robin order (operands of 0.4 MB:
# no tile bands); (2200, 2700, 12288): operands of 60 MB, so the tiles go in
# bands of 16 m-blocks, a band of 16 and a narrower last band of 2
GEMM_SHAPES = [(64, 512, 256), (128, 256, 128), (200, 300, 208), (1, 1, 16), (129, 257, 16),
               (333, 600, 1024), (512, 768, 3072), (16, 48, 12288), (2500, 600, 128), (2200, 2700, 12288)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_int8_gemm_i32_exact(q, M, N, K):
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    A = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    B = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    C = q.qlin_int8_gemm_i32(dev(A), dev(B)).cpu().numpy().astype(np.int64)
    # |C| <= K * 127^2 < 2^31: the fp64 products and sums are exact
    ref = (A.numpy().astype(np.float64) @ B.numpy().astype(np.float64).T).astype(np.int64)
    assert np.array_equal(C, ref)


@pytest.mark.parametrize("M,N,K,outl", [
    (200, 300, 208, []),                                                     # no outlier
    (200, 300, 208, [(5, 7, 8.0), (199, 200, -30.0), (6, 7, 5.0)]),          # <= 8
    (300, 520, 512, [(i * 3, 40 * i + 1, 6.5 + i) for i in range(12)]),      # 9..16
    (300, 520, 512, [(i * 3, 16 * i + 3, -6.5 - i) for i in range(32)]),     # 17..32
    (300, 520, 512, [(i * 3, 15 * i + 3, -6.5 - i) for i in range(33)]),     # > 32: global path
    (130, 260, 3072, [(0, 2, 9.0), (1, 2, 5.99), (2, 3071, -6.01), (3, 1500, 5.5)]),
])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_int8_outlier_gemm_int32_exact(q, M, N, K, outl, dtype):
    """The fused path's int32 accumulator (the MMA sums every column, the
    epilogue takes the outlier columns' products back out) equals the
    oracle's int8 part, sum over k not in O of Xq Wq, exactly."""
    X = rand_x(M, K, M + 5 * N, dtype, outl)
    W = rand_w(N, K, M + 5 * N, dtype)
    Wq, s_w = q.qlin_quantize_weight(dev(W), q.QLIN_W_INT8_ROW)
    ws = q.workspace(q.QLIN_OP_INT8_OUTLIER, M, N, K, "cuda")
    q.qlin_int8_outlier_prepare(dev(X), Wq, s_w, THR, ws)
    C = q.qlin_int8_outlier_gemm_i32(M, K, Wq, ws).cpu().numpy().astype(np.int64)
    r = oracle.int8_outlier_prep(X, THR)
    ref = r["Xq"].astype(np.int64) @ Wq.cpu().numpy().astype(np.int64).T
    assert np.array_equal(C, ref)


# Stream-K: the int32 accumulator of a tile cut between CTAs is the sum of
# their partials, so it stays exact under every schedule. Schedule 2 cuts the
# work down to one k-block per CTA: (300, 520, 512) has 9 tiles of 4 k-blocks
# (each tile in 4 CTAs), (130, 260, 3072) 4 tiles of 24 (each in 24 CTAs),
# (1000, 1100, 2048) 40 tiles of 16 over 148 CTAs (ranges of 4-5 k-blocks
# that start and end inside tiles); (2048, 5120, 256) has 320 tiles, more
# than two waves: the first 148 go whole, the other 172 are cut into ranges.
SK_CASES = [
    (300, 520, 512, []),
    (300, 520, 512, [(i * 3, 40 * i + 1, 6.5 + i) for i in range(12)]),
    (300, 520, 512, [(i * 3, 16 * i + 3, -6.5 - i) for i in range(32)]),
    (300, 520, 512, [(i * 3, 15 * i + 3, -6.5 - i) for i in range(33)]),
    (130, 260, 3072, [(0, 2, 9.0), (1, 2, 5.99), (2, 3071, -6.01), (3, 1500, 5.5)]),
    (1000, 1100, 2048, [(i * 7, (i * 131) % 2048, 7.0 + i) for i in range(20)]),
    (2048, 5120, 256, [(i * 50, (i * 37) % 256, -7.0 - i) for i in range(10)]),
]


@pytest.fixture
def schedule(q):
    yield q.qlin_set_gemm_schedule
    q.qlin_set_gemm_schedule(0)


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("M,N,K,outl", SK_CASES)
def test_int8_outlier_gemm_int32_exact_any_schedule(q, schedule, mode, M, N, K, outl):
    X = rand_x(M, K, M + 5 * N, torch.bfloat16, outl)
    W = rand_w(N, K, M + 5 * N)
    Wq, s_w = q.qlin_quantize_weight(dev(W), q.QLIN_W_INT8_ROW)
    ws = q.workspace(q.QLIN_OP_INT8_OUTLIER, M, N, K, "cuda")
    schedule(mode)
    q.qlin_int8_outlier_prepare(dev(X), Wq, s_w, THR, ws)
    C1 = q.qlin_int8_outlier_gemm_i32(M, K, Wq, ws).cpu().numpy().astype(np.int64)
    # a second launch on the same workspace: the arrival counters were left at zero
    C2 = q.qlin_int8_outlier_gemm_i32(M, K, Wq, ws).cpu().numpy().astype(np.int64)
    r = oracle.int8_outlier_prep(X, THR)
    # |sum| < 2^31, so the float64 product is exact
    ref = (r["Xq"].astype(np.float64) @ Wq.cpu().numpy().astype(np.float64).T).astype(np.int64)
    assert np.array_equal(C1, ref)
    assert np.array_equal(C2, ref)


@pytest.mark.parametrize("M,N,K,outl", SK_CASES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_int8_forward_stream_k(q, schedule, M, N, K, outl, dtype):
    X = rand_x(M, K, M + N, dtype, outl)
    W = rand_w(N, K, M + N, dtype)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(2)) * 0.1).to(dtype)
    schedule(2)
    Y, r = run_int8_forward(q, X, W, bias)
    assert_rows_close(Y, r, what=f"stream-K {M}x{N}x{K}")
    if len(outl) == 0 or len(outl) > 16:
        # same per-element arithmetic as whole 128 x 256 tiles: equal bit for bit
        schedule(1)
        Y1, _ = run_int8_forward(q, X, W, bias)
        assert np.array_equal(as_bits(Y), as_bits(Y1))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_int8_forward_split_k_automatic(q, dtype):
    """One 128 x 256 tile over K = 16384: the automatic schedule cuts its 128
    k-blocks over 16 CTAs (stream-K as split-K)."""
    M, N, K = 128, 256, 16384
    X = rand_x(M, K, 77, dtype, [(3, 100, 9.0), (90, 16000, -7.5)])
    W = rand_w(N, K, 77, dtype)
    Y, r = run_int8_forward(q, X, W)
    assert_rows_close(Y, r, what="split-K")


def test_int8_gemm_i32_extremes(q):
    # every code at +-127 at K = 12288: |C| = 12288 * 127^2 = 198,193,152
    K = 12288
    A = torch.full((130, K), 127, dtype=torch.int8)
    A[1] = -127
    B = torch.full((260, K), 127, dtype=torch.int8)
    B[5] = -127
    C = q.qlin_int8_gemm_i32(dev(A), dev(B)).cpu()
    assert C[0, 0].item() == 198193152 and C[1, 0].item() == -198193152 and C[1, 5].item() == 198193152


# ---------------------------------------------------------------------------
# LLM.int8 forward
# ---------------------------------------------------------------------------

def run_int8_forward(q, X, W, bias=None, thr=THR, rows=None):
    Wq, s_w = q.qlin_quantize_weight(dev(W), q.QLIN_W_INT8_ROW)
    Y = q.qlin_int8_outlier_forward(dev(X), Wq, s_w, thr, bias=None if bias is None else dev(bias))
    r = oracle.int8_outlier_forward(X, Wq.cpu().numpy(), s_w.cpu().numpy(), thr, bias=bias, rows=rows)
    Yc = Y.cpu() if rows is None else Y.cpu()[rows]
    return Yc, r


def test_int8_forward_tiny_workload(q):
    wl = workloads.get_workload("tiny_int8")
    X, W, bias = workloads.make_linear(wl, wl.linears[0])
    Y, r = run_int8_forward(q, X, W, bias)
    assert Y.dtype == torch.float16
    assert_rows_close(Y, r, what="tiny")


@pytest.mark.parametrize("M,N,K,outl", [
    (200, 300, 208, [(5, 7, 8.0), (199, 200, -30.0)]),
    (333, 520, 1024, [(i, (i * 13) % 1024, 9.0) for i in range(0, 333, 7)]),
    (1, 1, 16, [(0, 3, 7.0)]),
    (257, 129, 64, []),
    (300, 520, 512, [(i * 3, 40 * i + 1, 6.5 + i) for i in range(12)]),        # 9..16 outliers
    (300, 520, 512, [(i * 3, 16 * i + 3, -6.5 - i) for i in range(30)]),       # 17..32 outliers
    (300, 520, 512, [(i * 3, 16 * i + 3, -6.5 - i) for i in range(32)]),       # exactly 32
    (300, 520, 512, [(i * 3, 15 * i + 3, -6.5 - i) for i in range(33)]),       # 33: global path
    (70, 264, 32768, [(0, 5, 9.0), (69, 32767, -8.0), (35, 20000, 6.5)]),      # the largest K
])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_int8_forward_ragged(q, M, N, K, outl, dtype):
    X = rand_x(M, K, M + N, dtype, outl)
    W = rand_w(N, K, M + N, dtype)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(1)) * 0.1).to(dtype)
    Y, r = run_int8_forward(q, X, W, bias)
    assert_rows_close(Y, r, what=f"{M}x{N}x{K}")


def test_int8_forward_all_outliers(q):
    M, N, K = 70, 300, 256
    X = rand_x(M, K, 3).float()
    X[M - 1, :] = 8.0
    X = X.to(torch.bfloat16)
    W = rand_w(N, K, 3)
    Y, r = run_int8_forward(q, X, W)
    assert_rows_close(Y, r, what="all outliers")


@pytest.mark.parametrize("thr", [float("inf"), 0.0])
def test_int8_forward_decomposition_off(q, thr):
    M, N, K = 130, 260, 512
    X = rand_x(M, K, 4, outliers=[(3, 3, 40.0)])
    W = rand_w(N, K, 4)
    Y, r = run_int8_forward(q, X, W, thr=thr)
    assert_rows_close(Y, r, what="no decomposition")


def test_int8_forward_zero_rows(q):
    M, N, K = 50, 64, 128
    X = rand_x(M, K, 8).float()
    X[3] = 0.0
    X[4, :] = 0.0
    X[4, 10] = 12.0                     # only an outlier in this row: its int8 scale is 0
    X = X.to(torch.bfloat16)
    W = rand_w(N, K, 8)
    Y, r = run_int8_forward(q, X, W)
    assert_rows_close(Y, r, what="zero rows")
    assert torch.all(Y[3] == 0)


def test_int8_forward_empty(q):
    X = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros((32, 64), dtype=torch.int8, device="cuda")
    s = torch.ones(32, device="cuda")
    Y = q.qlin_int8_outlier_forward(X, Wq, s)
    assert Y.shape == (0, 32)


@pytest.mark.parametrize("li", [0, 1])
def test_int8_forward_dit1024_full_size(q, li):
    """1024^2 DiT MLP up (li=0) and down (li=1) projections, full size,
    prep compared in full and the output on a sample of rows."""
    wl = workloads.get_workload("dit1024_int8_mlp")
    lin = wl.linears[li]
    X, W, bias = workloads.make_linear(wl, lin, index=li)
    Xc, Wc = dev(X), dev(W)
    p = q.qlin_int8_prep(Xc, THR)
    r = oracle.int8_outlier_prep(X, THR)
    n = int(p["count"].item())
    assert n == r["count"] and n > 0
    assert np.array_equal(p["O"].cpu().numpy()[:n], r["O"])
    assert np.array_equal(p["s_x"].cpu().numpy(), r["s_x"])
    assert np.array_equal(p["Xq"].cpu().numpy(), r["Xq"])
    Wq, s_w = q.qlin_quantize_weight(Wc, q.QLIN_W_INT8_ROW)
    rq, rs = oracle.quantize_weight(W, "int8_row")
    assert np.array_equal(Wq.cpu().numpy(), rq) and np.array_equal(s_w.cpu().numpy(), rs)
    Y = q.qlin_int8_outlier_forward(Xc, Wq, s_w, THR)
    C = q.qlin_int8_gemm_i32(p["Xq"], Wq)
    rows = sample_rows(lin.M, n=512, seed=li, must=[255, 256])
    ro = oracle.int8_outlier_forward(X, rq, rs, THR, rows=rows)
    assert np.array_equal(C.cpu().numpy()[rows], ro["C"])
    assert_rows_close(Y, ro, rows=rows, what=lin.name)


# ---------------------------------------------------------------------------
# FP8 forward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(64, 512, 256), (200, 300, 208), (333, 520, 1024)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_fp8_static_forward(q, M, N, K, dtype):
    X = rand_x(M, K, M, dtype, [(1, 2, 30.0)])
    Xcal = rand_x(M, K, M + 1, dtype)
    W = rand_w(N, K, M, dtype)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(2)) * 0.1).to(dtype)
    Wq, ws = q.qlin_quantize_weight(dev(W), q.QLIN_W_FP8_TENSOR)
    xs = q.qlin_calibrate_input_scale(dev(Xcal))
    Y = q.qlin_fp8_forward(dev(X), Wq, ws, q.QLIN_W_FP8_TENSOR, x_scale=xs, bias=dev(bias))
    codes, _ = q.qlin_fp8_prep(dev(X), xs)
    r = oracle.fp8_forward(X, Wq.cpu().numpy(), ws.cpu().numpy(), x_scale=xs.item(), bias=bias)
    assert np.array_equal(codes.cpu().numpy(), r["Xq"])
    assert_rows_close(Y, r, extra=EXTRA_FP8, what="fp8 static")


@pytest.mark.parametrize("M,N,K", [(64, 512, 256), (200, 300, 208), (130, 4096, 12288), (70, 264, 32768)])
def test_fp8_dynamic_forward(q, M, N, K):
    X = rand_x(M, K, M + 5, torch.bfloat16, [(0, 7, 12992.0), (5, 7, 9024.0)])
    W = rand_w(N, K, M + 5)
    Wq, sb = q.qlin_quantize_weight(dev(W), q.QLIN_W_FP8_CHANNEL)
    Y = q.qlin_fp8_forward(dev(X), Wq, sb, q.QLIN_W_FP8_CHANNEL)
    codes, s_x = q.qlin_fp8_prep(dev(X), None)
    r = oracle.fp8_forward(X, Wq.cpu().numpy(), as_bits(sb).reshape(-1), x_scale=None)
    assert np.array_equal(codes.cpu().numpy(), r["Xq"])
    assert np.array_equal(s_x.cpu().numpy(), r["s_x"])
    assert_rows_close(Y, r, extra=EXTRA_FP8, what="fp8 dynamic")


def test_fp8_static_dit1024_qkv_full_size(q):
    wl = workloads.get_workload("dit1024_fp8_static_qkv")
    lin = wl.linears[0]
    X, W, bias = workloads.make_linear(wl, lin)
    Xcal = workloads.make_calibration(wl, lin)
    Xc = dev(X)
    Wq, ws = q.qlin_quantize_weight(dev(W), q.QLIN_W_FP8_TENSOR)
    xs = q.qlin_calibrate_input_scale(dev(Xcal))
    assert xs.item() == oracle.absmax_scale(Xcal, 448.0)
    codes, _ = q.qlin_fp8_prep(Xc, xs)
    assert np.array_equal(codes.cpu().numpy(), oracle.fp8_static_prep(X, xs.item()))
    Y = q.qlin_fp8_forward(Xc, Wq, ws, q.QLIN_W_FP8_TENSOR, x_scale=xs)
    rows = sample_rows(lin.M, n=12, seed=3)
    r = oracle.fp8_forward(X, Wq.cpu().numpy(), ws.cpu().numpy(), x_scale=xs.item(), rows=rows)
    assert_rows_close(Y, r, rows=rows, extra=EXTRA_FP8, what="qkv")


@pytest.mark.parametrize("li", [0, 2])
def test_fp8_dynamic_text_encoder_full_size(q, li):
    wl = workloads.get_workload("te_fp8_dynamic_mlp")
    lin = wl.linears[li]
    X, W, bias = workloads.make_linear(wl, lin, index=li)
    Xc = dev(X)
    Wq, sb = q.qlin_quantize_weight(dev(W), q.QLIN_W_FP8_CHANNEL)
    rq, rs = oracle.quantize_weight(W, "fp8_channel")
    assert np.array_equal(Wq.cpu().numpy(), rq) and np.array_equal(as_bits(sb).reshape(-1), rs)
    codes, s_x = q.qlin_fp8_prep(Xc, None)
    rc, rsx = oracle.fp8_dynamic_prep(X)
    assert np.array_equal(codes.cpu().numpy(), rc) and np.array_equal(s_x.cpu().numpy(), rsx)
    Y = q.qlin_fp8_forward(Xc, Wq, sb, q.QLIN_W_FP8_CHANNEL)
    rows = sample_rows(lin.M, n=12, seed=li, must=[0, 5])
    r = oracle.fp8_forward(X, rq, rs, x_scale=None, rows=rows)
    assert_rows_close(Y, r, rows=rows, extra=EXTRA_FP8, what=lin.name)


# ---------------------------------------------------------------------------
# W4A8: int4 per-group-128 weights, per-token int8 activations
# ---------------------------------------------------------------------------

def _unpack_int4(packed, K):
    """int4 codes [N,K] from the packed [N,K/2] bytes: byte b of each 16-byte
    block holds element b of the block's 32 in its low nibble, b + 16 in its
    high nibble, two's complement."""
    b = packed.reshape(packed.shape[0], K // 32, 16)
    nib = np.concatenate([b & 0x0F, b >> 4], axis=2).reshape(packed.shape[0], K).astype(np.int64)
    return np.where(nib >= 8, nib - 16, nib)


@pytest.mark.parametrize("M,K", [(64, 128), (129, 1024), (333, 3072), (7, 12288)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_w4a8_prep_parity(q, M, K, dtype):
    """W4A8 activations: per-token int8 with no outlier split, i.e. the
    LLM.int8 prep with the decomposition off."""
    X = rand_x(M, K, 3 * M + K, dtype, [(0, 5, 40.0), (M - 1, K - 1, -9.0)])
    Xq, s_x = q.qlin_w4a8_prep(dev(X))
    r = oracle.int8_outlier_prep(X, float("inf"))
    assert r["count"] == 0
    assert np.array_equal(Xq.cpu().numpy(), r["Xq"])
    assert np.array_equal(s_x.cpu().numpy(), r["s_x"])


@pytest.mark.parametrize("M,N,K", [(64, 128, 128), (200, 300, 256), (129, 257, 1024), (333, 520, 3072)])
def test_w4a8_group_int32_exact(q, M, N, K):
    X = rand_x(M, K, M + K)
    W = rand_w(N, K, N + K)
    Wq4, sw = q.qlin_quantize_weight(dev(W), q.QLIN_W_INT4_G128)
    p = q.qlin_int8_prep(dev(X), 0.0)
    Xq = p["Xq"]
    u = _unpack_int4(Wq4.cpu().numpy(), K)
    xq = Xq.cpu().numpy().astype(np.int64)
    for g in sorted({0, K // 128 - 1, (K // 128) // 2}):
        C = q.qlin_w4a8_group_i32(Xq, Wq4, g).cpu().numpy().astype(np.int64)
        sl = slice(g * 128, (g + 1) * 128)
        assert np.array_equal(C, xq[:, sl] @ u[:, sl].T), g


@pytest.mark.parametrize("M,N,K", [(64, 128, 128), (200, 300, 256), (129, 257, 1024), (333, 520, 3072)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_w4a8_forward(q, M, N, K, dtype):
    X = rand_x(M, K, M + 2 * K, dtype, [(1, 5, 30.0)])
    W = rand_w(N, K, N + 3, dtype)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(4)) * 0.1).to(dtype)
    Wq4, sw = q.qlin_quantize_weight(dev(W), q.QLIN_W_INT4_G128)
    rq, rs = oracle.quantize_weight(W, "int4_g128")
    assert np.array_equal(Wq4.cpu().numpy(), rq) and np.array_equal(sw.cpu().numpy(), rs)
    Y = q.qlin_w4a8_forward(dev(X), Wq4, sw, bias=dev(bias))
    r = oracle.w4a8_forward(X, rq, rs, group=128, bias=bias)
    assert_rows_close(Y, r, extra=EXTRA_FP8, what=f"w4a8 {M}x{N}x{K}")
