"""Pins for the oracle's linear-layer functions (CPU only).

The checks reduce the oracle's layer functions to things fixed outside it:
the page facts in tests/golden/page_facts.json, special cases that collapse
to a textbook routine (pure vector-wise int8, a plain fp matmul), numpy's
integer and fp64 matmul on tiny inputs, closed forms, and torch's own casts
for the dequant rule weight.to(bf16) * weight_scale.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")
with open(GOLDEN) as _f:
    FACTS = json.load(_f)
THR = FACTS["outlier_threshold"]["value"]


def bits_to_f64(bits, dt):
    return oracle.bits_to_torch(np.ascontiguousarray(bits), dt).double().numpy()


def rand_x(M, K, seed, dtype=torch.bfloat16, clip=None):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((M, K), generator=g)
    if clip is not None:
        x = x.clamp(-clip, clip)
    return x.to(dtype)


def rand_w(N, K, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed + 17)
    return (torch.randn((N, K), generator=g) * 0.02).to(dtype)


# --------------------------------------------------------- outlier set ----

@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_threshold_boundary(dtype):
    assert THR == 6.0
    K = 64
    x = torch.zeros((4, K), dtype=torch.float32)
    # the next representable value above 6.0 in this dtype
    nxt = torch.tensor([THR], dtype=dtype)
    nxt = (nxt.view(torch.int16) + 1).view(dtype).item()
    x[0, 3] = THR            # exactly at the threshold: not an outlier (strict >)
    x[1, 5] = nxt            # just above: outlier
    x[2, 7] = -nxt           # just below -6: outlier (absolute value)
    x[3, 9] = -THR           # exactly -6: not an outlier
    x[0, 11] = 5.99
    X = x.to(dtype)
    assert nxt > THR
    r = oracle.int8_outlier_prep(X, THR)
    assert r["O"].tolist() == [5, 7]
    assert r["count"] == 2
    # the outlier columns carry zero codes and are copied exactly into X_O
    assert np.all(r["Xq"][:, [5, 7]] == 0)
    xo = bits_to_f64(r["X_O"], r["dt"])
    assert xo[1, 0] == nxt and xo[2, 1] == -nxt and xo[0, 0] == 0.0


def test_outlier_test_spans_all_tokens():
    # A column is an outlier when ANY token of the call exceeds the
    # threshold; its small values in other tokens are excluded too.
    X = rand_x(16, 128, 1, clip=2.0).float()
    X[7, 40] = 7.5
    X = X.to(torch.bfloat16)
    r = oracle.int8_outlier_prep(X, THR)
    assert r["O"].tolist() == [40]
    xf = X.float().numpy()
    keep = np.ones(128, bool)
    keep[40] = False
    expect_absmax = np.abs(xf[:, keep]).max(axis=1).astype(np.float32)
    assert np.array_equal(r["s_x"], expect_absmax / np.float32(127.0))


def test_threshold_disabled_values():
    X = rand_x(8, 64, 2)
    X[0, 0] = 100.0
    for thr in (0.0, -1.0, float("inf")):
        r = oracle.int8_outlier_prep(X, thr)
        assert r["count"] == 0


# ---------------------------------------- special cases of LLM.int8 ------

def vectorwise_int8_reference(X, Wq, s_w):
    """Plain vector-wise int8 written with torch/numpy primitives (no outliers)."""
    x = X.float()
    absmax = x.abs().amax(dim=1)
    s_x = absmax / torch.tensor(127.0)
    inv = torch.tensor(1.0) / s_x
    t = x * inv[:, None]
    q = torch.where(x == 0, torch.zeros_like(t), torch.round(t).clamp(-127, 127)).to(torch.int64)
    C = q.numpy() @ Wq.astype(np.int64).T
    Y = C.astype(np.float64) * s_x.double().numpy()[:, None] * s_w.astype(np.float64)[None, :]
    return q.numpy().astype(np.int8), s_x.numpy(), C, Y


@pytest.mark.parametrize("how", ["clipped", "threshold_inf", "threshold_zero"])
def test_no_outliers_equals_pure_vectorwise_int8(how):
    M, K, N = 24, 160, 40
    if how == "clipped":
        X, thr = rand_x(M, K, 3, clip=THR), THR
    else:
        X = rand_x(M, K, 3)
        X[2, 9] = 50.0
        thr = float("inf") if how == "threshold_inf" else 0.0
    W = rand_w(N, K, 3)
    Wq, s_w = oracle.quantize_weight(W, "int8_row")
    q_ref, s_ref, C_ref, Y_ref = vectorwise_int8_reference(X, Wq, s_w)
    p = oracle.int8_outlier_prep(X, thr)
    assert p["count"] == 0
    assert np.array_equal(p["Xq"], q_ref)
    assert np.array_equal(p["s_x"], s_ref)
    r = oracle.int8_outlier_forward(X, Wq, s_w, thr)
    assert np.array_equal(r["C"].astype(np.int64), C_ref)
    np.testing.assert_allclose(r["Y64"], Y_ref, rtol=1e-12, atol=1e-12)


def test_all_outliers_equals_plain_fp_matmul():
    M, K, N = 12, 96, 20
    X = rand_x(M, K, 4).float()
    X[M - 1, :] = 8.0                         # every column exceeds the threshold somewhere
    X = X.to(torch.bfloat16)
    W = rand_w(N, K, 4)
    Wq, s_w = oracle.quantize_weight(W, "int8_row")
    p = oracle.int8_outlier_prep(X, THR)
    assert p["count"] == K and np.all(p["Xq"] == 0)
    r = oracle.int8_outlier_forward(X, Wq, s_w, THR)
    assert np.all(r["C"] == 0)
    # dequant rule weight.to(bf16) * weight_scale, through torch's own ops
    W_deq = (torch.from_numpy(Wq).float() * torch.from_numpy(s_w)[:, None]).to(torch.bfloat16)
    Y_ref = X.double().numpy() @ W_deq.double().numpy().T
    np.testing.assert_allclose(r["Y64"], Y_ref, rtol=1e-12, atol=1e-12)


def test_outlier_weights_follow_dequant_rule():
    W = rand_w(32, 64, 5)
    Wq, s_w = oracle.quantize_weight(W, "int8_row")
    O = np.array([0, 3, 63], np.int32)
    for dtype, dt in ((torch.bfloat16, oracle.BF16), (torch.float16, oracle.F16)):
        got = oracle.outlier_weights(Wq, s_w, O, dt)
        ref = (torch.from_numpy(Wq[:, O]).float() * torch.from_numpy(s_w)[:, None]).to(dtype)
        assert np.array_equal(got, ref.view(torch.int16).numpy().view(np.uint16))


def test_mixed_decomposition_matches_split_sum():
    # Y = int8 part + fp part, each checked against numpy on its own.
    M, K, N = 20, 128, 24
    X = rand_x(M, K, 6).float()
    X[3, 10] = -9.0
    X[15, 100] = 12.0
    X = X.to(torch.float16)
    W = rand_w(N, K, 6, torch.float16)
    bias = (torch.arange(N, dtype=torch.float32) / 7).to(torch.float16)
    Wq, s_w = oracle.quantize_weight(W, "int8_row")
    p = oracle.int8_outlier_prep(X, THR)
    assert p["O"].tolist() == [10, 100]
    r = oracle.int8_outlier_forward(X, Wq, s_w, THR, bias=bias)
    C = p["Xq"].astype(np.int64) @ Wq.astype(np.int64).T
    assert np.array_equal(r["C"].astype(np.int64), C)
    W_deq = (torch.from_numpy(Wq[:, p["O"]]).float() * torch.from_numpy(s_w)[:, None]).to(torch.float16)
    F = X.double().numpy()[:, p["O"]] @ W_deq.double().numpy().T
    Y = C * p["s_x"].astype(np.float64)[:, None] * s_w.astype(np.float64)[None, :] + F + bias.double().numpy()
    np.testing.assert_allclose(r["Y64"], Y, rtol=1e-12, atol=1e-12)
    # the rounded output is the fp16 rounding of Y64 (torch's cast from exact fp32 values)
    yb = torch.from_numpy(r["Y64"]).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    mism = np.nonzero(yb != r["Y"])[0]
    # torch casts fp64 -> fp16 through fp32; a double rounding may differ by one ulp
    assert mism.size <= 2


def test_brute_force_tiny_int32():
    # every code pattern of a 2x2x2 block at extreme values, and random
    # tiny shapes, against numpy's int64 matmul
    rng = np.random.default_rng(7)
    for M, N, K in [(1, 1, 16), (2, 3, 32), (4, 4, 48), (3, 2, 16)]:
        for trial in range(4):
            X = torch.from_numpy(rng.uniform(-5.9, 5.9, (M, K)).astype(np.float32)).to(torch.bfloat16)
            W = torch.from_numpy(rng.normal(0, 0.02, (N, K)).astype(np.float32)).to(torch.bfloat16)
            Wq, s_w = oracle.quantize_weight(W, "int8_row")
            p = oracle.int8_outlier_prep(X, THR)
            r = oracle.int8_outlier_forward(X, Wq, s_w, THR)
            assert np.array_equal(r["C"].astype(np.int64),
                                  p["Xq"].astype(np.int64) @ Wq.astype(np.int64).T)
    # all sign patterns of +-absmax rows: codes are exactly +-127
    for pattern in range(16):
        signs = np.array([1 if (pattern >> b) & 1 else -1 for b in range(4)], np.float32)
        X = torch.from_numpy(np.tile(signs, (2, 4)) * 3.0).to(torch.bfloat16)     # [2,16]
        W = torch.from_numpy(np.tile(signs[::-1].copy(), (3, 4)) * 0.5).to(torch.bfloat16)
        Wq, s_w = oracle.quantize_weight(W, "int8_row")
        p = oracle.int8_outlier_prep(X, THR)
        assert set(np.unique(np.abs(p["Xq"]))) == {127}
        r = oracle.int8_outlier_forward(X, Wq, s_w, THR)
        assert np.array_equal(r["C"].astype(np.int64), p["Xq"].astype(np.int64) @ Wq.astype(np.int64).T)


def test_int32_bound_at_largest_k():
    # K = 12288 with every code at 127: C = 12288 * 127^2 = 198,193,152 < 2^31
    K = 12288
    X = torch.ones((1, K), dtype=torch.bfloat16)
    W = torch.full((2, K), 0.25, dtype=torch.bfloat16)
    W[1] = -0.25
    Wq, s_w = oracle.quantize_weight(W, "int8_row")
    r = oracle.int8_outlier_forward(X, Wq, s_w, THR)
    assert r["C"].tolist() == [[198193152, -198193152]]
    assert 198193152 < 2 ** 31


def test_massive_activation_goes_to_fp_path():
    f = FACTS["massive_activation_text_encoder"]
    wl = workloads.get_workload("te_fp8_dynamic_mlp")
    lin = workloads.Linear("t", 16, 4096, 8)
    X, W, _ = workloads.make_linear(wl, lin)
    assert X[0, f["channel"]].item() == 12992.0 and X[5, f["channel"]].item() == 9024.0
    p = oracle.int8_outlier_prep(X, THR)
    assert f["channel"] in p["O"].tolist()
    # the massive value does not enter the int8 row scale
    assert p["s_x"][0] < np.float32(THR) / np.float32(127.0) * np.float32(1.0001)


# ------------------------------------------------------------------ FP8 ---

def decode_e4m3_torch(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def test_fp8_static_acc_exact_and_scaled():
    M, K, N = 16, 128, 24
    X = rand_x(M, K, 8)
    W = rand_w(N, K, 8)
    Wq, ws = oracle.quantize_weight(W, "fp8_tensor")
    assert ws[0] == np.float32(np.abs(W.float().numpy()).max()) / np.float32(448.0)
    x_scale = oracle.absmax_scale(rand_x(M, K, 9), 448.0)
    r = oracle.fp8_forward(X, Wq, ws, x_scale=x_scale)
    a = decode_e4m3_torch(r["Xq"])
    b = decode_e4m3_torch(Wq)
    acc = a @ b.T
    assert np.array_equal(r["acc"], acc)                    # exact in fp64
    np.testing.assert_allclose(r["Y64"], acc * float(x_scale) * float(ws[0]), rtol=1e-15)
    # activations above input_scale*448 saturate to +-448
    inv = np.float32(1.0) / np.float32(x_scale)
    big = X.float().numpy() * inv > 464
    assert np.all(r["Xq"][big] == 0x7E)


def test_fp8_codes_vs_torch_cast():
    X = rand_x(32, 64, 10)
    s = oracle.absmax_scale(X, 448.0)
    codes = oracle.fp8_static_prep(X, s)
    inv = torch.tensor(1.0, dtype=torch.float32) / torch.tensor(s, dtype=torch.float32)
    ref = (X.float() * inv).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def test_fp8_dynamic_scales_and_channel_dequant():
    M, K, N = 8, 256, 16
    X = rand_x(M, K, 11).float()
    X[0, 2] = 12992.0                               # massive value: row scale = 29 exactly
    X = X.to(torch.bfloat16)
    W = rand_w(N, K, 11)
    Wq, sb = oracle.quantize_weight(W, "fp8_channel")
    assert sb.dtype == np.uint16 and sb.shape == (N,)  # bf16 [out, 1]
    # weight.to(bf16) * weight_scale recovers W to within e4m3's relative step (2^-4 half-ulp)
    w_scale = torch.from_numpy(sb.view(np.int16)).view(torch.bfloat16)[:, None]
    deq = (torch.from_numpy(Wq).view(torch.float8_e4m3fn).to(torch.bfloat16) * w_scale).float()
    wf = W.float()
    rowmax = wf.abs().amax(1, keepdim=True)
    assert torch.all((deq - wf).abs() <= rowmax * 2.0 ** -4 * 1.02 + 1e-30)
    r = oracle.fp8_forward(X, Wq, sb, x_scale=None)
    assert r["s_x"][0] == 29.0
    a = decode_e4m3_torch(r["Xq"])
    acc = a @ decode_e4m3_torch(Wq).T
    assert np.array_equal(r["acc"], acc)
    sw = w_scale.double().numpy().reshape(-1)
    np.testing.assert_allclose(r["Y64"], acc * r["s_x"].astype(np.float64)[:, None] * sw[None, :],
                               rtol=1e-15)


# ---------------------------------------------------------------- W4A8 ---

def unpack_int4(packed, K):
    """int4 codes [N,K] from the packed [N,K/2] bytes: byte b of each 16-byte
    block holds element b of the block's 32 in its low nibble, b + 16 in its
    high nibble, two's complement."""
    b = packed.reshape(packed.shape[0], K // 32, 16)
    nib = np.concatenate([b & 0x0F, b >> 4], axis=2).reshape(packed.shape[0], K).astype(np.int16)
    return np.where(nib >= 8, nib - 16, nib)


# ---------------------------------------------------------------------------
# Weight-only FP8 (Text-Encoder-FP8 page, "Format": weight.to(bf16) * weight_scale,
# activations unquantised)
# ---------------------------------------------------------------------------

def _finite_e4m3_codes(shape, seed):
    g = np.random.default_rng(seed)
    c = g.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C                       # no NaN codes
    return c


def test_fp8_weight_only_dequant_is_torch_rule():
    """W_deq equals torch's own float8 cast and bf16 multiply, bit for bit,
    on every code at several scales and on random codes and scales."""
    codes = np.tile(np.arange(256, dtype=np.uint8), (6, 1))
    codes[(codes & 0x7F) == 0x7F] = 0
    scales = torch.tensor([1.0, 0.5, 3.0e-3, 1.0 / 448, 7.1875, 2.0 ** -20], dtype=torch.bfloat16)
    g = torch.Generator().manual_seed(31)
    rc = _finite_e4m3_codes((64, 96), 31)
    rs = (torch.rand(64, generator=g) * 0.05 + 1e-4).to(torch.bfloat16)
    for c, s in ((codes, scales), (rc, rs)):
        bits = s.view(torch.int16).numpy().view(np.uint16)
        got = oracle.fp8_weight_only_dequant(c, bits)
        ref = (torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.bfloat16) * s[:, None])
        assert np.array_equal(got, ref.view(torch.int16).numpy().view(np.uint16))


def test_fp8_weight_only_unit_scale_is_plain_matmul():
    """With all scales 1 the weights are the decoded codes, so Y64 is the
    fp64 matmul of X with torch's decode of the codes."""
    M, K, N = 12, 160, 20
    X = rand_x(M, K, 32)
    codes = _finite_e4m3_codes((N, K), 32)
    ones = np.full((N,), 0x3F80, np.uint16)            # bf16 1.0
    r = oracle.fp8_weight_only_forward(X, codes, ones)
    ref = X.double().numpy() @ decode_e4m3_torch(codes).T
    np.testing.assert_allclose(r["Y64"], ref, rtol=1e-12, atol=1e-12)


def test_fp8_weight_only_closed_form_and_rounding():
    """X = 1 and one code per row: Y64 = K * bf16(decode(c) * s) + bias, and
    Y is Y64 rounded once to the activation dtype."""
    M, K, N = 3, 64, 5
    X = torch.ones((M, K), dtype=torch.bfloat16)
    codes = np.zeros((N, K), np.uint8)
    cvals = [0x38, 0x41, 0xC6, 0x01, 0x7E]             # 1, 2.25, -14, the smallest subnormal, 448
    for j, c in enumerate(cvals):
        codes[j, :] = c
    s = torch.tensor([0.5, 0.0999, -3.0, 1024.0, 0.013], dtype=torch.bfloat16)
    bias = torch.tensor([0.0, 1.5, -2.0, 0.25, 100.0], dtype=torch.bfloat16)
    r = oracle.fp8_weight_only_forward(X, codes, s.view(torch.int16).numpy().view(np.uint16), bias=bias)
    w = (torch.from_numpy(codes[:, :1]).view(torch.float8_e4m3fn).to(torch.bfloat16) * s[:, None]).double()
    ref = K * w.numpy().reshape(-1) + bias.double().numpy()
    assert np.array_equal(r["Y64"], np.tile(ref, (M, 1)))
    y = torch.from_numpy(r["Y64"]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(r["Y"], y)


def test_int4_pack_layout_and_range():
    W = rand_w(8, 256, 12)
    q, s = oracle.quantize_weight(W, "int4_g128")
    assert q.shape == (8, 128) and s.shape == (8, 2)
    u = unpack_int4(q, 256)
    assert u.min() >= -7 and u.max() <= 7
    for j in range(8):
        for k in (0, 1, 2, 127, 128, 255):
            assert oracle.lib().orc_int4_unpack(q.ctypes.data, 256, j, k) == u[j, k]
    # scale = group absmax / 7
    wf = W.float().numpy().reshape(8, 2, 128)
    assert np.array_equal(s, np.abs(wf).max(axis=2).astype(np.float32) / np.float32(7.0))


def test_int4_pack_bytes_by_hand():
    """The packed bytes of known codes, written out by hand: weights that are
    exact multiples of their group's step 0.5 (each group holds a +-3.5, so
    s = 3.5 / 7 = 0.5 and the code of w is 2w). Byte b of the 16-byte block m
    must hold code 32m + b in its low nibble and code 32m + b + 16 in its high
    nibble, two's complement; swapping the nibbles, packing even/odd pairs or
    dropping the sign would each change a byte here."""
    K = 256
    codes = np.array([[((5 * k + 3 * j) % 15) - 7 for k in range(K)] for j in range(3)], np.int64)
    codes[:, ::128] = 7   # a full-scale code in every group
    W = torch.tensor(codes * 0.5, dtype=torch.float32).to(torch.bfloat16)
    q, s = oracle.quantize_weight(W, "int4_g128")
    assert np.all(s == np.float32(0.5))
    for j in range(3):
        for m in range(K // 32):
            for b in range(16):
                lo, hi = codes[j, 32 * m + b] & 0xF, codes[j, 32 * m + b + 16] & 0xF
                assert int(q[j, 16 * m + b]) == (lo | (hi << 4)), (j, m, b)


def test_w4a8_equal_group_scales_reduce_to_per_channel():
    M, K, N, G = 6, 384, 10, 128
    X = rand_x(M, K, 13)
    g = torch.Generator().manual_seed(14)
    W = torch.randn((N, K), generator=g) * 0.02
    W.view(N, K // G, G)[:, :, 0] = 0.1           # identical absmax in every group -> equal scales
    W = W.to(torch.bfloat16)
    q, s = oracle.quantize_weight(W, "int4_g128")
    assert np.all(s == s[:, :1])
    r = oracle.w4a8_forward(X, q, s, group=G, want_cg=True)
    u = unpack_int4(q, K).astype(np.int64)
    C = r["Xq"].astype(np.int64) @ u.T
    assert np.array_equal(r["Cg"].sum(axis=2).astype(np.int64), C)
    for gi in range(K // G):
        sl = slice(gi * G, (gi + 1) * G)
        assert np.array_equal(r["Cg"][:, :, gi].astype(np.int64),
                              r["Xq"][:, sl].astype(np.int64) @ u[:, sl].T)
    Y = C * r["s_x"].astype(np.float64)[:, None] * s[:, 0].astype(np.float64)[None, :]
    np.testing.assert_allclose(r["Y64"], Y, rtol=1e-12)
    # its activation codes are the pure vector-wise int8 codes
    p = oracle.int8_outlier_prep(X, 0.0)
    assert np.array_equal(p["Xq"], r["Xq"]) and np.array_equal(p["s_x"], r["s_x"])


def test_w4a8_unequal_group_scales_within_rounding_bound():
    """Groups whose scales differ by up to 50x: the output stays within the
    half-step bound of X W^T + b (every int4 code is its weight rounded to the
    nearest step of its own group's scale, every int8 code its activation to
    the nearest step of the row scale), per-group int32 sums equal numpy's
    integer matmul of the unpacked codes, and a swapped pair of group scales
    breaks the bound. A wrong group index in the scale combination fails here."""
    M, K, N, G = 6, 512, 9, 128
    X = rand_x(M, K, 31)
    g = torch.Generator().manual_seed(32)
    W = torch.randn((N, K), generator=g) * 0.02
    for gi, f in enumerate((1.0, 50.0, 0.2, 7.0)):   # a different magnitude in every group
        W[:, gi * G:(gi + 1) * G] *= f
    W = W.to(torch.bfloat16)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(33)) * 0.1).to(torch.bfloat16)
    q, s = oracle.quantize_weight(W, "int4_g128")
    assert np.all(s.max(axis=1) > 40 * s.min(axis=1))
    r = oracle.w4a8_forward(X, q, s, group=G, bias=bias, want_cg=True)
    u = unpack_int4(q, K).astype(np.int64)
    for gi in range(K // G):
        sl = slice(gi * G, (gi + 1) * G)
        assert np.array_equal(r["Cg"][:, :, gi].astype(np.int64), r["Xq"][:, sl].astype(np.int64) @ u[:, sl].T)
    x = X.double().numpy()
    w = W.double().numpy()
    exact = x @ w.T + bias.double().numpy()[None, :]
    sx = r["s_x"].astype(np.float64)[:, None, None]
    sw = np.repeat(s.astype(np.float64), G, axis=1)[None, :, :]
    bound = ((np.abs(x)[:, None, :] + sx / 2) * sw / 2 + np.abs(w)[None, :, :] * sx / 2).sum(axis=2)
    err = np.abs(r["Y64"] - exact)
    assert np.all(err <= bound * (1 + 1e-6) + 1e-12)
    assert np.linalg.norm(err) < 0.25 * np.linalg.norm(exact)   # int4 steps: about 11% noise here
    # the scale-weighted group sum the page's format defines, from the oracle's own partials
    y = r["s_x"].astype(np.float64)[:, None] * (r["Cg"].astype(np.float64) * s.astype(np.float64)[None]).sum(axis=2)
    np.testing.assert_allclose(r["Y64"], y + bias.double().numpy()[None, :], rtol=1e-12, atol=1e-12)
    # the scales of groups 0 and 1 exchanged: far outside the bound
    s_bad = s.copy()
    s_bad[:, [0, 1]] = s_bad[:, [1, 0]]
    bad = oracle.w4a8_forward(X, q, s_bad, group=G, bias=bias)
    assert np.any(np.abs(bad["Y64"] - exact) > bound)


def test_rows_subset_matches_full():
    wl = workloads.get_workload("tiny_int8")
    X, W, bias = workloads.make_linear(wl, wl.linears[0])
    Wq, s_w = oracle.quantize_weight(W, "int8_row")
    full = oracle.int8_outlier_forward(X, Wq, s_w, THR, bias=bias)
    rows = [0, 5, 63, 17]
    sub = oracle.int8_outlier_forward(X, Wq, s_w, THR, bias=bias, rows=rows)
    assert np.array_equal(sub["C"], full["C"][rows])
    assert np.array_equal(sub["Y64"], full["Y64"][rows])


def test_zero_rows_and_degenerate_scales():
    X = rand_x(4, 64, 15).float()
    X[1] = 0.0
    X = X.to(torch.bfloat16)
    p = oracle.int8_outlier_prep(X, THR)
    assert p["s_x"][1] == 0.0 and np.all(p["Xq"][1] == 0)
    assert np.all(np.isfinite(p["s_x"])) and np.all(p["s_x"][[0, 2, 3]] > 0)
    xq, sx = oracle.fp8_dynamic_prep(X)
    assert sx[1] == 0.0 and np.all(xq[1] == 0)


# ---------------------------------------------------------------------------
# Block-scaled int8 weights: 8-bit codes with one scale per 32 weights of a
# row (the text-encoder page's comparison with GGUF Q8_0)
# ---------------------------------------------------------------------------

def test_int8_block_of_whole_row_is_per_channel():
    W = rand_w(12, 96, 21)
    qb, sb = oracle.quantize_weight(W, "int8_block", group=96)
    qr, sr = oracle.quantize_weight(W, "int8_row")
    assert np.array_equal(qb, qr) and np.array_equal(sb[:, 0], sr)


def test_int8_block_scales_follow_each_slice():
    N, K, B = 9, 160, 32
    W = rand_w(N, K, 22).float()
    W[3, 64:96] = 0.0                                 # an all-zero block: scale 0, codes 0
    W[5, 40] = 0.5                                    # one large weight moves only its own block
    W = W.to(torch.bfloat16)
    q, s = oracle.quantize_weight(W, "int8_block", group=B)
    assert s.shape == (N, K // B)
    assert s[3, 2] == 0.0 and np.all(q[3, 64:96] == 0)
    for b in range(K // B):
        qs, ss = oracle.quantize_weight(W[:, b * B:(b + 1) * B].contiguous(), "int8_row")
        assert np.array_equal(q[:, b * B:(b + 1) * B], qs)
        assert np.array_equal(s[:, b], ss)
    assert np.abs(q).max() == 127 and q.min() >= -127
    # the large weight sets its block's scale: 0.5 / 127 in fp32
    assert s[5, 1] == np.float32(np.float32(0.5) / np.float32(127.0))


def test_int8_block_equal_scales_reduce_to_vectorwise():
    M, K, N, B = 7, 128, 11, 32
    X = rand_x(M, K, 23)
    g = torch.Generator().manual_seed(24)
    W = torch.randn((N, K), generator=g) * 0.02
    W.view(N, K // B, B)[:, :, 5] = -0.0625          # identical absmax in every block of a row
    W = W.to(torch.bfloat16)
    q, s = oracle.quantize_weight(W, "int8_block", group=B)
    assert np.all(s == s[:, :1])
    r = oracle.int8_block_forward(X, q, s, block=B, want_cb=True)
    qr, sr = oracle.quantize_weight(W, "int8_row")
    assert np.array_equal(q, qr) and np.array_equal(s[:, 0], sr)
    v = oracle.int8_outlier_forward(X, qr, sr, 0.0)
    assert np.array_equal(r["Cb"].sum(axis=2).astype(np.int64), v["C"].astype(np.int64))
    np.testing.assert_allclose(r["Y64"], v["Y64"], rtol=1e-12, atol=0.0)
    assert np.array_equal(r["Y"], v["Y"])


def test_int8_block_forward_within_rounding_bound():
    """|Y64 - (X W^T + b)| <= sum_k (|x| + s_x/2) * s_w/2 + |w| * s_x/2: each
    code is its value rounded to the nearest step of its scale."""
    M, K, N, B = 5, 192, 13, 32
    X = rand_x(M, K, 25)
    W = rand_w(N, K, 26)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(27)) * 0.1).to(torch.bfloat16)
    q, s = oracle.quantize_weight(W, "int8_block", group=B)
    r = oracle.int8_block_forward(X, q, s, block=B, bias=bias, want_cb=True)
    C = np.zeros((M, N, K // B), np.int64)
    for b in range(K // B):
        sl = slice(b * B, (b + 1) * B)
        C[:, :, b] = r["Xq"][:, sl].astype(np.int64) @ q[:, sl].astype(np.int64).T
    assert np.array_equal(r["Cb"].astype(np.int64), C)
    x = X.double().numpy()
    w = W.double().numpy()
    exact = x @ w.T + bias.double().numpy()[None, :]
    sx = r["s_x"].astype(np.float64)[:, None, None]
    sw = np.repeat(s.astype(np.float64), B, axis=1)[None, :, :]
    bound = ((np.abs(x)[:, None, :] + sx / 2) * sw / 2 + np.abs(w)[None, :, :] * sx / 2).sum(axis=2)
    err = np.abs(r["Y64"] - exact)
    assert np.all(err <= bound * (1 + 1e-6) + 1e-12)
    # and the bound is not vacuous: the error is a small part of |Y|
    assert np.linalg.norm(err) < 0.05 * np.linalg.norm(exact)
    # a transposed block scale breaks the bound somewhere
    s_bad = s.copy()
    s_bad[:, [0, 1]] = s_bad[:, [1, 0]]
    s_bad[:, 0] *= 3.0
    bad = oracle.int8_block_forward(X, q, s_bad, block=B, bias=bias)
    assert np.any(np.abs(bad["Y64"] - exact) > bound)


# ---------------------------------------------------------------------------
# Unquantised 16-bit linear (the layers kept in fp16)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_fp_linear_identity_returns_the_weight(dtype):
    K, N = 48, 20
    W = rand_w(N, K, 31, dtype)
    r = oracle.fp_linear_forward(torch.eye(K, dtype=dtype), W)
    assert np.array_equal(r["Y"], W.T.contiguous().view(torch.int16).numpy().view(np.uint16))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_fp_linear_small_integers_are_exact(dtype):
    """Integer inputs small enough that every sum is an integer the dtype
    holds exactly: the result is the integer matmul, brute force."""
    g = torch.Generator().manual_seed(32)
    M, K, N = 9, 40, 11
    xi = torch.randint(-3, 4, (M, K), generator=g)
    wi = torch.randint(-3, 4, (N, K), generator=g)
    bi = torch.randint(-5, 6, (N,), generator=g)
    r = oracle.fp_linear_forward(xi.to(dtype), wi.to(dtype), bias=bi.to(dtype))
    ref = np.zeros((M, N), np.int64)
    for i in range(M):
        for j in range(N):
            ref[i, j] = sum(int(xi[i, k]) * int(wi[j, k]) for k in range(K)) + int(bi[j])
    assert np.array_equal(r["Y64"], ref.astype(np.float64))
    assert np.abs(ref).max() <= 256                      # exact in bf16's 8-bit significand
    assert np.array_equal(oracle.bits_to_torch(r["Y"], r["dt"]).double().numpy(), ref.astype(np.float64))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_fp_linear_rounds_once_to_the_dtype(dtype):
    """Y is Y64 rounded to nearest even in the dtype (torch's own cast of the
    fp64 value), and Y64 is within fp64 summation error of X W^T + b."""
    X = rand_x(6, 128, 33, dtype)
    W = rand_w(14, 128, 34, dtype)
    bias = (torch.randn(14, generator=torch.Generator().manual_seed(35)) * 0.1).to(dtype)
    r = oracle.fp_linear_forward(X, W, bias=bias)
    cast = torch.from_numpy(r["Y64"]).to(dtype).contiguous().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(r["Y"], cast)
    x, w = X.double().numpy(), W.double().numpy()
    exact = x @ w.T + bias.double().numpy()[None, :]
    scale = np.abs(x) @ np.abs(w).T + np.abs(bias.double().numpy())[None, :]
    assert np.all(np.abs(r["Y64"] - exact) <= 1e-13 * scale)
    # rows= selects rows of the same result
    sub = oracle.fp_linear_forward(X, W, bias=bias, rows=[5, 0])
    assert np.array_equal(sub["Y"], r["Y"][[5, 0]])


def test_fp_linear_mixed_magnitudes_within_fp64_summation_bound():
    """Products spread over 2^-40 .. 2^40 with cancellation: the oracle adds
    the exact products one by one in fp64, so Y64 is within the recursive
    summation bound (K - 1) * 2^-53 * sum |x w| of the exact rational sum
    (Python fractions), and Y is Y64 rounded once to the dtype."""
    from fractions import Fraction
    g = torch.Generator().manual_seed(39)
    M, K, N = 4, 64, 6
    ex = torch.randint(-20, 21, (M, K), generator=g).double()
    ew = torch.randint(-20, 21, (N, K), generator=g).double()
    X = (torch.randn((M, K), generator=g).double() * torch.pow(2.0, ex)).to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g).double() * torch.pow(2.0, ew)).to(torch.bfloat16)
    X[:, 1] = -X[:, 0]                                     # exact cancellation of large pairs
    W[:, 1] = W[:, 0]
    r = oracle.fp_linear_forward(X, W)
    x, w = X.double().numpy(), W.double().numpy()
    for i in range(M):
        for j in range(N):
            exact = sum(Fraction(float(x[i, k])) * Fraction(float(w[j, k])) for k in range(K))
            mag = sum(abs(Fraction(float(x[i, k])) * Fraction(float(w[j, k]))) for k in range(K))
            assert abs(Fraction(float(r["Y64"][i, j])) - exact) <= Fraction(K - 1, 2 ** 53) * mag
    cast = torch.from_numpy(r["Y64"]).to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(r["Y"], cast)


def test_weight_only_fp8_at_unit_scale_is_the_16bit_linear():
    """With s_w = 1 the dequantised weight is the decoded e4m3 value itself,
    which bf16 holds exactly: the weight-only forward is then the plain
    16-bit linear of that weight."""
    N, K, M = 10, 64, 5
    codes = _finite_e4m3_codes((N, K), 36)
    one = np.full(N, 0x3F80, np.uint16)                     # bf16 1.0
    Wd = torch.from_numpy(oracle.fp8_weight_only_dequant(codes, one).view(np.int16)).view(torch.bfloat16)
    assert np.array_equal(Wd.double().numpy(), decode_e4m3_torch(codes))
    X = rand_x(M, K, 37)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(38)) * 0.1).to(torch.bfloat16)
    a = oracle.fp8_weight_only_forward(X, codes, one, bias=bias)
    b = oracle.fp_linear_forward(X, Wd, bias=bias)
    assert np.array_equal(a["Y"], b["Y"]) and np.array_equal(a["Y64"], b["Y64"])
