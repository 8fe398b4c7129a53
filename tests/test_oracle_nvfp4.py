"""Pins of the NVFP4 weight oracle (oracle/oracle.c), against things outside it.

The format is a reading (the Darkstar pages name NVFP4 as their primary
release and give no layout): E2M1 codes, one E4M3 scale per 16 consecutive
weights of a row, one fp32 scale per tensor, s_t = absmax / (6 * 448). The
pins: the E2M1 code table written out by hand; rounding ties and saturation
by hand; the nearest-value-ties-to-even property on a dense grid; the packed
bytes, block scales and tensor scale of a hand-built weight; the forward
against a library matmul of weights decoded here independently (torch's
float8_e4m3fn for the scales, the packing unpacked in numpy); and the
half-step bound, which a swapped pair of block scales breaks.
"""
import numpy as np
import torch

import oracle

# E2M1 code -> value, written from the format (sign bit 3; exponent 0 subnormal)
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_e2m1_decode_table():
    for c, v in enumerate(E2M1):
        got = oracle.e2m1_decode(c)
        assert got == v and np.signbit(got) == np.signbit(v), (c, got, v)


def test_e2m1_encode_ties_and_saturation():
    cases = [(0.0, 0), (-0.0, 8), (0.25, 0), (0.2500001, 1), (0.3, 1), (0.75, 2), (1.25, 2), (1.2500001, 3),
             (1.75, 4), (2.5, 4), (2.5000002, 5), (3.5, 6), (5.0, 6), (5.0000005, 7), (6.0, 7), (7.0, 7), (1e30, 7),
             (-0.3, 9), (-3.5, 14), (-100.0, 15)]
    for t, c in cases:
        assert oracle.e2m1_encode(t) == c, (t, oracle.e2m1_encode(t), c)


def test_e2m1_encode_is_nearest_ties_to_even():
    mags = np.array(E2M1[:8])
    ts = np.concatenate([np.arange(-8.0, 8.0, 1.0 / 512), np.random.default_rng(5).uniform(-7, 7, 2000)])
    for t in ts.astype(np.float32):
        c = oracle.e2m1_encode(float(t))
        v = E2M1[c]
        d = abs(v - float(t))
        dists = np.abs(mags - abs(float(t)))
        assert d == dists.min(), (t, c)
        if np.count_nonzero(dists == d) > 1:
            assert (c & 1) == 0, ("tie not to the even mantissa", t, c)
        if t != 0:
            assert ((c & 8) != 0) == (t < 0)


def test_nvfp4_packed_bytes_scales_by_hand():
    """K = 32 (one block of 32): row 0 holds every magnitude in block 0 at
    step 1 and in block 1 at step 2; row 1 holds 2688 (so absmax/2688 = 1)
    and a zero block."""
    base = [0.5, 1, 1.5, 2, 3, 4, 6, 0, -0.5, -1, -1.5, -2, -3, -4, -6, 0]
    codes0 = [1, 2, 3, 4, 5, 6, 7, 0, 9, 10, 11, 12, 13, 14, 15, 0]
    W = torch.zeros((2, 32), dtype=torch.float32)
    W[0, :16] = torch.tensor(base)
    W[0, 16:] = 2 * torch.tensor(base, dtype=torch.float32)
    W[1, 0] = 2688.0
    q, sb, st = oracle.quantize_weight_nvfp4(W.to(torch.bfloat16))
    assert st == 1.0
    # block scales: e4m3(6/6) = 1.0 = 0x38, e4m3(12/6) = 2.0 = 0x40, e4m3(2688/6) = 448 = 0x7E, a zero block 0
    assert list(sb[0]) == [0x38, 0x40] and list(sb[1]) == [0x7E, 0x00]
    # byte b: code of element b (low nibble), code of element b + 16 (high nibble)
    assert list(q[0]) == [c | (c << 4) for c in codes0]
    assert list(q[1]) == [0x07] + [0] * 15


def _decode_np(q, sb, st, K):
    """W' = decode(code) * decode(s_b) * s_t with the packing and both decodes done here."""
    N = q.shape[0]
    b = q.reshape(N, K // 32, 16)
    codes = np.concatenate([b & 0x0F, b >> 4], axis=2).reshape(N, K)
    vals = np.array(E2M1, np.float64)[codes]
    scales = torch.from_numpy(sb.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return vals * np.repeat(scales, 16, axis=1) * float(st)


def test_nvfp4_forward_matches_matmul_of_decoded_weights():
    g = torch.Generator().manual_seed(9)
    M, N, K = 5, 24, 256
    X = torch.randn((M, K), generator=g).to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16)
    bias = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16)
    q, sb, st = oracle.quantize_weight_nvfp4(W)
    r = oracle.nvfp4_weight_only_forward(X, q, sb, st, bias=bias)
    ref = X.double().numpy() @ _decode_np(q, sb, st, K).T + bias.double().numpy()
    assert np.allclose(r["Y64"], ref, rtol=1e-12, atol=1e-12)


def test_nvfp4_within_half_step_and_swapped_scales_break_it():
    g = torch.Generator().manual_seed(11)
    N, K = 16, 128
    W = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16)
    q, sb, st = oracle.quantize_weight_nvfp4(W)
    w = W.double().numpy()
    scales = torch.from_numpy(sb.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    d = np.repeat(scales, 16, axis=1) * st            # each element's block step
    wd = _decode_np(q, sb, st, K)
    # half the E2M1 spacing around the decoded value, in units of d (the step
    # below 2 is 0.5, below 4 it is 1, above it 2; at a boundary the larger)
    a = np.abs(wd / np.where(d == 0, 1, d))
    half = np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0))
    err = np.abs(w - wd)
    assert np.all(err <= half * d * (1 + 1e-6) + 1e-30)
    # two blocks' scales exchanged: the decoded weights leave the bound
    sb2 = sb.copy()
    sb2[:, [0, 1]] = sb2[:, [1, 0]]
    wd2 = _decode_np(q, sb2, st, K)
    d2 = np.repeat(torch.from_numpy(sb2.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy(), 16, axis=1) * st
    a2 = np.abs(wd2 / np.where(d2 == 0, 1, d2))
    half2 = np.where(a2 < 2, 0.25, np.where(a2 < 4, 0.5, 1.0))
    assert not np.all(np.abs(w - wd2) <= half2 * d2 * (1 + 1e-6) + 1e-30)


def test_nvfp4_w4a4_forward_matches_matmul_of_both_decoded_operands():
    """W4A4: the activations quantised per call by the same rule as a weight
    (their tensor scale from the call's absmax); the forward against a
    matmul of both operands decoded here."""
    g = torch.Generator().manual_seed(13)
    M, N, K = 6, 20, 192
    X = torch.randn((M, K), generator=g).to(torch.bfloat16)
    X[2, 5] = 90.0                      # a large entry: that row's block scale and the tensor scale follow it
    W = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16)
    bias = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16)
    q, sb, st = oracle.quantize_weight_nvfp4(W)
    r = oracle.nvfp4_forward(X, q, sb, st, bias=bias)
    qx, sbx, stx = oracle.quantize_weight_nvfp4(X)
    assert np.array_equal(r["Xq"], qx) and np.array_equal(r["s_bx"], sbx) and r["s_tx"] == stx
    assert stx == np.float32(90.0) / np.float32(2688.0)
    ref = _decode_np(qx, sbx, stx, K) @ _decode_np(q, sb, st, K).T + bias.double().numpy()
    assert np.allclose(r["Y64"], ref, rtol=1e-12, atol=1e-12)
    # only the listed rows are computed, in the listed order
    rr = oracle.nvfp4_forward(X, q, sb, st, bias=bias, rows=[4, 0])
    assert np.array_equal(rr["Y64"], r["Y64"][[4, 0]])


def test_nvfp4_w4a4_close_to_the_unquantised_product():
    """The W4A4 output is the unquantised product up to 4-bit noise (about
    14% normwise here, with 4-bit codes on both sides), and leaving out the
    activations' tensor scale, a plausible slip, moves it far outside that."""
    g = torch.Generator().manual_seed(17)
    M, N, K = 4, 12, 512
    X = torch.randn((M, K), generator=g).to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16)
    q, sb, st = oracle.quantize_weight_nvfp4(W)
    r = oracle.nvfp4_forward(X, q, sb, st)
    exact = X.double().numpy() @ W.double().numpy().T
    rel = np.linalg.norm(r["Y64"] - exact) / np.linalg.norm(exact)
    assert 1e-3 < rel < 0.3, rel   # 4-bit codes on both sides: about 14% here
    wrong = r["Y64"] / r["s_tx"]      # the same sum without the activations' tensor scale
    assert np.linalg.norm(wrong - exact) / np.linalg.norm(exact) > 1.0
