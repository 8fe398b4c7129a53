"""Pins for the oracle's scalar codecs (CPU only).

Each check compares the oracle against something that does not come from
the oracle: the format definitions, torch's own float8/bf16/fp16 casts,
closed-form half-way cases, or the facts the pages print
(tests/golden/page_facts.json).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def facts():
    with open(GOLDEN) as f:
        return json.load(f)


def all_16bit_as_f32(dtype):
    bits = torch.arange(0, 65536, dtype=torch.int32).to(torch.int16)
    return bits.view(dtype).float()


# ---------------------------------------------------------------- E4M3 ----

def test_e4m3_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan_ref = np.isnan(ref)
    assert np.array_equal(nan_ref, np.isnan(ours))
    assert set(np.nonzero(nan_ref)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ref[~nan_ref], ours[~nan_ref])


def test_e4m3_format_facts():
    # 3-bit mantissa (page fact) -> 8 codes per binade; max finite 448;
    # smallest subnormal 2^-9; smallest normal 2^-6.
    assert facts()["e4m3_mantissa_bits"]["value"] == 3
    vals = sorted(oracle.e4m3_decode(c) for c in range(0x7F))
    assert vals[-1] == 448.0
    assert vals[1] == 2.0 ** -9
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6
    binade = [v for v in vals if 1.0 <= v < 2.0]
    assert len(binade) == 2 ** 3
    assert binade == [1.0 + m / 8 for m in range(8)]


def _grid_probe_values():
    """Every positive e4m3 value, the midpoints between neighbours and the
    nearest fp32 numbers on both sides of each, plus their negatives."""
    pos = sorted(oracle.e4m3_decode(c) for c in range(0x7F))
    pts = []
    grid = pos + [480.0]                      # 480 = the next grid point above 448
    for a, b in zip(grid[:-1], grid[1:]):
        mid = np.float32((a + b) / 2)
        pts += [np.float32(a), mid, np.nextafter(mid, np.float32(np.inf)),
                np.nextafter(mid, np.float32(-np.inf))]
    pts += [np.float32(v) for v in (1e-30, 2.0 ** -10, 2.0 ** -11, 500.0, 1e6, 3e38)]
    pts = np.array(pts, dtype=np.float32)
    return np.concatenate([pts, -pts])


def _random_f32(n, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(n).astype(np.float32) * np.float32(2.0) ** rng.integers(-14, 10, n).astype(np.float32)
    return x


def test_e4m3_encoders_agree_on_probe_points():
    for t in _grid_probe_values():
        assert oracle.e4m3_encode(float(t)) == oracle.e4m3_encode_search(float(t)), t


def test_e4m3_encoders_agree_on_all_bf16_values():
    vals = all_16bit_as_f32(torch.bfloat16).numpy()
    vals = vals[np.isfinite(vals)]
    # every 7th pattern keeps the test to a few seconds; together with the
    # probe points every rounding boundary is still covered
    for t in vals[::7]:
        assert oracle.e4m3_encode(float(t)) == oracle.e4m3_encode_search(float(t)), t


def test_e4m3_encode_matches_torch_cast():
    # torch's CPU float8 cast rounds to nearest even but maps overflow to
    # NaN; pre-clamping to +-448 turns that into the satfinite behaviour.
    vals = np.concatenate([_grid_probe_values(), _random_f32(20000),
                           all_16bit_as_f32(torch.float16).numpy()])
    vals = vals[np.isfinite(vals)]
    ref = torch.from_numpy(vals).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(float(t)) for t in vals], dtype=np.uint8)
    bad = np.nonzero(ref != ours)[0]
    assert bad.size == 0, [(vals[i], ref[i], ours[i]) for i in bad[:5]]


def test_e4m3_saturates_and_nan():
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE
    assert oracle.e4m3_encode(float("inf")) == 0x7E
    assert oracle.e4m3_encode(float("nan")) == 0x7F
    assert oracle.e4m3_encode(-2.0 ** -11) == 0x80      # negative values rounding to zero keep the sign
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00       # tie at half the smallest subnormal -> even (0)
    assert oracle.e4m3_encode(1.5 * 2.0 ** -9) == 0x02  # tie between m=1 and m=2 -> even


# ---------------------------------------------------------------- int8 ----

@pytest.mark.parametrize("t,expect", [(0.5, 0), (-0.5, 0), (1.5, 2), (-1.5, -2), (2.5, 2),
                                      (-2.5, -2), (126.5, 126), (127.49, 127), (127.6, 127),
                                      (-130.0, -127), (1e30, 127)])
def test_int8_round_half_even_and_clamp(t, expect):
    assert oracle.q_int8(t, 1.0) == expect


@pytest.mark.parametrize("absmax", [6.0, 1.0, 3.140625, 1e-3, 1e-38, 2.0 ** -130, 9024.0])
def test_int8_codes_all_bf16_values_vs_torch_round(absmax):
    # scale = absmax/127, inv = 1/scale, code = clamp(round_half_even(v*inv)):
    # torch.round (half to even) on fp32 tensors is the independent routine.
    s = oracle.int8_scale(absmax)
    assert s == float(np.float32(absmax) / np.float32(127.0))
    inv = np.float32(1.0) / np.float32(s)
    v = all_16bit_as_f32(torch.bfloat16)
    v = v[torch.isfinite(v) & (v.abs() <= absmax)]
    t = v * torch.tensor(inv, dtype=torch.float32)
    ref = torch.where(v == 0, torch.zeros_like(t), torch.round(t).clamp(-127, 127)).to(torch.int32)
    sub = slice(None, None, 5)
    ours = torch.tensor([oracle.q_int8(float(x), float(inv)) for x in v[sub].tolist()], dtype=torch.int32)
    assert torch.equal(ours, ref[sub])


# ------------------------------------------------------- 16-bit formats ----

@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_widening_all_patterns_matches_torch(dtype):
    L = oracle.lib()
    fn = L.orc_f16_to_double if dtype == torch.float16 else L.orc_bf16_to_double
    ref = all_16bit_as_f32(dtype).double().numpy()
    ours = np.array([fn(b) for b in range(65536)])
    fin = np.isfinite(ref)
    assert np.array_equal(np.isnan(ref), np.isnan(ours))
    assert np.array_equal(ref[fin], ours[fin])
    assert np.array_equal(ref[np.isinf(ref)], ours[np.isinf(ref)])


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_narrowing_matches_torch_cast(dtype):
    L = oracle.lib()
    fn = L.orc_double_to_f16 if dtype == torch.float16 else L.orc_double_to_bf16
    x = np.concatenate([_random_f32(20000, seed=3),
                        np.array([65504.0, 65519.0, 65520.0, 1e-8, 6e-8, -3e-5, 2.0 ** -25,
                                  3.0 * 2.0 ** -26, 1.00390625, 1.01171875], np.float32)])
    ref = torch.from_numpy(x).to(dtype).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([fn(float(v)) for v in x], dtype=np.uint16)
    bad = np.nonzero(ref != ours)[0]
    assert bad.size == 0, [(x[i], hex(ref[i]), hex(ours[i])) for i in bad[:5]]


def test_massive_activation_values_in_bf16():
    # The pages' massive activations (about 9000 and 13000) are stored in
    # bf16 by the workloads: 8 significant bits give 9024 and 12992.
    f = facts()["massive_activation_text_encoder"]
    L = oracle.lib()
    got = [L.orc_bf16_to_double(L.orc_double_to_bf16(v)) for v in f["values"]]
    assert got == [9024.0, 12992.0]
    # the dynamic per-token FP8 scale of the row holding 12992 is 12992/448 = 29 exactly
    assert oracle.e4m3_scale(12992.0) == 29.0
    assert oracle.q_e4m3(12992.0, 1.0 / 29.0) == 0x7E
    assert math.isclose(oracle.e4m3_scale(9024.0), 9024.0 / 448.0, rel_tol=1e-7)


def test_e4m3_encoder_matches_bitfield_encoder_on_all_fp32():
    """Exhaustive pin of the E4M3 encoder: every one of the 2^32 fp32 bit
    patterns gives the same code from the grid-rounding encoder (double
    arithmetic) and from an integer encoder on the fp32 bit fields (round bit
    and sticky bit on the 24-bit significand)."""
    chunk = 1 << 28
    for lo in range(0, 1 << 32, chunk):
        assert oracle.e4m3_compare_encoders(lo, chunk) == 0, hex(lo)
