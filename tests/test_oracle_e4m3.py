"""Pins of the oracle's E4M3 codec: the OCP table, torch's float8_e4m3fn as a black box, round trips (CPU only)."""
import math

import numpy as np
import torch

from oracle import e4m3


def check_spec_values(golden, decode=e4m3.decode, encode=e4m3.encode):
    for code_hex, val in golden("e4m3_spec_values.txt"):
        code = int(code_hex, 16)
        got = float(decode(np.array([code], dtype=np.uint8))[0])
        if val == "nan":
            assert math.isnan(got)
            continue
        want = float(val)
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), (code_hex, got, want)
        assert int(encode(np.array([want]))[0]) == code, code_hex


def _torch_decode_all():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def check_decode_vs_torch(decode=e4m3.decode):
    ref = _torch_decode_all()
    got = decode(np.arange(256, dtype=np.uint8))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def check_encode_vs_torch(encode=e4m3.encode):
    """Every float32 in a dense sweep of [-448, 448], plus all midpoints between codes, vs torch's RNE cast."""
    vals = _torch_decode_all()
    finite = np.unique(vals[~np.isnan(vals)])
    mids = (finite[:-1] + finite[1:]) / 2
    rng = np.random.default_rng(11)
    sweep = np.concatenate([
        finite, mids, np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
        np.nextafter(mids.astype(np.float32), np.float32(-np.inf)),
        rng.uniform(-448, 448, 200000), rng.standard_normal(200000) * 0.01,
        np.ldexp(rng.uniform(1, 2, 20000), rng.integers(-14, -5, 20000)),
    ]).astype(np.float32)
    sweep = sweep[np.abs(sweep) <= 448]
    ref = torch.from_numpy(sweep).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = encode(sweep)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(sweep[i]), int(got[i]), int(ref[i])) for i in bad[:5]]


def test_spec_values(golden):
    check_spec_values(golden)


def test_decode_all_codes_vs_torch():
    check_decode_vs_torch()


def test_encode_vs_torch():
    check_encode_vs_torch()


def test_round_trip_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    vals = e4m3.decode(codes)
    ok = ~np.isnan(vals)
    assert np.array_equal(e4m3.encode(vals[ok]), codes[ok])


def test_ties_to_even():
    # Halfway between 1.0 (0x38, even mantissa) and 1.125 (0x39) -> 1.0; between 1.125 and 1.25 (0x3a) -> 1.25.
    assert int(e4m3.encode(np.array([1.0625]))[0]) == 0x38
    assert int(e4m3.encode(np.array([1.1875]))[0]) == 0x3A
    # Subnormal midpoint: 1.5 * 2^-9 lies between codes 1 and 2 -> 2 (even).
    assert int(e4m3.encode(np.array([1.5 * 2.0 ** -9]))[0]) == 0x02
    # Below half the smallest subnormal rounds to zero; exactly half rounds to even (zero).
    assert int(e4m3.encode(np.array([2.0 ** -10]))[0]) == 0x00
    assert int(e4m3.encode(np.array([2.0 ** -10 * 1.0001]))[0]) == 0x01


def test_saturation_and_nan():
    big = np.array([448.0, 449.0, 464.0, 480.0, 1e6, np.inf, -1e30, -np.inf], dtype=np.float64)
    assert e4m3.encode(big).tolist() == [0x7E] * 6 + [0xFE] * 2
    assert int(e4m3.encode(np.array([np.nan]))[0]) & 0x7F == 0x7F


def test_quantize_is_float32_multiply_then_encode():
    """quantize(x, s) == torch cast of float32(x) * float32(1/s), for non-power-of-two scales."""
    rng = np.random.default_rng(12)
    x = (rng.standard_normal(100000) * 3).astype(np.float32)
    for scale in (0.011160714, 0.0267, 1.0 / 56.0, 0.5):
        inv = torch.tensor(1.0, dtype=torch.float32) / torch.tensor(scale, dtype=torch.float32)
        prod = torch.from_numpy(x) * inv
        ref = prod.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(e4m3.quantize(x, scale), ref)


def test_tabulated_quantize_equals_the_codec():
    """The full-size GPU tests look the oracle's codes up in quantize's value on every bf16 pattern;
    that lookup must equal quantize applied element by element (random draws, the extremes, NaN/inf)."""
    from tests import oracle_case
    g = torch.Generator().manual_seed(3)
    src = torch.cat([torch.randn(200000, generator=g) * 3, torch.tensor([0.0, -0.0, 1e30, -1e30, 448.0, 500.0,
                                                                          float("inf"), float("nan")])])
    src = src.to(torch.bfloat16)
    for scale in (5.5 / 448, 1.0, 0.013):
        direct = e4m3.quantize(src.float().numpy(), scale)
        assert np.array_equal(oracle_case.e4m3_codes_of_bf16(src, scale), direct)
        assert np.array_equal(oracle_case.e4m3_values(direct, scale), e4m3.dequantize(direct, scale),
                              equal_nan=True)
