"""Pins the oracle's E4M3 codec and FP8-cache decode to things other than
itself: the encoding's closed forms, torch's float8_e4m3fn cast on its
in-range domain, saturation / tie cases, and round trips."""
import math

import numpy as np
import torch

import oracle
from oracle import fp8


def test_code_values_closed_forms():
    t = fp8.E4M3_TABLE
    assert t[0x00] == 0.0 and math.copysign(1.0, t[0x80]) == -1.0
    assert t[0x38] == 1.0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x01] == 2.0 ** -9          # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9      # largest subnormal
    assert t[0x08] == 2.0 ** -6          # smallest normal
    assert t[0x3F] == 1.875 and t[0x40] == 2.0
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    assert np.isfinite(t).sum() == 254
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)      # codes 0..126 increase with value


def test_table_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    np.testing.assert_array_equal(np.isnan(codes), np.isnan(fp8.E4M3_TABLE))
    ok = ~np.isnan(codes)
    np.testing.assert_array_equal(codes[ok], fp8.E4M3_TABLE[ok])


def test_encode_matches_torch_in_range():
    g = torch.Generator().manual_seed(0)
    x = torch.cat([
        torch.randn(200_000, generator=g) * 3,
        torch.randn(50_000, generator=g) * 1e-2,     # subnormal range
        (torch.rand(50_000, generator=g) * 2 - 1) * 460,
        torch.tensor([0.0, -0.0, 2 ** -10, 3 * 2 ** -11, 1.0625, 1.1875, 447.9, 463.9, -463.9]),
    ]).float()
    want = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = fp8.e4m3_encode(x.numpy())
    np.testing.assert_array_equal(got, want)


def test_ties_go_to_the_even_code():
    # exact midpoints between consecutive codes
    for c in range(0, 0x7E):
        mid = (fp8.E4M3_TABLE[c] + fp8.E4M3_TABLE[c + 1]) / 2
        want = c if c % 2 == 0 else c + 1
        assert fp8.e4m3_encode([mid])[0] == want
        assert fp8.e4m3_encode([-mid])[0] == want | 0x80


def test_saturation_and_nan():
    got = fp8.e4m3_encode([448.0, 464.0, 500.0, 1e30, float("inf"), -1e9, float("-inf")])
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert fp8.e4m3_encode([float("nan")])[0] & 0x7F == 0x7F


def test_round_trip_every_finite_code():
    codes = np.array([c for c in range(256) if not math.isnan(fp8.E4M3_TABLE[c])], dtype=np.uint8)
    np.testing.assert_array_equal(fp8.e4m3_encode(fp8.E4M3_TABLE[codes]), codes)


def test_quantize_divides_in_fp32():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(10_000, generator=g).bfloat16().float()
    scale = 0.0371
    want = (x / torch.tensor(scale, dtype=torch.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    np.testing.assert_array_equal(fp8.quantize(x.numpy(), scale), want.numpy())


def _tie_inputs(scale):
    # x whose fp32 quotient x / scale is exactly the midpoint of two adjacent
    # normal E4M3 values while the exact (fp64) quotient is not: writing
    # rounds the fp32 quotient, so these go to the even code
    vals = fp8.E4M3_TABLE[:0x7F].astype(np.float64)
    out = []
    for i in range(8, 0x7E):
        m = (vals[i] + vals[i + 1]) / 2
        x = np.float32(m * float(scale))
        for _ in range(64):
            x = np.nextafter(x, np.float32(-np.inf))
        for _ in range(129):
            if float(np.float32(x) / scale) == m and float(x) / float(scale) != m:
                out.append(x)
            x = np.nextafter(x, np.float32(np.inf))
    return np.array(out, dtype=np.float32)


def test_quantize_divides_in_fp32_at_ties():
    scale = np.float32(0.0371)
    x = _tie_inputs(scale)
    assert len(x) > 50
    want = (torch.from_numpy(x) / torch.tensor(float(scale), dtype=torch.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8)
    np.testing.assert_array_equal(fp8.quantize(x, float(scale)), want.numpy())


def test_fp8_decode_is_decode_of_the_dequantized_cache():
    rng = np.random.default_rng(3)
    nb, hkv, B, D = 6, 2, 16, 8
    kc = rng.integers(0, 256, (nb, hkv, B, D)).astype(np.uint8)
    vc = rng.integers(0, 256, (nb, hkv, B, D)).astype(np.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x10  # no NaN codes in a real cache
    vc[(vc & 0x7F) == 0x7F] = 0x10
    bt = np.array([[3, 1, 4], [0, 5, 2]])
    q = rng.standard_normal((2, 4, D))
    got = fp8.paged_decode_fp8(q, kc, vc, bt, [40, 17], 0.3, 0.5, 0.25, hkv)
    want = oracle.paged_decode(q, fp8.E4M3_TABLE[kc] * 0.5, fp8.E4M3_TABLE[vc] * 0.25, bt,
                               [40, 17], 0.3, hkv)
    np.testing.assert_array_equal(got, want)
    # v_scale multiplies the output (attention is linear in V)
    twice = fp8.paged_decode_fp8(q, kc, vc, bt, [40, 17], 0.3, 0.5, 0.5, hkv)
    np.testing.assert_allclose(twice, 2 * got, rtol=1e-12, atol=1e-12)
