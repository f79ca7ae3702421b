"""Pins of the oracle's IEEE 754 binary16 / bfloat16 conversions against
library casts (numpy float16, torch bfloat16) and the definition of directed
rounding (the two neighbours that bracket a value)."""
import numpy as np
import pytest
import torch


def _edge_f32(rng, n):
    x = np.concatenate([
        rng.standard_normal(n).astype(np.float32),
        (rng.standard_normal(n) * 1e-5).astype(np.float32),      # fp16 subnormal range
        (rng.standard_normal(n) * 3e4).astype(np.float32),       # near fp16 overflow
        np.float32([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e30, -1e30,
                    5.96e-8, 2.98e-8, 2.99e-8, 6.1035e-5, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]),
    ])
    # exact halfway points between adjacent fp16 values
    h = rng.integers(0, 0x7bff, n).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    return np.concatenate([x, ((lo + hi) / 2).astype(np.float32)])


def test_f16_nearest_even_matches_numpy(orc):
    x = _edge_f32(np.random.default_rng(1), 3000)
    ref = x.astype(np.float16).view(np.uint16)
    got = np.array([orc.f16_from_f32(v, orc.RND_NEAREST_EVEN) for v in x], np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_f16_directed_rounding_brackets(orc):
    x = _edge_f32(np.random.default_rng(2), 2000)
    x = x[np.abs(x) <= 65504]
    for v in x:
        dn = orc.f32_from_f16(orc.f16_from_f32(v, orc.RND_DOWN))
        up = orc.f32_from_f16(orc.f16_from_f32(v, orc.RND_UP))
        assert dn <= v <= up
        if np.float32(v) == np.float32(np.float16(v)):
            assert dn == up == v
        else:
            # adjacent fp16 values: nothing representable strictly between them
            assert _ordinal(up) - _ordinal(dn) == 1


def _ordinal(v):
    h = int(np.float16(v).view(np.uint16))
    return -(h & 0x7FFF) if h & 0x8000 else h


def test_f16_directed_overflow(orc):
    assert orc.f16_from_f32(1e6, orc.RND_DOWN) == 0x7bff
    assert orc.f16_from_f32(1e6, orc.RND_UP) == 0x7c00
    assert orc.f16_from_f32(-1e6, orc.RND_DOWN) == 0xfc00
    assert orc.f16_from_f32(-1e6, orc.RND_UP) == 0xfbff


def test_f16_decode_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([orc.f32_from_f16(int(b)) for b in bits], np.float32)
    finite = np.isfinite(ref)
    np.testing.assert_array_equal(got[finite], ref[finite])
    assert np.all(np.isnan(got[np.isnan(ref)]))


def test_bf16_nearest_even_matches_torch(orc):
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(3000).astype(np.float32),
                        (rng.standard_normal(500) * 1e-38).astype(np.float32),
                        (rng.standard_normal(500) * 1e38).astype(np.float32),
                        np.float32([3.3895314e38, -3.3895314e38, 0.0, -0.0])])
    # halfway points between adjacent bf16 values
    b = rng.integers(0, 0x7f00, 500).astype(np.uint32)
    x = np.concatenate([x, (((b << 16) | 0x8000).astype(np.uint32)).view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.bf16_from_f32(v) for v in x], np.uint16)
    np.testing.assert_array_equal(got, ref)
    for v in x[:100]:
        bb = orc.bf16_from_f32(v)
        assert orc.f32_from_bf16(bb) == torch.tensor(v).to(torch.bfloat16).float().item()
