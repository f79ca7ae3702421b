"""Pins of the oracle's INT2 group codec (QuantWM article, '1. QSAC': the
residual is quantized to 2 bits with a per-group fp16 scale and zero):
hand-derived cases, the codes-in-range and half-step error invariants, and a
per-element brute force over the four levels."""
import json
import os

import numpy as np
import pytest

GOLD = os.path.join(os.path.dirname(__file__), "golden", "codec_cases.json")


def _expand(expr, n=32):
    return np.array([eval(expr, {}, {"i": i}) for i in range(n)], dtype=np.float64)


def test_golden_codec_cases(orc):
    cases = json.load(open(GOLD))["cases"]
    assert len(cases) >= 4
    for c in cases:
        x = _expand(c["x"]).astype(np.float32)
        s, z, codes, deq = orc.codec_group(x)
        assert s == c["scale_bits"], c["name"]
        assert z == c["zero_bits"], c["name"]
        assert np.float16(c["scale"]).view(np.uint16) == s
        assert np.float16(c["zero"]).view(np.uint16) == z
        np.testing.assert_array_equal(codes, _expand(c["codes"]).astype(np.uint8), err_msg=c["name"])


def _groups(rng, n):
    out = []
    for k in range(n):
        kind = k % 5
        if kind == 0:
            x = rng.standard_normal(32)
        elif kind == 1:
            x = rng.standard_normal(32) * np.exp(rng.uniform(-8, 6)) + rng.uniform(-50, 50)
        elif kind == 2:
            x = np.round(rng.standard_normal(32) * 4) / 4        # many repeats / exact values
        elif kind == 3:
            x = np.full(32, rng.standard_normal())               # constant
        else:
            x = rng.standard_normal(32) * 1e-3 + 1e3             # large offset, tiny spread
        out.append(x.astype(np.float32))
    return out


def test_codec_invariants(orc):
    rng = np.random.default_rng(7)
    for x in _groups(rng, 600):
        s_b, z_b, codes, deq = orc.codec_group(x)
        s = float(np.uint16(s_b).view(np.float16))
        z = float(np.uint16(z_b).view(np.float16))
        assert codes.max() <= 3
        assert z <= x.min()                          # zero rounded down below the minimum
        assert z + 3 * s >= x.max() - 4 * np.spacing(np.float32(abs(x).max()))
        slop = 8 * 2.0 ** -24 * (abs(z) + 3 * s)
        assert np.all(np.abs(deq.astype(np.float64) - x) <= s / 2 + slop + 1e-30)


def test_codec_brute_force_levels(orc):
    """Each code is the level whose dequantized value is nearest to x; an exact
    tie between two levels (within 2 fp32 ulps) may go either way."""
    rng = np.random.default_rng(8)
    ties = 0
    for x in _groups(rng, 600):
        s_b, z_b, codes, deq = orc.codec_group(x)
        s = np.float32(np.uint16(s_b).view(np.float16))
        z = np.float32(np.uint16(z_b).view(np.float16))
        levels = np.array([np.float64(np.float32(l) * s + z) for l in range(4)])
        err = np.abs(levels[None, :] - x.astype(np.float64)[:, None])
        best = err.min(1)
        mine = err[np.arange(32), codes]
        tol = 2 * np.spacing(np.abs(x).astype(np.float32)).astype(np.float64) + 2 * np.spacing(s)
        ok = mine <= best + tol
        assert np.all(ok)
        ties += int(np.sum((mine > best)))
    assert ties < 60


def test_codec_constant_and_zero_scale(orc):
    x = np.full(32, 0.3, np.float32)
    s_b, z_b, codes, deq = orc.codec_group(x)
    s = float(np.uint16(s_b).view(np.float16))
    assert np.all(codes <= 3)
    assert np.all(np.abs(deq - x) <= s / 2 + 1e-7)
    x = np.full(32, 2.5, np.float32)                # fp16-exact constant: scale 0
    s_b, z_b, codes, deq = orc.codec_group(x)
    assert s_b == 0 and np.all(codes == 0) and np.all(deq == 2.5)
