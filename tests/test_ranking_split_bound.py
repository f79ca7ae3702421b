"""The quantizer's tensor-core ranking feeds each key's products x_c =
fp32(w_c k_c), scaled by 2^e so that max |x| 2^e lies in [2^14, 2^15), to
the tensor cores as fp16 hi = fp16(x 2^e) and lo = fp16(x 2^e - hi). Its
error bound takes |x 2^e - hi - lo| <= 2^-22 |x 2^e| + 2^-25 per channel and
hi, lo finite. These CPU checks pin that split on random, wide-range and
edge values (fp16 round-to-nearest-even as numpy implements it, the same
rounding as the kernel's conversion)."""
import numpy as np


def _split(x32):
    """hi, lo and the scale exponent of one key's products (fp32 array)."""
    mx = np.max(np.abs(x32)).astype(np.float32)
    biased = int((np.array([mx], np.float32).view(np.uint32)[0] >> 23) & 0xFF)
    # the exponent field of the largest |x|: e = 14 - E for a normal maximum,
    # 0 for a zero or subnormal one, limited to [-126, 126]
    e = max(-126, min(126, 14 - (biased - 127))) if biased > 0 else 0
    y = (x32 * np.float32(2.0) ** np.float32(e)).astype(np.float32)
    hi = y.astype(np.float16)
    lo = (y - hi.astype(np.float32)).astype(np.float32).astype(np.float16)
    return y, hi, lo, e, biased > 0


def _check(x32):
    y, hi, lo, e, normal = _split(x32)
    assert np.all(np.isfinite(hi)) and np.all(np.isfinite(lo))
    if normal and e not in (-126, 126):
        assert 2.0 ** 14 <= np.max(np.abs(y)) < 2.0 ** 15
    err = np.abs(y.astype(np.float64) - hi.astype(np.float64) - lo.astype(np.float64))
    bound = 2.0 ** -22 * np.abs(y.astype(np.float64)) + 2.0 ** -25
    assert np.all(err <= bound), float(np.max(err / bound))


def test_split_bound_random_keys():
    rng = np.random.default_rng(5)
    for _ in range(200):
        w = rng.gamma(0.5, 2.0, 128).astype(np.float32)
        k = (rng.standard_normal(128) * rng.choice([1e-3, 1.0, 30.0])).astype(np.float32)
        _check((w * k).astype(np.float32))


def test_split_bound_wide_exponents_and_tiny_channels():
    rng = np.random.default_rng(6)
    for _ in range(200):
        x = (rng.standard_normal(128) * np.exp2(rng.integers(-40, 40, 128))).astype(np.float32)
        _check(x)
    x = np.zeros(128, np.float32)
    x[0] = 1.0
    x[1:] = np.float32(2.0 ** -30)          # far below hi's reach: lo and the absolute term carry them
    _check(x)


def test_split_bound_edge_values():
    _check(np.zeros(128, np.float32))
    _check(np.full(128, np.float32(3.4e38)))                      # e < 0: scaled down exactly
    _check(np.full(128, np.float32(1e-38)))                       # subnormal maximum: e = 0
    _check(np.full(128, np.float32(2.0 ** -120)))                 # e clamped at 126
    x = np.linspace(-1, 1, 128, dtype=np.float32) * np.float32(2.0 ** 15 - 1)
    _check(x)
