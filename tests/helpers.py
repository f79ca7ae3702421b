"""Shared helpers of the parity tests (no method arithmetic here)."""
from __future__ import annotations

import os

import numpy as np

import workloads as wl


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_attention_close(got, ref, max_abs=2e-3, rel=1e-3, what=""):
    """The attention tolerance: max-abs 2e-3 and relative L2 1e-3 against the
    oracle run on the same dequantized values."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref).max() if got.size else 0.0
    r = rel_l2(got, ref) if got.size else 0.0
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    if os.environ.get("KV2_TEST_REPORT"):
        print(f"[attention error] {what}: max-abs {err:.3e} rel-L2 {r:.3e}")
    assert err <= max_abs and r <= rel, f"{what}: max-abs {err:.3e} rel-L2 {r:.3e}"
    return err, r


def assert_bf16_attention_close(got, ref, max_abs=2e-3, rel=1e-3, what=""):
    """A bf16 output is the kernel's fp32 result rounded to bf16: within the fp32
    tolerance of the oracle plus half a bf16 ulp of the value (the output's own
    rounding, which can fall on the other side of a rounding boundary than the
    rounding of the oracle), and within the relative-L2 tolerance of the bf16
    rounding of the oracle."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    a = np.abs(ref)
    ulp = np.where(a > 0, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-38))) - 7), 2.0 ** -133)
    err = np.abs(got - ref)
    bad = err > max_abs + 0.5 * ulp
    r = rel_l2(got, bf16_round(ref))
    assert not bad.any() and r <= rel, \
        f"{what}: {int(bad.sum())} elements beyond max-abs {max_abs} + ulp/2 (worst {err.max():.3e}); rel-L2 {r:.3e}"
    return float(err.max()), r


def bf16_round(x):
    """fp64/fp32 -> bf16 -> fp32 (round to nearest even) via torch."""
    import torch
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def f16_ulp_diff(a_bits, b_bits):
    """Distance in fp16 ulps between two arrays of fp16 bit patterns."""
    def ordinal(h):
        h = h.astype(np.int32)
        return np.where(h & 0x8000, -(h & 0x7FFF), h & 0x7FFF)
    return np.abs(ordinal(np.asarray(a_bits)) - ordinal(np.asarray(b_bits)))


def to_dev(x, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def host_cache(s: wl.Spec, centroids, capacity=None, psac_fmt=0):
    cap = s.capacity if capacity is None else capacity
    cap = (cap + 15) // 16 * 16
    return wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, cap, centroids, psac_fmt, s.group)


def gpu_cache_like(pc, fit=None):
    """Device cache with the same geometry as host cache ``pc``, its packed
    contents copied in, and (optionally) the fitted statistics."""
    import torch
    import bit_kv_cache_centroid_b200 as kv2
    paged = getattr(pc, "table", None) is not None
    c = kv2.Cache(pc.B, pc.H_kv, pc.d, pc.M, pc.r, pc.capacity,
                  torch.from_numpy(pc.centroids.view(np.int16)), psac_fmt=getattr(pc, "psac_fmt", 0),
                  page_tokens=pc.page if paged else 0, num_pages=pc.k_code.shape[0] if paged else 0,
                  group=getattr(pc, "group", 32))
    c.load_packed(pc)
    if fit is not None:
        c.set_fit(torch.from_numpy(fit.P), torch.from_numpy(fit.w), torch.from_numpy(fit.Wg))
    return c
