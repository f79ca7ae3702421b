"""Shared helpers of the parity tests (no method arithmetic here)."""
from __future__ import annotations

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
    assert err <= max_abs and r <= rel, f"{what}: max-abs {err:.3e} rel-L2 {r:.3e}"
    return err, r


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


def host_cache(s: wl.Spec, centroids, capacity=None):
    cap = s.capacity if capacity is None else capacity
    cap = (cap + 15) // 16 * 16
    return wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, cap, centroids)


def gpu_cache_like(pc, fit=None):
    """Device cache with the same geometry as host cache ``pc``, its packed
    contents copied in, and (optionally) the fitted statistics."""
    import torch
    import bit_kv_cache_centroid_b200 as kv2
    c = kv2.Cache(pc.B, pc.H_kv, pc.d, pc.M, pc.r, pc.capacity,
                  torch.from_numpy(pc.centroids.view(np.int16)))
    c.load_packed(pc)
    if fit is not None:
        c.set_fit(torch.from_numpy(fit.P), torch.from_numpy(fit.w), torch.from_numpy(fit.Wg))
    return c
