"""Pins of the oracle's INT8 PSAC coefficients (one fp16 scale per token; the
compensation information of QuantWM article "2. PSAC" stored compactly).

* quantizing the same keys in both formats gives the same codes, centres and
  scales/zeros (only the coefficients' storage differs);
* every int8 code is within +-127 and the largest is 126 or 127 (the scale is
  the fp16 round-up of max|a| / 127);
* code * scale is within half a scale step (plus the fp16 coefficient's own
  half ulp) of the fp16-format coefficient;
* decode logits of the two formats differ by at most sum_i |u_i| times that
  bound; on a grid where code * scale is exact both formats give the same
  decode output.
"""
import numpy as np

import workloads as wl


def _quantized_pair(orc):
    w = wl.make("tiny")
    s = w.spec
    f = orc.fit(w.Qhist, s.H_kv, s.r)
    caches = []
    for fmt in (0, 1):
        pc = wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, s.capacity, w.centroids, psac_fmt=fmt)
        orc.quantize(pc, w.K[:, :s.T], w.V[:, :s.T], 0, s.C, f.P, f.w, f.Wg)
        caches.append(pc)
    return w, s, f, caches


def test_same_codes_and_bounded_int8_coefficients(orc):
    w, s, f, (p16, p8) = _quantized_pair(orc)
    T = s.T
    for name in ("k_code", "v_code", "k_sz", "v_sz", "cidx"):
        assert np.array_equal(getattr(p16, name)[:, :, :T], getattr(p8, name)[:, :, :T])
    a16 = wl.f16_values(p16.psac[:, :, :T]).astype(np.float64)
    q = p8.psac[:, :, :T].astype(np.int32)
    sc = wl.f16_values(p8.psac_scale[:, :, :T]).astype(np.float64)
    assert np.all(np.abs(q) <= 127)
    nz = np.abs(a16).max(-1) > 0
    assert np.all(np.isin(np.abs(q).max(-1)[nz], (126, 127)))
    ulp = np.spacing(np.abs(a16).astype(np.float16)).astype(np.float64)
    err = np.abs(q * sc[..., None] - a16)
    assert np.all(err <= 0.5 * sc[..., None] * (1 + 1e-6) + 0.5 * ulp + 1e-12)


def test_decode_logits_within_the_coefficient_bound(orc):
    w, s, f, (p16, p8) = _quantized_pair(orc)
    rng = np.random.default_rng(3)
    q = rng.standard_normal(s.d)
    u = np.abs(q @ f.P[0].astype(np.float64))
    lg16 = orc.decode_logits(p16, f.P, 0, 0, s.T, q)
    lg8 = orc.decode_logits(p8, f.P, 0, 0, s.T, q)
    sc = wl.f16_values(p8.psac_scale[0, 0, :s.T]).astype(np.float64)
    a16 = wl.f16_values(p16.psac[0, 0, :s.T]).astype(np.float64)
    ulp = np.spacing(np.abs(a16).astype(np.float16)).astype(np.float64)
    bound = ((0.5 * sc[:, None] + 0.5 * ulp) * u[None, :]).sum(-1) * (1 + 1e-6) + 1e-12
    assert np.all(np.abs(lg16 - lg8) <= bound)
    assert np.any(lg16 != lg8)                      # the storage really differs


def test_exact_grid_gives_identical_decode(orc):
    s = wl.spec("tiny", T=40, r=8)
    p8 = wl.random_packed_cache(s, T=40, psac_fmt=1)
    p8.psac_scale[:] = wl.f16_bits(np.full(p8.psac_scale.shape, 1.0 / 64))   # code * scale exact in fp16
    p16 = wl.PackedCache(p8.B, p8.H_kv, p8.d, p8.M, p8.r, p8.capacity, p8.k_code, p8.v_code, p8.k_sz, p8.v_sz,
                         p8.cidx, wl.f16_bits(p8.psac.astype(np.float64) / 64), p8.centroids)
    rng = np.random.default_rng(8)
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    for h in range(s.H_kv):
        P[h] = np.linalg.qr(rng.standard_normal((s.d, s.d)))[0][:, :s.r]
    Q = wl.bf16_bits(rng.standard_normal((s.B, s.H_q, s.d)).astype(np.float32))
    assert np.array_equal(orc.decode(p8, P, 40, Q, 0.125), orc.decode(p16, P, 40, Q, 0.125))
