"""Pins of the oracle at quantization groups of 64 and 128 channels (one fp16
scale and zero per group of consecutive channels; QuantWM article, '1. QSAC',
and the compression count of its evaluation, which fixes no group size):

* each stored (scale, zero) covers its own group of channels and no more: the
  zero at or just below the group's minimum, zero + 3 scale at or above its
  maximum, the scale within fp16 rounding of a third of its range, and every
  dequantized channel within half a scale of its value;
* residuals that are constant on each group reconstruct exactly (scale 0, no
  PSAC coefficient), while a group spanning two different constants does not;
* with one group per row, the QSAC choice among all centres is the centre of
  least residual range (the estimate reduces to W s^2);
* W over one whole-row group is the trace of the query Gram matrix (the sum of
  its eigenvalues), and W of a larger group is the sum of its channels' w;
* attention over a cache with groups of 64 or 128 equals, bit for bit,
  attention over the same cache written with groups of 32 (each scale and
  zero repeated) for decode, chunk and logits; decode also matches a
  two-pass softmax over independently unpacked rows;
* centre fitting assigns exactly as the append does at the same group size.
"""
import dataclasses

import numpy as np
import pytest

import workloads as wl


def unpack_codes(words, d):
    """Channel c sits in word c // 16 at bits 2 (c % 16) .. 2 (c % 16) + 1."""
    c = np.arange(d)
    return (words[..., c // 16] >> (2 * (c % 16)).astype(np.uint32)) & 3


def unpack_sz(sz):
    s = wl.f16_values((sz & 0xFFFF).astype(np.uint16)).astype(np.float64)
    z = wl.f16_values((sz >> 16).astype(np.uint16)).astype(np.float64)
    return s, z


def _basis(H, d, r, seed):
    rng = np.random.default_rng(seed)
    P = np.zeros((H, d, r), np.float32)
    for h in range(H):
        P[h] = np.linalg.qr(rng.standard_normal((d, d)))[0][:, :r]
    return P


def _quantized(orc, group, C=None, **ov):
    w = wl.make("tiny", **ov)
    s = w.spec
    f = orc.fit(w.Qhist, s.H_kv, s.r, group)
    pc = wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, s.capacity, w.centroids, group=group)
    dbg = orc.quantize(pc, w.K[:, :s.T], w.V[:, :s.T], 0, s.C if C is None else C, f.P, f.w, f.Wg,
                       debug=True)
    return w, f, pc, dbg


@pytest.mark.parametrize("group", [32, 64, 128])
def test_each_scale_and_zero_cover_their_own_group(orc, group):
    w, f, pc, _ = _quantized(orc, group, d=128, T=160)
    s = w.spec
    ng = s.d // group
    keys = wl.bf16_values(w.K)[0, :s.T]                 # fp32 [T][H][d]
    vals = wl.bf16_values(w.V)[0, :s.T]
    mu = wl.f16_values(w.centroids)                     # fp32 [H][M][d]
    for h in range(s.H_kv):
        # residuals in fp32, formed as the append forms them
        x = keys[:, h] - mu[h][pc.cidx[0, h, :s.T].astype(int)]
        for name, rows in (("k", x), ("v", vals[:, h])):
            sc, ze = unpack_sz(getattr(pc, name + "_sz")[0, h, :s.T])       # [T][ng]
            xg = rows.astype(np.float64).reshape(s.T, ng, group)
            lo, hi = xg.min(-1), xg.max(-1)
            ulp_lo = np.spacing(np.abs(lo).astype(np.float16)).astype(np.float64)
            assert np.all(ze <= lo), name
            assert np.all(ze >= lo - 2 * ulp_lo), name
            top = 4 * np.spacing(np.abs(xg).max(-1).astype(np.float32)).astype(np.float64)
            assert np.all(ze + 3 * sc >= hi - top), name
            assert np.all(sc <= (hi - lo + 2 * ulp_lo) / 3 * (1 + 2.0 ** -9) + 2.0 ** -24), name
            codes = unpack_codes(getattr(pc, name + "_code")[0, h, :s.T], s.d).reshape(s.T, ng, group)
            deq = codes * sc[..., None] + ze[..., None]
            slop = 8 * 2.0 ** -24 * (np.abs(ze) + 3 * sc)
            assert np.all(np.abs(deq - xg) <= sc[..., None] / 2 + slop[..., None] + 1e-30), name


def _block_constant_cache(orc, group, block, seed=3):
    """Keys and values constant on blocks of `block` channels (fp16-exact
    values, neighbouring blocks different), one zero centre, quantized with
    groups of `group`."""
    rng = np.random.default_rng(seed)
    d, T, r = 128, 48, 8
    levels = np.array([-2.5, -1.0, -0.375, 0.0, 0.25, 1.5, 3.0], np.float32)
    nb = d // block
    pick = np.zeros((2, T, nb), int)
    for i in range(2):
        for t in range(T):
            row = rng.choice(len(levels), nb, replace=False)      # blocks differ
            pick[i, t] = row
    K = np.repeat(levels[pick[0]], block, axis=-1).reshape(1, T, 1, d)
    V = np.repeat(levels[pick[1]], block, axis=-1).reshape(1, T, 1, d)
    cent = np.zeros((1, 1, d), np.uint16)
    P = _basis(1, d, r, seed)
    wts = np.ones((1, d), np.float32)
    Wg = np.full((1, d // group), float(group), np.float32)
    pc = wl.PackedCache.empty(1, 1, d, 1, r, T, cent, group=group)
    orc.quantize(pc, wl.bf16_bits(K), wl.bf16_bits(V), 0, 1, P, wts, Wg)
    return pc, K[0, :, 0].astype(np.float64), V[0, :, 0].astype(np.float64), P


@pytest.mark.parametrize("group", [32, 64])
def test_group_constant_residuals_reconstruct_exactly(orc, group):
    pc, K, V, P = _block_constant_cache(orc, group, block=64)
    assert np.all(pc.k_sz & 0xFFFF == 0) and np.all(pc.v_sz & 0xFFFF == 0)
    assert np.all(pc.k_code == 0) and np.all(pc.v_code == 0)
    assert np.all(pc.psac == 0)
    _, kz = unpack_sz(pc.k_sz[0, 0])
    _, vz = unpack_sz(pc.v_sz[0, 0])
    g = np.arange(128) // group
    np.testing.assert_array_equal(kz[:, g], K)
    np.testing.assert_array_equal(vz[:, g], V)
    q = np.random.default_rng(1).standard_normal(128)
    np.testing.assert_allclose(orc.decode_logits(pc, P, 0, 0, K.shape[0], q), K @ q, rtol=1e-14, atol=1e-11)


def test_group_spanning_two_constants_is_not_exact(orc):
    """One group over two constant blocks: a non-zero scale, the lower block
    at code 0 (its value is the fp16 zero), the upper at code 3; the
    reconstruction is exact only where a third of the gap is an fp16 value."""
    pc, K, V, P = _block_constant_cache(orc, 128, block=64)
    s, z = unpack_sz(pc.k_sz[0, 0])
    assert np.all(s > 0)
    codes = unpack_codes(pc.k_code[0, 0], 128).reshape(-1, 2, 64)
    upper = K[:, ::64].argmax(1)                                  # block of the larger value
    for t in range(K.shape[0]):
        assert np.all(codes[t, upper[t]] == 3) and np.all(codes[t, 1 - upper[t]] == 0), t
    deq = unpack_codes(pc.k_code[0, 0], 128) * s[:, :1] + z[:, :1]
    err = np.abs(deq - K).max(1)
    gap3 = (K.max(1) - K.min(1)) / 3
    exact16 = gap3.astype(np.float16).astype(np.float64) == gap3
    assert np.all((err == 0) == exact16)
    assert np.any(err > 0) and np.any(pc.psac != 0)


def test_single_group_choice_is_least_residual_range(orc):
    """group = d: E_j = W s_j^2 is monotone in the scale, so with every centre
    a candidate the chosen centre's scale is the least, and its residual range
    the least up to fp16 rounding of the scales."""
    w, f, pc, _ = _quantized(orc, 64, C=16, T=96)
    s = w.spec
    keys = wl.bf16_values(w.K)[0, :s.T]
    mu = wl.f16_values(w.centroids)
    near = 0
    for h in range(s.H_kv):
        for t in range(s.T):
            x = (keys[t, h][None, :] - mu[h]).astype(np.float64)          # [M][d]
            lo, hi = x.min(1), x.max(1)
            ulp_lo = np.spacing(np.abs(lo).astype(np.float16)).astype(np.float64)
            upper = (hi - lo + 2 * ulp_lo) / 3 * (1 + 2.0 ** -9) + 2.0 ** -24
            j = int(pc.cidx[0, h, t])
            sc = float(unpack_sz(pc.k_sz[0, h, t])[0][0])
            assert sc <= upper.min() * (1 + 1e-7), (h, t)
            assert sc >= (hi[j] - lo[j]) / 3 * (1 - 2.0 ** -20), (h, t)
            rng_ = hi - lo
            if j != int(rng_.argmin()):
                jm = int(rng_.argmin())
                assert rng_[j] <= (rng_[jm] + 2 * ulp_lo[jm]) * (1 + 2.0 ** -8), (h, t, j, jm)
                near += 1
    assert near <= 8


def test_whole_row_W_is_the_trace(orc):
    w = wl.make("tiny", d=128)
    s = w.spec
    f32 = orc.fit(w.Qhist, s.H_kv, s.r, 32)
    f64 = orc.fit(w.Qhist, s.H_kv, s.r, 64)
    f128 = orc.fit(w.Qhist, s.H_kv, s.r, 128)
    for f in (f64, f128):
        np.testing.assert_array_equal(f.w, f32.w)
        np.testing.assert_array_equal(f.P, f32.P)
        np.testing.assert_array_equal(f.evals, f32.evals)
    trace = f32.evals.sum(1)
    np.testing.assert_allclose(f128.Wg[:, 0], trace, rtol=2e-5)
    np.testing.assert_allclose(f32.Wg.astype(np.float64).sum(1), trace, rtol=2e-5)
    wsum = f32.w.astype(np.float64).reshape(s.H_kv, 2, 64).sum(-1)
    np.testing.assert_allclose(f64.Wg, wsum, rtol=4e-6)


def _as_group32(pc):
    """The same cache with every (scale, zero) repeated over its 32-channel
    sub-groups."""
    rep = pc.group // 32
    return dataclasses.replace(pc, k_sz=np.repeat(pc.k_sz, rep, axis=-1),
                               v_sz=np.repeat(pc.v_sz, rep, axis=-1), group=32)


@pytest.mark.parametrize("group,fmt", [(64, 0), (128, 0), (128, 1)])
def test_attention_equals_the_repeated_group32_cache(orc, group, fmt):
    s = wl.spec("tiny", d=128, H_kv=2, H_q=4, M=16, r=8, T=300, B=2, group=group)
    pc = wl.random_packed_cache(s, T=300, seed=group + fmt, psac_fmt=fmt)
    assert pc.k_sz.shape[-1] == 128 // group
    p32 = _as_group32(pc)
    P = _basis(2, 128, 8, 4)
    rng = np.random.default_rng(6)
    Q = wl.bf16_bits(rng.standard_normal((2, 4, 128)).astype(np.float32))
    for length in (1, 177, 300):
        assert np.array_equal(orc.decode(pc, P, length, Q, 0.09), orc.decode(p32, P, length, Q, 0.09))
    q = rng.standard_normal(128)
    assert np.array_equal(orc.decode_logits(pc, P, 1, 1, 300, q), orc.decode_logits(p32, P, 1, 1, 300, q))
    Qc = wl.bf16_bits(rng.standard_normal((2, 12, 4, 128)).astype(np.float32))
    Ks = wl.bf16_bits(rng.standard_normal((2, 12, 2, 128)).astype(np.float32))
    Vs = wl.bf16_bits(rng.standard_normal((2, 12, 2, 128)).astype(np.float32))
    rows = np.array([(b, i, hq) for b in range(2) for i in range(0, 12, 3) for hq in range(4)], np.int32)
    assert np.array_equal(orc.chunk(pc, P, 250, Qc, Ks, Vs, 4, 0.09, rows),
                          orc.chunk(p32, P, 250, Qc, Ks, Vs, 4, 0.09, rows))


def test_decode_two_pass_softmax_group128(orc):
    w, f, pc, _ = _quantized(orc, 128, d=128, T=200)
    s = w.spec
    scale = 1.0 / np.sqrt(s.d)
    out = orc.decode(pc, f.P, s.T, w.Qdec, scale)
    q = wl.bf16_values(w.Qdec).astype(np.float64)
    for hq in range(s.H_q):
        h = hq // s.G
        kc = unpack_codes(pc.k_code[0, h, :s.T], s.d).astype(np.float64)
        vc = unpack_codes(pc.v_code[0, h, :s.T], s.d).astype(np.float64)
        ks, kz = unpack_sz(pc.k_sz[0, h, :s.T])
        vs, vz = unpack_sz(pc.v_sz[0, h, :s.T])
        mu = wl.f16_values(w.centroids[h]).astype(np.float64)[pc.cidx[0, h, :s.T].astype(int)]
        khat = mu + kc * ks + kz                          # one group per row: [T][1] broadcasts
        vhat = vc * vs + vz
        u = q[0, hq] @ f.P[h].astype(np.float64)
        a = wl.f16_values(pc.psac[0, h, :s.T]).astype(np.float64)
        lg = (khat @ q[0, hq] + a @ u) * scale
        p = np.exp(lg - lg.max())
        np.testing.assert_allclose(out[0, hq], (p[:, None] * vhat).sum(0) / p.sum(), rtol=1e-10, atol=1e-12)


def test_centre_fitting_assigns_as_the_append(orc):
    assigns = {}
    for group in (32, 128):
        w, f, pc, _ = _quantized(orc, group, d=128, T=128)
        s = w.spec
        X = np.ascontiguousarray(w.K[0, :s.T])                    # [n][H_kv][d]
        _, a = orc.fit_centroids(X, s.M, s.C, f.w, f.Wg, w.centroids, iters=1, group=group)
        np.testing.assert_array_equal(a.T, pc.cidx[0, :, :s.T].astype(np.int32))
        assigns[group] = a
    # the group size reaches the decision
    assert np.any(assigns[32] != assigns[128])


def test_bad_group_is_refused(orc):
    w = wl.make("tiny")
    s = w.spec
    with pytest.raises(ValueError):
        orc.fit(w.Qhist, s.H_kv, s.r, 48)
    f = orc.fit(w.Qhist, s.H_kv, s.r)
    pc = wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, s.capacity, w.centroids, group=64)
    with pytest.raises(ValueError):
        orc.quantize(pc, w.K[:, :s.T], w.V[:, :s.T], 0, s.C, f.P, f.w, f.Wg)    # W of groups of 32
