"""Pins of the oracle's PSAC coefficients and attention over the packed cache.

PSAC (QuantWM article, '2. PSAC'): with r = d the compensated logits are the
unquantized-Key logits up to the fp16 rounding of the coefficients; with r = 0
they are the plain centre + residual (QVG-style) logits; the coefficients are
the projection of the quantization error on the basis.
Attention: two-pass fp64 softmax over independently unpacked values, the
centroid-only closed form (zero scales), the single-token and empty cases, and
the block-causal frame mask of the chunk call.
"""
import numpy as np
import pytest

import workloads as wl


def unpack_codes(words, d):
    """Format decoding written independently of the oracle: channel c sits in
    word c // 16 at bits 2 (c % 16) .. 2 (c % 16) + 1."""
    c = np.arange(d)
    return (words[..., c // 16] >> (2 * (c % 16)).astype(np.uint32)) & 3


def unpack_sz(sz):
    s = wl.f16_values((sz & 0xFFFF).astype(np.uint16)).astype(np.float64)
    z = wl.f16_values((sz >> 16).astype(np.uint16)).astype(np.float64)
    return s, z


def dequant(pc, b, h, T):
    """Exact dequantized K (centre + residual) and V rows [T][d] in fp64."""
    d = pc.d
    kc = unpack_codes(pc.k_code[b, h, :T], d).astype(np.float64)
    vc = unpack_codes(pc.v_code[b, h, :T], d).astype(np.float64)
    ks, kz = unpack_sz(pc.k_sz[b, h, :T])
    vs, vz = unpack_sz(pc.v_sz[b, h, :T])
    g = np.arange(d) // 32
    mu = wl.f16_values(pc.centroids[h]).astype(np.float64)[pc.cidx[b, h, :T].astype(int)]
    return mu + kc * ks[:, g] + kz[:, g], vc * vs[:, g] + vz[:, g]


def _quantized(orc, r, **ov):
    w = wl.make("tiny", r=r, **ov)
    s = w.spec
    f = orc.fit(w.Qhist, s.H_kv, r)
    pc = wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, r, s.capacity, w.centroids)
    orc.quantize(pc, w.K[:, :s.T], w.V[:, :s.T], 0, s.C, f.P, f.w, f.Wg)
    return w, f, pc


def test_psac_full_rank_restores_exact_key_logits(orc):
    w, f, pc = _quantized(orc, r=64)
    s = w.spec
    keys = wl.bf16_values(w.K).astype(np.float64)
    q = wl.bf16_values(w.Qdec).astype(np.float64)[0]            # [H_q][d]
    for h in range(s.H_kv):
        got = orc.decode_logits(pc, f.P, 0, h, s.T, q[h])
        exact = keys[0, :s.T, h] @ q[h]
        u = q[h] @ f.P[h].astype(np.float64)
        a = wl.f16_values(pc.psac[0, h, :s.T]).astype(np.float64)
        bound = (np.abs(u)[None, :] * np.abs(a)).sum(1) * 2.0 ** -11 \
            + np.abs(q[h]).sum() * np.abs(keys[0, :s.T, h]).max(1) * 2.0 ** -22 + 1e-9
        assert np.all(np.abs(got - exact) <= bound)
        # and PSAC really moved the logits: without it the error is much larger
        khat, _ = dequant(pc, 0, h, s.T)
        qvg = khat @ q[h]
        assert np.abs(qvg - exact).mean() > 20 * np.abs(got - exact).mean()


def test_psac_rank_zero_is_centre_plus_residual(orc):
    w, f, pc = _quantized(orc, r=0)
    s = w.spec
    q = wl.bf16_values(w.Qdec).astype(np.float64)[0]
    for h in range(s.H_kv):
        khat, _ = dequant(pc, 0, h, s.T)
        got = orc.decode_logits(pc, f.P, 0, h, s.T, q[h])
        np.testing.assert_allclose(got, khat @ q[h], rtol=1e-13, atol=1e-12)


def test_psac_coefficients_project_the_error(orc):
    w, f, pc = _quantized(orc, r=8)
    s = w.spec
    keys = wl.bf16_values(w.K).astype(np.float64)
    for h in range(s.H_kv):
        khat, _ = dequant(pc, 0, h, s.T)
        e = keys[0, :s.T, h] - khat                                  # [T][d]
        want = e @ f.P[h].astype(np.float64)                        # [T][r]
        got = wl.f16_values(pc.psac[0, h, :s.T]).astype(np.float64)
        ulp = np.spacing(np.abs(want).astype(np.float16)).astype(np.float64)
        assert np.all(np.abs(got - want) <= ulp + 1e-6 * np.abs(e).sum(1, keepdims=True))


def test_qsac_choice_does_not_depend_on_rank(orc):
    _, _, a = _quantized(orc, r=0)
    _, _, b = _quantized(orc, r=16)
    np.testing.assert_array_equal(a.cidx, b.cidx)
    np.testing.assert_array_equal(a.k_code, b.k_code)
    np.testing.assert_array_equal(a.v_code, b.v_code)


def _softmax_out(logits, vals):
    m = logits.max()
    p = np.exp(logits - m)
    return (p[:, None] * vals).sum(0) / p.sum()


def test_decode_two_pass_softmax(orc):
    w, f, pc = _quantized(orc, r=8)
    s = w.spec
    scale = 1.0 / np.sqrt(s.d)
    out = orc.decode(pc, f.P, s.T, w.Qdec, scale)
    q = wl.bf16_values(w.Qdec).astype(np.float64)
    for hq in range(s.H_q):
        h = hq // s.G
        khat, vhat = dequant(pc, 0, h, s.T)
        u = q[0, hq] @ f.P[h].astype(np.float64)
        a = wl.f16_values(pc.psac[0, h, :s.T]).astype(np.float64)
        lg = (khat @ q[0, hq] + a @ u) * scale
        np.testing.assert_allclose(out[0, hq], _softmax_out(lg, vhat), rtol=1e-10, atol=1e-12)


def test_decode_centroid_only_closed_form(orc):
    """All scales zero: every key is its centre plus its zero, every value its
    zero; PSAC coefficients zero. Attention over centres in closed form."""
    s = wl.spec("tiny", T=40)
    pc = wl.random_packed_cache(s, T=40)
    pc.k_sz[:] &= 0xFFFF0000
    pc.v_sz[:] &= 0xFFFF0000
    pc.psac[:] = 0
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    rng = np.random.default_rng(5)
    Q = wl.bf16_bits(rng.standard_normal((1, s.H_q, s.d)).astype(np.float32))
    out = orc.decode(pc, P, 40, Q, 0.125)
    q = wl.bf16_values(Q).astype(np.float64)
    for h in range(s.H_kv):
        mu = wl.f16_values(pc.centroids[h]).astype(np.float64)[pc.cidx[0, h, :40].astype(int)]
        _, kz = unpack_sz(pc.k_sz[0, h, :40])
        _, vz = unpack_sz(pc.v_sz[0, h, :40])
        g = np.arange(s.d) // 32
        lg = ((mu + kz[:, g]) @ q[0, h]) * 0.125
        np.testing.assert_allclose(out[0, h], _softmax_out(lg, vz[:, g]), rtol=1e-10, atol=1e-12)


def test_decode_single_and_empty(orc):
    s = wl.spec("tiny", T=8)
    pc = wl.random_packed_cache(s, T=8)
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    Q = wl.bf16_bits(np.ones((1, s.H_q, s.d), np.float32))
    one = orc.decode(pc, P, 1, Q, 0.1)
    for h in range(s.H_kv):
        _, vhat = dequant(pc, 0, h, 1)
        np.testing.assert_allclose(one[0, h], vhat[0], rtol=1e-14)
    assert np.all(orc.decode(pc, P, 0, Q, 0.1) == 0.0)


def test_chunk_mask_and_dense_self_attention(orc):
    """Empty cache: each query attends densely (fp64) to the self keys of its
    own and earlier frames; values enter at fp16 operand precision."""
    s = wl.spec("tiny", T=0, Nq=24, frame_tokens=8, H_q=4, H_kv=2)
    rng = np.random.default_rng(6)
    Q = wl.bf16_bits(rng.standard_normal((1, 24, 4, s.d)).astype(np.float32))
    Ks = wl.bf16_bits(rng.standard_normal((1, 24, 2, s.d)).astype(np.float32))
    Vs = wl.bf16_bits(rng.standard_normal((1, 24, 2, s.d)).astype(np.float32))
    pc = wl.random_packed_cache(s, T=0)
    rows = np.array([(0, i, hq) for i in range(24) for hq in range(4)], np.int32)
    out = orc.chunk(pc, np.zeros((2, s.d, s.r), np.float32), 0, Q, Ks, Vs, 8, 0.2, rows)
    q = wl.bf16_values(Q).astype(np.float64)
    k = wl.bf16_values(Ks).astype(np.float64)
    v = wl.f16_values(wl.f16_bits(wl.bf16_values(Vs))).astype(np.float64)
    for n, (_, i, hq) in enumerate(rows):
        h = hq // 2
        vis = (i // 8 + 1) * 8
        lg = k[0, :vis, h] @ q[0, i, hq] * 0.2
        np.testing.assert_allclose(out[n], _softmax_out(lg, v[0, :vis, h]), rtol=1e-10, atol=1e-12)


def test_chunk_cache_part_equals_decode_when_exact(orc):
    """Cache values chosen so the chunk's fp16 operands are exact, and self
    keys that no query can select: the chunk call reduces to decode."""
    s = wl.spec("tiny", T=48, Nq=8, frame_tokens=4, r=8)
    pc = wl.random_packed_cache(s, T=48)
    rng = np.random.default_rng(9)
    # scale/zero/centres on a coarse binary grid -> exact in bf16/fp16
    sc = wl.f16_bits(rng.integers(1, 8, pc.k_sz.shape) / 8.0).astype(np.uint32)
    ze = wl.f16_bits(-rng.integers(0, 8, pc.k_sz.shape) / 8.0).astype(np.uint32)
    pc.k_sz[:] = sc | (ze << 16)
    pc.v_sz[:] = sc | (ze << 16)
    pc.centroids = wl.f16_bits(rng.integers(-8, 8, pc.centroids.shape) / 4.0)
    pc.psac[:] = wl.f16_bits(rng.integers(-4, 4, pc.psac.shape) / 16.0)
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    for h in range(s.H_kv):
        P[h, :s.r, :] = np.eye(s.r)                  # qP = first r channels (exact in fp16)
    qf = np.zeros((1, 8, s.H_q, s.d), np.float32)
    qf[..., 0] = 2.0
    qf[..., 1:] = rng.integers(-3, 4, qf[..., 1:].shape) / 4.0
    Q = wl.bf16_bits(qf)
    Ks = np.zeros((1, 8, s.H_kv, s.d), np.float32)
    Ks[..., 0] = -4000.0
    Ks = wl.bf16_bits(Ks)
    Vs = wl.bf16_bits(np.ones((1, 8, s.H_kv, s.d), np.float32))
    rows = np.array([(0, i, hq) for i in range(8) for hq in range(s.H_q)], np.int32)
    out = orc.chunk(pc, P, 48, Q, Ks, Vs, 4, 0.125, rows)
    for n, (_, i, hq) in enumerate(rows):
        dec = orc.decode(pc, P, 48, Q[:, i], 0.125)[0, hq]
        np.testing.assert_allclose(out[n], dec, rtol=1e-12, atol=1e-12)


def test_chunk_operand_rounding_hand_derived(orc):
    """Two cached tokens whose chunk operands round (fp16 arithmetic, one
    rounding per operation; derived by hand):
      K_hat = fp16(code s + fp16(z + mu)): z = 1024, mu = 0.25, s = 0.5.
        token 0, code 1: fp16(0.5 + fp16(1024.25) = 1024) = fp16(1024.5) =
        1024 (a tie, to even; the exact key is 1024.75);
        token 1, code 0: fp16(0 + 1024) = 1024 (exact 1024.25).
      So the chunk's two logits are equal and token 0 takes weight 1/2 exactly,
      where decode (exact keys) sees a gap of 0.5 * sm_scale.
      V_hat = fp16(code s + z) in channel 32 (group 1): token 0 code 1, s = 1,
        z = 2048: fp16(2049) = 2048 (a tie, to even); token 1: 0.
      Channel 0 of V: token 0 has zero 1, token 1 zero 0.
    A self key of -4000 on channel 0 takes no weight (logit -500)."""
    d = 64
    f16 = lambda x: int(np.float16(x).view(np.uint16))
    cent = np.zeros((1, 1, d), np.uint16)
    cent[0, 0, 0] = f16(0.25)
    pc = wl.PackedCache.empty(1, 1, d, 1, 0, 16, cent)
    pc.k_code[0, 0, 0, 0] = 1                          # token 0, channel 0: code 1
    pc.k_sz[0, 0, :2, 0] = f16(0.5) | (f16(1024.0) << 16)
    pc.v_code[0, 0, 0, 2] = 1                          # token 0, channel 32: code 1
    pc.v_sz[0, 0, 0, 0] = f16(0.0) | (f16(1.0) << 16)
    pc.v_sz[0, 0, 0, 1] = f16(1.0) | (f16(2048.0) << 16)
    q = np.zeros((1, 1, 1, d), np.float32)
    q[..., 0] = 1.0
    Q = wl.bf16_bits(q)
    Ks = np.zeros((1, 1, 1, d), np.float32)
    Ks[..., 0] = -4000.0
    Vs = np.zeros((1, 1, 1, d), np.float32)
    P = np.zeros((1, d, 0), np.float32)
    scale = 0.125
    out = orc.chunk(pc, P, 2, Q, wl.bf16_bits(Ks), wl.bf16_bits(Vs), 1, scale, np.array([(0, 0, 0)], np.int32))[0]
    assert out[0] == 0.5
    assert out[32] == 1024.0
    dec = orc.decode(pc, P, 2, Q[:, 0], scale)[0, 0]
    p0 = 1.0 / (1.0 + np.exp(-0.5 * scale))          # exact keys 1024.75 and 1024.25
    np.testing.assert_allclose(dec[0], p0, rtol=1e-14)
    np.testing.assert_allclose(dec[32], p0 * 2049.0, rtol=1e-14)


def test_chunk_psac_query_rounding_hand_derived(orc):
    """The chunk's PSAC operand u = fp16(q P): with q = e_0 and P[0][0] =
    fp32(1/3) = 0.3333333432674408, u = 0.333251953125 (fp16 of 1/3, rounded
    down). Two cached tokens identical but for their coefficient (1 and 0):
    the chunk weights token 0 by sigmoid(u * scale), decode by
    sigmoid(fp32(1/3) * scale); the values are 1 and 0 in channel 0."""
    d = 64
    f16 = lambda x: int(np.float16(x).view(np.uint16))
    pc = wl.PackedCache.empty(1, 1, d, 1, 8, 16, np.zeros((1, 1, d), np.uint16))
    pc.psac[0, 0, 0, 0] = f16(1.0)
    pc.v_sz[0, 0, 0, 0] = f16(1.0) << 16                 # token 0: values 1 in channels 0..31
    P = np.zeros((1, d, 8), np.float32)
    P[0, 0, 0] = np.float32(1.0 / 3.0)
    q = np.zeros((1, 1, 1, d), np.float32)
    q[..., 0] = 1.0
    Q = wl.bf16_bits(q)
    Ks = np.zeros((1, 1, 1, d), np.float32)
    Ks[..., 0] = -4000.0
    scale = 2.0
    out = orc.chunk(pc, P, 2, Q, wl.bf16_bits(Ks), wl.bf16_bits(np.zeros((1, 1, 1, d), np.float32)), 1, scale,
                    np.array([(0, 0, 0)], np.int32))[0]
    u16 = 0.333251953125
    assert float(np.float16(1.0 / 3.0)) == u16
    np.testing.assert_allclose(out[0], 1.0 / (1.0 + np.exp(-u16 * scale)), rtol=1e-14)
    dec = orc.decode(pc, P, 2, Q[:, 0], scale)[0, 0]
    np.testing.assert_allclose(dec[0], 1.0 / (1.0 + np.exp(-float(np.float32(1.0 / 3.0)) * scale)), rtol=1e-14)
