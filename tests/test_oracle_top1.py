"""Pins of the oracle's retrieval helpers (most-attended token per query; the
retrieval shift that QuantWM's introduction and Table 1 discuss).

* on a packed cache whose dequantized keys are exact in bf16 and without
  PSAC, the packed argmax equals the dense argmax over those keys, computed
  by a plain fp64 dot product (two independent routes to the same logits);
* a key planted as a large multiple of the query wins in both;
* length 0 gives -1.
"""
import numpy as np

import workloads as wl


def _exact_cache(rng, s, T):
    pc = wl.random_packed_cache(s, T=T, seed=5)
    ng = s.d // 32
    sc = wl.f16_bits(rng.integers(1, 4, pc.k_sz.shape) / 4.0).astype(np.uint32)
    ze = wl.f16_bits(-rng.integers(0, 4, pc.k_sz.shape) / 4.0).astype(np.uint32)
    pc.k_sz[:] = sc | (ze << 16)
    pc.centroids = wl.f16_bits(rng.integers(-8, 8, pc.centroids.shape) / 4.0)
    return pc, ng


def _dequant(pc, T):
    """The keys of the cache as fp64 (centre + code * s + z), [B][T][H][d]."""
    B, H, d = pc.B, pc.H_kv, pc.d
    out = np.zeros((B, T, H, d))
    cent = wl.f16_values(pc.centroids).astype(np.float64)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                words = pc.k_code[b, h, t]
                codes = np.array([(words[c // 16] >> (2 * (c % 16))) & 3 for c in range(d)], np.float64)
                sz = pc.k_sz[b, h, t]
                s = wl.f16_values((sz & 0xFFFF).astype(np.uint16)).astype(np.float64)
                z = wl.f16_values((sz >> 16).astype(np.uint16)).astype(np.float64)
                out[b, t, h] = cent[h, pc.cidx[b, h, t]] + codes * np.repeat(s, 32) + np.repeat(z, 32)
    return out


def test_packed_argmax_equals_dense_argmax_on_exact_keys(orc):
    rng = np.random.default_rng(21)
    s = wl.spec("tiny", d=64, H_kv=2, H_q=4, M=16, r=0, T=300, B=2)
    pc, _ = _exact_cache(rng, s, 300)
    K = _dequant(pc, 300)
    Kb = wl.bf16_bits(K.astype(np.float32))
    assert np.array_equal(wl.bf16_values(Kb).astype(np.float64), K)        # exact in bf16
    Q = wl.bf16_bits(rng.integers(-4, 5, (2, 5, 4, 64)).astype(np.float32) / 4.0)
    top_p, lg_p = orc.decode_top1(pc, np.zeros((2, 64, 0), np.float32), 300, Q)
    top_d, lg_d = orc.dense_top1(Kb, Q)
    np.testing.assert_allclose(lg_p, lg_d, rtol=0, atol=1e-9)
    assert np.array_equal(top_p, top_d)


def test_planted_key_wins(orc):
    rng = np.random.default_rng(4)
    K = rng.standard_normal((1, 50, 1, 32)).astype(np.float32)
    q = rng.standard_normal(32).astype(np.float32)
    K[0, 37, 0] = 5.0 * q
    top, _ = orc.dense_top1(wl.bf16_bits(K), wl.bf16_bits(q[None, None, None, :]))
    assert top[0, 0, 0] == 37


def test_empty_length(orc):
    s = wl.spec("tiny", d=64, H_kv=1, H_q=1, M=16, r=8, T=16, B=1)
    pc = wl.random_packed_cache(s, T=16)
    Q = wl.bf16_bits(np.ones((1, 2, 1, 64), np.float32))
    top, _ = orc.decode_top1(pc, np.zeros((1, 64, 8), np.float32), 0, Q)
    assert np.all(top == -1)
