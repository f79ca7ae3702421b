"""Pins of the oracle's paged cache addressing (pages of consecutive tokens of
one sequence in a shared pool, found through a block table): a paged copy of
a cache, pages in a shuffled order among spare pages, gives exactly the
decode, chunk and logits of the contiguous cache, and an append into a paged
cache writes exactly the fields of the contiguous append."""
import numpy as np

import workloads as wl


def _basis(H, d, r, seed):
    rng = np.random.default_rng(seed)
    P = np.zeros((H, d, r), np.float32)
    for h in range(H):
        P[h] = np.linalg.qr(rng.standard_normal((d, d)))[0][:, :r]
    return P


def test_paged_copy_decodes_identically(orc):
    s = wl.spec("tiny", d=64, H_kv=2, H_q=4, M=16, r=8, T=512, B=2)
    pc = wl.random_packed_cache(s, T=512, seed=3)
    pg = wl.to_paged(pc, page=128, n_pages=pc.B * pc.capacity // 128 + 3, seed=7)
    P = _basis(2, 64, 8, 1)
    rng = np.random.default_rng(2)
    Q = wl.bf16_bits(rng.standard_normal((2, 4, 64)).astype(np.float32))
    for length in (1, 300, 512):
        assert np.array_equal(orc.decode(pc, P, length, Q, 0.125), orc.decode(pg, P, length, Q, 0.125))
    q = rng.standard_normal(64)
    assert np.array_equal(orc.decode_logits(pc, P, 1, 1, 512, q), orc.decode_logits(pg, P, 1, 1, 512, q))


def test_paged_copy_chunk_identically(orc):
    s = wl.spec("tiny", d=128, H_kv=2, H_q=2, M=16, r=8, T=256, B=1)
    pc = wl.random_packed_cache(s, T=256, seed=4)
    pg = wl.to_paged(pc, page=128, n_pages=pc.B * pc.capacity // 128 + 2, seed=1)
    P = _basis(2, 128, 8, 2)
    rng = np.random.default_rng(5)
    Q = wl.bf16_bits(rng.standard_normal((1, 16, 2, 128)).astype(np.float32))
    Ks = wl.bf16_bits(rng.standard_normal((1, 16, 2, 128)).astype(np.float32))
    Vs = wl.bf16_bits(rng.standard_normal((1, 16, 2, 128)).astype(np.float32))
    rows = np.array([(0, i, h) for i in range(16) for h in range(2)], np.int32)
    assert np.array_equal(orc.chunk(pc, P, 200, Q, Ks, Vs, 8, 0.1, rows), orc.chunk(pg, P, 200, Q, Ks, Vs, 8, 0.1, rows))


def test_append_into_pages_matches_contiguous(orc):
    w = wl.make("tiny")
    s = w.spec
    f = orc.fit(w.Qhist, s.H_kv, s.r)
    cap = (s.T + 127) // 128 * 128
    flat = wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, cap, w.centroids)
    paged = wl.to_paged(wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, cap, w.centroids), 128,
                        s.B * cap // 128 + 2, seed=3)
    for pc in (flat, paged):
        orc.quantize(pc, w.K[:, :s.T], w.V[:, :s.T], 0, s.C, f.P, f.w, f.Wg)
    for name in ("k_code", "v_code", "k_sz", "v_sz", "cidx", "psac"):
        a, pa = getattr(flat, name), getattr(paged, name)
        for b in range(s.B):
            for i in range(cap // 128):
                got = pa[paged.table[b, i]]
                want = a[b, :, i * 128:(i + 1) * 128]
                t_hi = min(128, s.T - i * 128)
                if t_hi > 0:
                    assert np.array_equal(got[:, :t_hi], want[:, :t_hi]), name
