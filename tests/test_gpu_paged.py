"""GPU paged cache (pages of consecutive tokens from a shared pool, found
through a block table): the same tokens stored as shuffled pages among spare
pages give bit-identical decode, chunk and top-1 results to the contiguous
cache, an append through the table writes the same fields as a contiguous
append, and the paged decode matches the oracle."""
import numpy as np
import pytest
import torch

import workloads as wl
from helpers import assert_attention_close, gpu_cache_like, to_dev

pytestmark = pytest.mark.gpu


def _padded(pc, page):
    """pc with its capacity rounded up to a whole number of pages."""
    cap = (pc.capacity + page - 1) // page * page
    if cap == pc.capacity:
        return pc
    out = wl.PackedCache.empty(pc.B, pc.H_kv, pc.d, pc.M, pc.r, cap, pc.centroids, pc.psac_fmt)
    for n in ("k_code", "v_code", "k_sz", "v_sz", "cidx", "psac", "psac_scale"):
        a = getattr(pc, n)
        if a is not None:
            getattr(out, n)[:, :, :pc.capacity] = a
    return out


def _basis(H, d, r, seed):
    rng = np.random.default_rng(seed)
    P = np.zeros((H, d, r), np.float32)
    for h in range(H):
        P[h] = np.linalg.qr(rng.standard_normal((d, d)))[0][:, :r]
    return P


@pytest.mark.parametrize("page,G,M,r,T,length,fmt", [
    (128, 4, 64, 8, 1500, 1437, 0),
    (256, 1, 512, 16, 1300, 1300, 1),
])
def test_decode_and_top1_identical_to_contiguous(orc, page, G, M, r, T, length, fmt):
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=128, H_kv=2, H_q=2 * G, M=M, r=r, T=T, B=2)
    pc = _padded(wl.random_packed_cache(s, T=T, seed=M + r, psac_fmt=fmt), page)
    pg = wl.to_paged(pc, page, pc.B * pc.capacity // page + 3, seed=page)
    P = _basis(2, 128, r, 5)
    gc, gp = gpu_cache_like(pc), gpu_cache_like(pg)
    for c in (gc, gp):
        c.P.copy_(torch.from_numpy(P))
    rng = np.random.default_rng(length)
    Q = to_dev(wl.bf16_bits(rng.standard_normal((2, s.H_q, 128)).astype(np.float32)), torch.int16)
    a = kv2.kv2_attention_decode(gc, length, Q, 0.09)
    b = kv2.kv2_attention_decode(gp, length, Q, 0.09)
    assert torch.equal(a, b)
    Qn = Q.view(2, 1, s.H_q, 128).repeat(1, 3, 1, 1)
    assert torch.equal(kv2.kv2_decode_top1(gc, length, Qn), kv2.kv2_decode_top1(gp, length, Qn))
    ref = orc.decode(pg, P, length, Q.cpu().numpy().view(np.uint16), 0.09)
    assert_attention_close(b.cpu().numpy(), ref, what=f"paged decode page{page}")


def test_chunk_identical_to_contiguous():
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=128, H_kv=2, H_q=4, M=256, r=8, T=700, B=1)
    pc = _padded(wl.random_packed_cache(s, T=700, seed=3), 128)
    pg = wl.to_paged(pc, 128, pc.capacity // 128 + 4, seed=9)
    gc, gp = gpu_cache_like(pc), gpu_cache_like(pg)
    P = torch.from_numpy(_basis(2, 128, 8, 6))
    gc.P.copy_(P)
    gp.P.copy_(P)
    rng = np.random.default_rng(4)
    Q, Ks, Vs = (to_dev(wl.bf16_bits(rng.standard_normal(sh).astype(np.float32)), torch.int16)
                 for sh in ((1, 300, 4, 128), (1, 300, 2, 128), (1, 300, 2, 128)))
    a = kv2.kv2_attention_chunk(gc, 613, Q, Ks, Vs, 100, 0.09)
    b = kv2.kv2_attention_chunk(gp, 613, Q, Ks, Vs, 100, 0.09)
    assert torch.equal(a, b)


def test_append_through_the_block_table(orc):
    import bit_kv_cache_centroid_b200 as kv2
    w = wl.make("tiny", T=600, n_new=1)
    s = w.spec
    f = orc.fit(w.Qhist, s.H_kv, s.r)
    cap = 768
    flat = wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, cap, w.centroids)
    paged = wl.to_paged(flat, 256, s.B * cap // 256 + 2, seed=11)
    gc, gp = gpu_cache_like(flat, fit=f), gpu_cache_like(paged, fit=f)
    K = to_dev(np.ascontiguousarray(w.K[:, :s.T]), torch.int16)
    V = to_dev(np.ascontiguousarray(w.V[:, :s.T]), torch.int16)
    for c in (gc, gp):
        kv2.kv2_quantize_append(c, K[:, :500].contiguous(), V[:, :500].contiguous(), 37, s.C)
    torch.cuda.synchronize()
    hf, hp = gc.to_host(), gp.to_host()
    for name in ("k_code", "v_code", "k_sz", "v_sz", "cidx", "psac"):
        for b in range(s.B):
            for i in range(cap // 256):
                lo, hi = max(37, i * 256), min(537, (i + 1) * 256)
                if lo < hi:
                    got = hp[name][paged.table[b, i]][:, lo - i * 256:hi - i * 256]
                    assert np.array_equal(got, hf[name][b, :, lo:hi]), name
    Q = to_dev(w.Qdec, torch.int16)
    assert torch.equal(kv2.kv2_attention_decode(gc, 537, Q, 0.1), kv2.kv2_attention_decode(gp, 537, Q, 0.1))


@pytest.mark.parametrize("fmt,M", [(0, 64), (1, 512)])
def test_evict_and_retrieve_a_page(orc, fmt, M):
    """Long-horizon memory: a page stored to host memory is the page's slice of
    every stream back to back; after the page is cleared on the device (its
    slot reused) the decode changes, and after the image is loaded into a spare
    page of the pool and the block-table entry points there, decode and top-1
    are bit-identical to before; the retrieved cache still matches the oracle."""
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=128, H_kv=2, H_q=8, M=M, r=8, T=1024, B=2)
    pc = wl.random_packed_cache(s, T=1024, seed=21 + fmt, psac_fmt=fmt)
    n_pages = pc.B * pc.capacity // 128 + 4
    pg = wl.to_paged(pc, 128, n_pages, seed=2)
    gp = gpu_cache_like(pg)
    P = _basis(2, 128, 8, 5)
    gp.P.copy_(torch.from_numpy(P))
    rng = np.random.default_rng(3)
    Q = to_dev(wl.bf16_bits(rng.standard_normal((2, 8, 128)).astype(np.float32)), torch.int16)
    before = kv2.kv2_attention_decode(gp, 1000, Q, 0.09)
    top_before = kv2.kv2_decode_top1(gp, 1000, Q)
    src = int(pg.table[1, 2])                       # tokens 256..383 of sequence 1
    spare = sorted(set(range(n_pages)) - set(pg.table.ravel().tolist()))[0]
    img = kv2.kv2_page_store(gp, src)
    torch.cuda.synchronize()
    names = ["k_code", "v_code", "k_sz", "v_sz", "cidx", "psac"] + (["psac_scale"] if fmt == 1 else [])
    want = np.concatenate([np.ascontiguousarray(getattr(pg, n)[src]).reshape(-1).view(np.uint8) for n in names])
    assert img.numel() == kv2.kv2_page_bytes(gp) == want.size
    assert np.array_equal(img.numpy(), want)
    for n in names:
        getattr(gp, n)[src].zero_()
    assert not torch.equal(kv2.kv2_attention_decode(gp, 1000, Q, 0.09), before)
    kv2.kv2_page_load(gp, spare, img)
    gp.block_table[1, 2] = spare
    after = kv2.kv2_attention_decode(gp, 1000, Q, 0.09)
    assert torch.equal(after, before)
    assert torch.equal(kv2.kv2_decode_top1(gp, 1000, Q), top_before)
    moved = wl.to_paged(pc, 128, n_pages, seed=2)
    moved.table[1, 2] = spare
    for n in names:
        getattr(moved, n)[spare] = getattr(pg, n)[src]
    ref = orc.decode(moved, P, 1000, Q.cpu().numpy().view(np.uint16), 0.09)
    assert_attention_close(after.cpu().numpy(), ref, what=f"retrieved page fmt{fmt}")
