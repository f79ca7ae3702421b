"""GPU parity of kv2_decode_top1 / kv2_dense_top1 (most-attended token per
query) against the oracle: the token the kernel picks has the oracle's
largest logit up to fp32 rounding (near ties may go either way), and the
index itself agrees for nearly every query. Covers both PSAC formats, d = 64
and 128, GQA, several token ranges per query, length 0, and the retrieval
shift of a QSAC + PSAC cache against a nearest-centre cache on keys with the
video workloads' statistics."""
import numpy as np
import pytest
import torch

import workloads as wl
from helpers import gpu_cache_like, host_cache, to_dev

pytestmark = pytest.mark.gpu


def _basis(H, d, r, seed):
    rng = np.random.default_rng(seed)
    P = np.zeros((H, d, max(r, 0)), np.float32)
    for h in range(H):
        P[h] = np.linalg.qr(rng.standard_normal((d, d)))[0][:, :r]
    return P


def _check(top, ref_top, lg, what):
    top = top.reshape(ref_top.shape)
    mx = lg.max(-1)
    picked = np.take_along_axis(lg, top[..., None].astype(np.int64), -1)[..., 0]
    tol = 1e-5 * np.abs(lg).max(-1) + 1e-6
    assert np.all(picked >= mx - tol), f"{what}: a pick below the oracle maximum"
    assert np.mean(top == ref_top) >= 0.98, f"{what}: {np.mean(top == ref_top):.3f} of indices agree"


@pytest.mark.parametrize("d,G,M,r,T,length,nq,fmt", [
    (128, 4, 64, 8, 5000, 4999, 3, 0),     # two token ranges per query
    (128, 1, 512, 16, 1500, 1300, 4, 1),   # u16 ids, rank 16, int8 PSAC
    (64, 2, 16, 0, 700, 650, 5, 0),        # d = 64, no PSAC
])
def test_decode_top1(orc, d, G, M, r, T, length, nq, fmt):
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=d, H_kv=2, H_q=2 * G, M=M, r=r, T=T, B=2)
    pc = wl.random_packed_cache(s, T=T, seed=d + M + r, psac_fmt=fmt)
    P = _basis(s.H_kv, d, r, 3)
    gc = gpu_cache_like(pc)
    if r:
        gc.P.copy_(torch.from_numpy(P))
    rng = np.random.default_rng(length)
    Q = wl.bf16_bits(rng.standard_normal((s.B, nq, s.H_q, d)).astype(np.float32) * 1.5)
    top = kv2.kv2_decode_top1(gc, length, to_dev(Q, torch.int16)).cpu().numpy()
    ref_top, lg = orc.decode_top1(pc, P, length, Q)
    _check(top, ref_top, lg, f"packed d{d} G{G} M{M} r{r} fmt{fmt}")


def test_dense_top1(orc):
    import bit_kv_cache_centroid_b200 as kv2
    rng = np.random.default_rng(9)
    K = wl.bf16_bits(rng.standard_normal((2, 4500, 2, 128)).astype(np.float32))
    Q = wl.bf16_bits(rng.standard_normal((2, 6, 4, 128)).astype(np.float32))
    top = kv2.kv2_dense_top1(to_dev(K, torch.int16), to_dev(Q, torch.int16)).cpu().numpy()
    ref_top, lg = orc.dense_top1(K, Q)
    _check(top, ref_top, lg, "dense")


def test_empty_length_gives_minus_one():
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=128, H_kv=1, H_q=2, M=16, r=8, T=32, B=1)
    gc = gpu_cache_like(wl.random_packed_cache(s, T=32))
    top = kv2.kv2_decode_top1(gc, 0, torch.zeros((1, 3, 2, 128), dtype=torch.int16, device="cuda"))
    assert torch.all(top == -1)


def test_retrieval_shift_of_quantized_caches(orc):
    """Keys with the video statistics quantized two ways on the GPU (QSAC with
    C = 8 and PSAC rank 8; nearest centre, unit weights, no PSAC), their
    most-attended tokens against those of the exact keys; the packed top-1
    agrees with the oracle on the same cache."""
    import bit_kv_cache_centroid_b200 as kv2
    w = wl.make("quant_append", H_q=2, H_kv=2, T=1200, n_new=1, n_hist=128, Nq=16, frame_tokens=300, M=64)
    s = w.spec
    f = orc.fit(w.Qhist, s.H_kv, s.r)
    K = np.ascontiguousarray(w.K[:, :s.T])
    V = np.ascontiguousarray(w.V[:, :s.T])
    Q = np.ascontiguousarray(w.Qchunk[:, :16])
    dense = kv2.kv2_dense_top1(to_dev(K, torch.int16), to_dev(Q, torch.int16)).cpu().numpy()
    shifts = {}
    for name, C, unit, r in (("quantwm", 8, False, 8), ("qvg", 1, True, 0)):
        sp = s.with_(r=r)
        pc = host_cache(sp, w.centroids, capacity=s.T)
        fit = orc.fit(w.Qhist, s.H_kv, r) if r else f
        if unit:
            fit.w[:] = 1.0
            fit.Wg[:] = 32.0
        gc = gpu_cache_like(pc, fit=fit)
        kv2.kv2_quantize_append(gc, to_dev(K, torch.int16), to_dev(V, torch.int16), 0, C)
        top = kv2.kv2_decode_top1(gc, s.T, to_dev(Q, torch.int16)).cpu().numpy()
        shifts[name] = float(np.mean(top != dense))
        h = gc.to_host()
        ref = host_cache(sp, w.centroids, capacity=s.T)
        for n in ("k_code", "k_sz", "cidx"):
            getattr(ref, n)[...] = h[n]
        if r:
            ref.psac[..., :r] = h["psac"]
        ref_top, lg = orc.decode_top1(ref, fit.P, s.T, Q)
        _check(top, ref_top, lg, f"{name} cache")
    assert 0.0 <= shifts["quantwm"] <= 1.0 and 0.0 <= shifts["qvg"] <= 1.0
