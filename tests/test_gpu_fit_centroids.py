"""GPU parity of kv2_fit_centroids (QSAC-aware centre fitting) against the
oracle: the fitted fp16 centres and the last assignment, bit for bit, on keys
with the video workloads' statistics. Covers the short (one key per warp) and
general assignment paths, d = 64 and 128, M up to 512, a centre that no key
chooses, no-op calls, and the 40-head quantize configuration (sampled heads)."""
import numpy as np
import pytest
import torch

import workloads as wl
from helpers import to_dev

pytestmark = pytest.mark.gpu


def _keys(n, H, d, M, seed):
    """n keys per head (bf16 bits [n][H][d]), the workload's k-means centres
    (fp16 bits [H][M][d]) and the sensitivities w, Wg of a fit on its history
    queries."""
    w = wl.make("quant_append", seed=seed, H_q=H, H_kv=H, d=d, M=M, T=max(n, M), n_new=1, n_hist=128, Nq=0,
                frame_tokens=max(n, M), with_chunk=False)
    X = np.ascontiguousarray(w.K[0, :n])
    return w, X


def _run_gpu(X, cent, C, w, Wg, iters):
    import bit_kv_cache_centroid_b200 as kv2
    cd = to_dev(cent, torch.int16)
    out, assign = kv2.kv2_fit_centroids(to_dev(X, torch.int16), cd, C, to_dev(w), to_dev(Wg), iters)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16), assign.cpu().numpy()


def _check(orc, X, cent, C, f, iters):
    got_c, got_a = _run_gpu(X, cent, C, f.w, f.Wg, iters)
    ref_c, ref_a = orc.fit_centroids(X, cent.shape[1], C, f.w, f.Wg, cent, iters)
    assert np.array_equal(got_a, ref_a), f"assignments differ: {int((got_a != ref_a).sum())}"
    assert np.array_equal(got_c, ref_c), f"centres differ: {int((got_c != ref_c).sum())} fp16 values"
    return got_c, got_a


@pytest.mark.parametrize("n, H, d, M, C, iters", [
    (2048, 4, 128, 64, 4, 3),      # general path (8 keys per warp)
    (40, 2, 128, 256, 8, 2),       # short path (one key per warp), M > n
    (40, 2, 128, 16, 4, 3),        # short path, centres that move
    (900, 3, 64, 16, 4, 3),        # d = 64
    (700, 2, 128, 512, 8, 2),      # M = 512
    (333, 2, 128, 32, 32, 2),      # candidates = M, ragged key count
])
def test_fit_matches_oracle(orc, n, H, d, M, C, iters):
    w, X = _keys(n, H, d, M, seed=21 + n)
    f = orc.fit(w.Qhist, H, 8)
    _check(orc, X, w.centroids, C, f, iters)


def test_unchosen_centre_keeps_its_value_and_noops(orc):
    import bit_kv_cache_centroid_b200 as kv2
    w, X = _keys(512, 2, 128, 16, seed=5)
    f = orc.fit(w.Qhist, 2, 8)
    cent = w.centroids.copy()
    cent[:, 7] = wl.f16_bits(np.full((2, 128), 3000.0, np.float32))       # far from every key
    got_c, got_a = _check(orc, X, cent, 4, f, 2)
    assert not np.any(got_a == 7)
    assert np.array_equal(got_c[:, 7], cent[:, 7])
    same, _ = _run_gpu(X, cent, 4, f.w, f.Wg, 0)
    assert np.array_equal(same, cent)
    cd = to_dev(cent, torch.int16)
    kv2.kv2_fit_centroids(to_dev(X[:0], torch.int16), cd, 4, to_dev(f.w), to_dev(f.Wg), 3)
    torch.cuda.synchronize()
    assert np.array_equal(cd.cpu().numpy().view(np.uint16), cent)


def test_invalid_arguments_are_rejected():
    import bit_kv_cache_centroid_b200 as kv2
    X = torch.zeros((16, 2, 128), dtype=torch.int16, device="cuda")
    cent = torch.zeros((2, 8, 128), dtype=torch.int16, device="cuda")
    w = torch.ones((2, 128), device="cuda")
    Wg = torch.ones((2, 4), device="cuda")
    with pytest.raises(kv2.Kv2Error):
        kv2.kv2_fit_centroids(X, cent, 9, w, Wg, 1)                       # candidates > M
    with pytest.raises(kv2.Kv2Error):
        kv2.kv2_fit_centroids(X, cent, 2, w, Wg, 1, ws=torch.zeros(64, dtype=torch.uint8, device="cuda"))


@pytest.mark.slow
def test_quantize_configuration_sampled_heads(orc):
    """8,192 sample keys x 40 heads, M = 256, C = 8 (the quantize workload's
    table sizes); the oracle recomputes three heads."""
    n, H, d, M, C, iters = 8192, 40, 128, 256, 8, 2
    w, X = _keys(n, H, d, M, seed=3)
    f = orc.fit(w.Qhist, H, 8)
    got_c, got_a = _run_gpu(X, w.centroids, C, f.w, f.Wg, iters)
    heads = [0, 17, 39]
    sub = np.ascontiguousarray(X[:, heads])
    ref_c, ref_a = orc.fit_centroids(sub, M, C, f.w[heads], f.Wg[heads], w.centroids[heads], iters)
    assert np.array_equal(got_a[:, heads], ref_a)
    assert np.array_equal(got_c[heads], ref_c)
