"""Pins of the oracle's QSAC-aware centre fitting (QuantWM article, '1. QSAC':
the clustering picks INT2-friendly Key centres; the loop is read as Lloyd
iterations whose assignment step is the QSAC decision).

* candidates = 1 with unit weights: the textbook Lloyd k-means (nearest centre,
  centre = mean of its keys), recomputed here by brute force in fp64 on keys of
  a coarse grid, where every distance and sum is exact;
* well-separated blobs with candidates = M and unequal weights: one iteration
  gives every key its own blob's centre and every centre its blob's mean;
* a centre that no key chooses keeps its value; iters = 0 and n = 0 change
  nothing.
"""
import numpy as np

import workloads as wl


def _f16_from_f64(x):
    return np.asarray(x, np.float64).astype(np.float16).view(np.uint16)


def _grid_keys(rng, n, H, d, M):
    """Keys on a grid of 1/8, around M well-spread centres per head."""
    ctr = rng.integers(-32, 33, (H, M, d)) / 4.0
    lab = rng.integers(0, M, (n, H))
    X = np.empty((n, H, d))
    for h in range(H):
        X[:, h] = ctr[h, lab[:, h]] + rng.integers(-12, 13, (n, d)) / 8.0
    return X


def _lloyd_fp64(X, cent, iters):
    """Plain Lloyd k-means: nearest centre (fp64 squared distance, ties to the
    lower index), centre = mean of its keys (fp64, rounded to fp16), empty
    centres unchanged. X [n][H][d] fp64, cent fp16 bits [H][M][d]."""
    cent = cent.copy()
    n, H, d = X.shape
    assign = np.zeros((n, H), np.int32)
    for _ in range(iters):
        for h in range(H):
            c = cent[h].view(np.float16).astype(np.float64)
            dist = ((X[:, h, None, :] - c[None, :, :]) ** 2).sum(-1)
            a = dist.argmin(1)
            assign[:, h] = a
            for j in range(c.shape[0]):
                sel = a == j
                if sel.any():
                    cent[h, j] = _f16_from_f64(X[sel, h].sum(0) / sel.sum())
    return cent, assign


def test_single_candidate_unit_weights_is_lloyd(orc):
    rng = np.random.default_rng(11)
    n, H, d, M = 300, 2, 64, 8
    X = _grid_keys(rng, n, H, d, M)
    Xb = wl.bf16_bits(X.astype(np.float32))
    assert np.array_equal(wl.bf16_values(Xb).astype(np.float64), X)          # exact on the grid
    init = _f16_from_f64(X[rng.choice(n, M, replace=False)].transpose(1, 0, 2))
    w = np.ones((H, d), np.float32)
    Wg = np.full((H, d // 32), 32.0, np.float32)
    got_c, got_a = orc.fit_centroids(Xb, M, 1, w, Wg, init, iters=4)
    ref_c, ref_a = _lloyd_fp64(X, init, 4)
    assert np.array_equal(got_a, ref_a)
    assert np.array_equal(got_c, ref_c)


def test_separated_blobs_one_iteration_gives_blob_means(orc):
    rng = np.random.default_rng(12)
    H, d, M, per = 2, 128, 6, 40
    X = np.empty((M * per, H, d))
    means = np.empty((H, M, d))
    for h in range(H):
        for j in range(M):
            base = np.zeros(d)
            base[(j * 16) % d:(j * 16) % d + 16] = 40.0 * (1 + j)             # far apart
            pts = base + rng.integers(-8, 9, (per, d)) / 16.0
            X[j * per:(j + 1) * per, h] = pts
            means[h, j] = pts.mean(0)
    Xb = wl.bf16_bits(X.astype(np.float32))
    X = wl.bf16_values(Xb).astype(np.float64)
    # initial centres: one key of each blob
    init = _f16_from_f64(np.stack([X[j * per, :, :] for j in range(M)], 1))
    w = rng.uniform(0.5, 2.0, (H, d)).astype(np.float32)
    Wg = w.reshape(H, d // 32, 32).sum(-1).astype(np.float32)
    cent, assign = orc.fit_centroids(Xb, M, M, w, Wg, init, iters=1)
    labels = np.repeat(np.arange(M), per)
    for h in range(H):
        assert np.array_equal(assign[:, h], labels)
        for j in range(M):
            exact = X[j * per:(j + 1) * per, h].sum(0) / per
            assert np.array_equal(cent[h, j], _f16_from_f64(exact))


def test_unchosen_centre_keeps_its_value_and_noop_cases(orc):
    rng = np.random.default_rng(13)
    n, H, d, M = 64, 1, 64, 4
    X = _grid_keys(rng, n, H, d, 2)
    Xb = wl.bf16_bits(X.astype(np.float32))
    init = _f16_from_f64(np.concatenate([X[:3, 0], np.full((1, d), 1000.0)])[None])
    w = np.ones((H, d), np.float32)
    Wg = np.full((H, d // 32), 32.0, np.float32)
    cent, assign = orc.fit_centroids(Xb, M, 2, w, Wg, init, iters=3)
    assert not np.any(assign == 3)
    assert np.array_equal(cent[0, 3], init[0, 3])
    same, _ = orc.fit_centroids(Xb, M, 2, w, Wg, init, iters=0)
    assert np.array_equal(same, init)
    empty, a0 = orc.fit_centroids(Xb[:0], M, 2, w, Wg, init, iters=2)
    assert np.array_equal(empty, init) and a0.shape == (0, H)


def test_fixed_point_mean_truncates_below_one_unit(orc):
    """The update's mean counts each key value in whole 2^-24 units,
    truncated toward zero: a lone key of +-0.75 * 2^-24 (bf16-exact) leaves
    its channel of the centre at 0, where the exact mean would round to
    +-2^-24; values of whole units average exactly (2^-20 and 2^-23 -> 9
    units)."""
    d = 64
    X = np.zeros((2, 1, d), np.float32)
    X[0, 0, 0] = 0.75 * 2.0 ** -24
    X[0, 0, 1] = -0.75 * 2.0 ** -24
    X[0, 0, 2] = 2.0 ** -20
    X[1, 0, 2] = 2.0 ** -23
    Xb = wl.bf16_bits(X)
    assert np.array_equal(wl.bf16_values(Xb), X)
    w = np.ones((1, d), np.float32)
    Wg = np.full((1, d // 32), 32.0, np.float32)
    cent0 = wl.f16_bits(np.full((1, 1, d), 0.5, np.float32))
    cent, assign = orc.fit_centroids(Xb, 1, 1, w, Wg, cent0, 1)
    got = wl.f16_values(cent)[0, 0].astype(np.float64)
    assert got[0] == 0.0 and got[1] == 0.0
    assert got[2] == 9 * 2.0 ** -24                    # (16 + 2) / 2 units
    assert np.all(got[3:] == 0.0) and np.all(assign == 0)
