"""Exhaustive pins of the oracle on 4-element groups (QuantWM article, '1. QSAC':
asymmetric INT2 per group with an fp16 scale and zero; the oracle takes any
group size, and groups this small can be enumerated):

* the codec on every 4-element group over a grid of fp16-exact values, which
  includes constant groups, exact half-way points between levels and all
  orderings: the zero is the group minimum (exact in fp16), three scales
  reach the maximum and no smaller fp16 scale does, every code is a nearest
  level, and an exact tie between two levels takes the even code;
* QSAC with d = 16 in four 4-channel groups, M = 4 centres and every centre a
  candidate: the chosen centre has the least E_j = sum_g W_g s_g^2 of all
  four, computed from the codec's scales for each group (brute force).
"""
import itertools

import numpy as np

import workloads as wl

GRID = np.array([-1.5, -1.0, -0.5, -0.25, 0.0, 0.125, 0.5, 1.0, 2.75], np.float32)


def _f16(bits):
    return float(np.uint16(bits).view(np.float16))


def test_codec_on_every_four_element_group(orc):
    ties = 0
    for xs in itertools.product(GRID, repeat=4):
        x = np.array(xs, np.float32)
        sb, zb, codes, deq = orc.codec_group(x)
        s, z = _f16(sb), _f16(zb)
        lo, hi = float(x.min()), float(x.max())
        assert z == lo, xs                                   # fp16-exact minimum
        assert z + 3 * s >= hi, xs
        if s > 0:
            smaller = float(np.nextafter(np.float16(s), np.float16(0)))
            assert z + 3 * smaller < hi, xs                  # the least fp16 scale that reaches the maximum
        else:
            assert hi == lo and np.all(codes == 0), xs
        levels = z + s * np.arange(4)
        err = np.abs(levels[None, :] - x.astype(np.float64)[:, None])      # exact in fp64
        best = err.min(1)
        mine = err[np.arange(4), codes]
        assert np.all(mine == best), xs                      # a nearest level
        for i in range(4):
            nearest = np.flatnonzero(err[i] == best[i])
            if nearest.size == 2:                            # exact tie between two levels
                assert codes[i] % 2 == 0, (xs, i, codes[i])
                ties += 1
        assert np.array_equal(deq, levels[codes].astype(np.float32)), xs
    assert ties > 100                                        # the grid does exercise the tie rule


def test_qsac_with_four_channel_groups_is_bruteforce(orc):
    rng = np.random.default_rng(17)
    d, M, group, T, H = 16, 4, 4, 400, 2
    cent = wl.f16_bits(rng.standard_normal((H, M, d)).astype(np.float32))
    K = wl.bf16_bits((rng.standard_normal((1, T, H, d)) * np.linspace(0.3, 3.0, d)).astype(np.float32))
    V = wl.bf16_bits(rng.standard_normal((1, T, H, d)).astype(np.float32))
    w = rng.uniform(0.2, 3.0, (H, d)).astype(np.float32)
    Wg = w.reshape(H, d // group, group).sum(-1).astype(np.float32)
    pc = wl.PackedCache.empty(1, H, d, M, 0, T, cent, group=group)
    dbg = orc.quantize(pc, K, V, 0, M, np.zeros((H, d, 0), np.float32), w, Wg, debug=True)
    keys = wl.bf16_values(K)[0]
    mu = wl.f16_values(cent)
    near = 0
    for h in range(H):
        for t in range(T):
            E = np.zeros(M)
            for j in range(M):
                x = (keys[t, h] - mu[h, j]).astype(np.float32)
                for g in range(d // group):
                    sb, _, _, _ = orc.codec_group(x[g * group:(g + 1) * group])
                    E[j] += float(Wg[h, g]) * _f16(sb) ** 2
            got = int(pc.cidx[0, h, t])
            assert E[got] <= E.min() * (1 + 1e-6) + 1e-30, (h, t, got, E)
            near += int(got != int(E.argmin()))
            # the trace ranks all four centres and keeps the chosen estimate least
            assert sorted(dbg.cand[0, t, h].tolist()) == list(range(M))
    assert near <= 2
