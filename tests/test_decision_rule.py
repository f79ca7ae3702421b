"""The quantizer kernel settles a key whose candidate set its fast scores
leave open without exact distances when it can (QuantWM article, '1. QSAC':
the C centres of least weighted distance are the candidates, the one of
least estimated perturbation is chosen). This CPU test checks that rule
against the oracle's fp32 definitions on the oracle's own D_j and E_j (read
for every centre by running it with C = M):

* fast scores f_j = D_j + delta_j with |delta_j| <= b, the errors placed at
  the edges of b (the taken set pushed up, the others down) or at random;
* S = the C least f; no centre outside S with f <= max_S f + 2b: S is the
  choice's candidate set;
* otherwise the list L = S and the others under that threshold, a centre of
  S "sure" when f_i < min_{j not in S} f_j - 2b; the least (E, id) among the
  sure ones is the choice when it is below every doubtful one, else the C
  least (D, id) of L are the set.

Every decision the rule takes must equal the oracle's, and the oracle's own
candidate set must lie in L. The test also pins the oracle: its choice for
the workload's C equals the least (E, id) over its C least (D, id)."""
import numpy as np
import pytest

import workloads as wl


def _all_centres(orc, name, **ov):
    w = wl.make(name, with_chunk=False, **ov)
    s = w.spec
    f = orc.fit(w.Qhist, s.H_kv, s.r)
    K, V = w.K[:, :s.T], w.V[:, :s.T]
    pc = wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, s.capacity, w.centroids)
    dbg = orc.quantize(pc, K, V, 0, s.M, f.P, f.w, f.Wg, debug=True)     # C = M: every centre
    cand = dbg.cand.reshape(-1, s.M)
    D = np.empty(cand.shape, np.float64)
    E = np.empty(cand.shape, np.float64)
    rows = np.arange(cand.shape[0])[:, None]
    D[rows, cand] = dbg.score.reshape(-1, s.M)
    E[rows, cand] = dbg.E.reshape(-1, s.M)
    pc2 = wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, s.capacity, w.centroids)
    orc.quantize(pc2, K, V, 0, s.C, f.P, f.w, f.Wg)
    # chosen ids in the debug arrays' (b, t, h) row order
    cidx = pc2.cidx.reshape(s.B, s.H_kv, -1)[:, :, :s.T].transpose(0, 2, 1).reshape(-1).astype(np.int64)
    return D, E, cidx, s.C


def _least(keys_primary, ids):
    """index of the least (primary, id) pair."""
    return ids[np.lexsort((ids, keys_primary))[0]]


def _rule(f, b, D, E, C):
    """(choice, route) of the kernel's decision for one key."""
    M = f.size
    ids = np.arange(M)
    order = np.lexsort((ids, f))
    S, out = order[:C], order[C:]
    thr = f[S].max() + 2 * b
    near = out[f[out] <= thr]
    if near.size == 0:
        return _least(E[S], S), "fast", S
    L = np.concatenate([S, near])
    lim = f[out].min() - 2 * b
    sure = S[f[S] < lim]
    doubt = np.setdiff1d(L, sure)
    if sure.size:
        bs = (E[sure].min(), _least(E[sure], sure))
        bd_id = _least(E[doubt], doubt)
        if (E[bd_id], bd_id) > bs:
            return bs[1], "perturbation", L
    Lx = L[np.lexsort((L, D[L]))][:C]
    return _least(E[Lx], Lx), "exact", L


@pytest.mark.parametrize("name,ov", [
    ("tiny", dict(T=256)),
    ("quant_append", dict(H_q=4, H_kv=4, T=300, n_new=1, capacity=304, n_hist=256)),
])
def test_rule_matches_the_oracle(orc, name, ov):
    D, E, chosen, C = _all_centres(orc, name, **ov)
    n, M = D.shape
    ids = np.arange(M)
    rng = np.random.default_rng(11)
    routes = {"fast": 0, "perturbation": 0, "exact": 0}
    for i in range(n):
        # the oracle's choice by the definitions, on its own D and E
        top = ids[np.lexsort((ids, D[i]))][:C]
        want = _least(E[i, top], top)
        assert want == chosen[i], f"key {i}: oracle chose {chosen[i]}, definitions give {want}"
        gaps = np.diff(np.sort(D[i]))
        scale = np.median(gaps[gaps > 0]) if np.any(gaps > 0) else 1.0
        for bf in (0.05, 0.5, 3.0):
            b = bf * scale
            for mode in ("edges", "random"):
                if mode == "edges":
                    delta = np.where(np.isin(ids, top), b, -b)
                else:
                    delta = rng.uniform(-b, b, M)
                got, route, L = _rule(D[i] + delta, b, D[i], E[i], C)
                routes[route] += 1
                assert np.all(np.isin(top, L)), f"key {i}: an exact candidate fell outside the list"
                assert got == want, f"key {i}, b={b:.3g}, {mode}: rule chose {got} ({route}), oracle {want}"
    # the three routes are all taken, so each branch of the rule is exercised
    assert routes["fast"] and routes["perturbation"] and routes["exact"], routes
