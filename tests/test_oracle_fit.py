"""Pins of the oracle's PSAC basis fit (QuantWM article, '2. PSAC': historical
Query energy concentrates in a few principal directions) against
numpy.linalg.eigh, the sign/order rule and the synthetic query law."""
import numpy as np
import pytest

import workloads as wl


def _queries(H_q, H_kv, d, n, top=0.70, seed=0):
    s = wl.spec("tiny", H_q=H_q, H_kv=H_kv, d=d, n_hist=n, top_energy=top)
    rng = np.random.default_rng(seed)
    U = wl.query_bases(s, rng)
    return wl.bf16_bits(wl.draw_queries(s, rng, n, U)[0]), U


@pytest.mark.parametrize("H_q,H_kv,d,n,r", [(2, 2, 64, 64, 8), (8, 2, 128, 128, 16), (4, 1, 64, 50, 64)])
def test_fit_matches_eigh(orc, H_q, H_kv, d, n, r):
    Qh, _ = _queries(H_q, H_kv, d, n)
    f = orc.fit(Qh, H_kv, r)
    G = H_q // H_kv
    q = wl.bf16_values(Qh).astype(np.float64)                   # [n][H_q][d]
    for h in range(H_kv):
        X = q[:, h * G:(h + 1) * G, :].reshape(-1, d)
        S = X.T @ X / X.shape[0]
        lam, vec = np.linalg.eigh(S)
        lam, vec = lam[::-1], vec[:, ::-1]
        np.testing.assert_allclose(f.evals[h], lam, rtol=1e-9, atol=1e-12 * lam[0])
        np.testing.assert_allclose(f.w[h], np.diag(S).astype(np.float32), rtol=1e-7)
        np.testing.assert_allclose(f.Wg[h], np.diag(S).reshape(-1, 32).sum(1), rtol=1e-6)
        P = f.P[h].astype(np.float64)                              # [d][r]
        np.testing.assert_allclose(P.T @ P, np.eye(r), atol=1e-6)
        # the top-r subspace (well separated: graded spectrum)
        proj = vec[:, :r] @ vec[:, :r].T
        assert np.linalg.norm(P @ P.T - proj) < 1e-5
        # each vector: an eigenvector with the r largest eigenvalues, largest entry positive
        for i in range(r):
            v = P[:, i]
            assert abs(v @ S @ v - lam[i]) < 1e-6 * lam[0]
            assert v[np.argmax(np.abs(v))] > 0
        np.testing.assert_allclose(f.energy[h], lam[:r].sum() / lam.sum(), rtol=1e-9)


def test_fit_energy_of_query_law(orc):
    """The synthetic queries put 70% of their energy in 8 directions; the fit
    recovers that share (sampling noise only)."""
    Qh, U = _queries(4, 1, 128, 1024, top=0.70, seed=3)
    f = orc.fit(Qh, 1, 8)
    assert abs(f.energy[0] - 0.70) < 0.03
    # and the fitted subspace is the generating one
    Ptrue = U[0][:, :8]
    assert np.linalg.norm(f.P[0] @ f.P[0].T - Ptrue @ Ptrue.T) < 0.35


def test_fit_diagonal_closed_form(orc):
    """Queries along coordinate axes: S is diagonal with known entries, the
    eigenvectors are the axes (sign +1) in order of decreasing energy."""
    d, n = 64, 64
    q = np.zeros((n, 1, d), np.float32)
    amp = np.linspace(4.0, 0.5, d).astype(np.float32)
    for t in range(n):
        q[t, 0, t % d] = amp[t % d] * (1 if t % 2 == 0 else -1)
    Qh = wl.bf16_bits(q)
    f = orc.fit(Qh, 1, 4)
    vals = wl.bf16_values(Qh)[:, 0, :].astype(np.float64)
    S = vals.T @ vals / n
    np.testing.assert_allclose(f.evals[0], np.sort(np.diag(S))[::-1], rtol=1e-12)
    for i in range(4):
        e = np.zeros(d)
        e[i] = 1.0
        np.testing.assert_allclose(f.P[0][:, i], e, atol=1e-7)
