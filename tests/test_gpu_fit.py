"""GPU parity of kv2_fit_psac_basis against the oracle's fp64 fit: weights
to fp32 rounding, the top-r subspace by projector distance, each well
separated eigenvector with its sign, and the energy share."""
import numpy as np
import pytest
import torch

import workloads as wl
from helpers import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,H_q,H_kv,d,n,r", [
    ("tiny", 2, 2, 64, 64, 8),
    ("llm_decode", 32, 8, 128, 128, 8),
    ("quant_append", 8, 8, 128, 512, 8),
    ("long_horizon", 4, 4, 128, 512, 16),
])
def test_fit_matches_oracle(orc, name, H_q, H_kv, d, n, r):
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec(name, H_q=H_q, H_kv=H_kv, d=d, n_hist=n, r=r)
    rng = np.random.default_rng(s.seed)
    U = wl.query_bases(s, rng)
    Qh = wl.bf16_bits(wl.draw_queries(s, rng, n, U)[0])
    ref = orc.fit(Qh, H_kv, r)
    P, w, Wg, en = kv2.kv2_fit_psac_basis(to_dev(Qh, torch.int16), H_kv, r)
    torch.cuda.synchronize()
    P, w, Wg, en = (x.cpu().numpy() for x in (P, w, Wg, en))
    np.testing.assert_allclose(w, ref.w, rtol=2e-7, atol=0)
    np.testing.assert_allclose(Wg, ref.Wg, rtol=1e-6, atol=0)
    np.testing.assert_allclose(en, ref.energy, rtol=1e-5)
    for h in range(H_kv):
        Pg, Pr = P[h].astype(np.float64), ref.P[h].astype(np.float64)
        assert np.linalg.norm(Pg @ Pg.T - Pr @ Pr.T) <= 1e-4
        lam = ref.evals[h]
        for i in range(r):
            gap = min(abs(lam[i] - lam[i - 1]) if i else np.inf, abs(lam[i] - lam[i + 1]))
            if gap > 1e-3 * lam[0]:
                assert abs(Pg[:, i] @ Pr[:, i] - 1.0) <= 1e-5, (h, i)


def test_fit_rejects_bad_shapes():
    import bit_kv_cache_centroid_b200 as kv2
    Q = torch.zeros(8, 3, 64, dtype=torch.int16, device="cuda")
    with pytest.raises(kv2.Kv2Error):
        kv2.kv2_fit_psac_basis(Q, 2, 8)        # 3 query heads over 2 KV heads
