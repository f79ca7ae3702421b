"""Full-size attention parity on caches the library itself wrote from the
workloads' own keys (rather than ready-made random packed caches): the
library fits the Query statistics, quantizes the cached prefix with QSAC +
PSAC, and attends over it in the launch configuration the benchmark times.

* The packed bytes of sampled tokens equal the oracle quantizer's (centroid
  ids and code words bit-exact, scales, zeros and PSAC coefficients within
  1 fp16 ulp), given the library's fitted statistics.
* The attention outputs of sampled sequences / query rows match the oracle run
  on the packed cache the library wrote (max-abs 2e-3, rel-L2 1e-3).

Such caches carry the concentrated centroid-id and scale statistics of real
keys (outlier channels, smooth video fields) that random packed caches lack.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from helpers import assert_attention_close, f16_ulp_diff, host_cache, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _host_view(s, got, centroids, B=None):
    pc = host_cache(s, centroids)
    for name in ("k_code", "v_code", "k_sz", "v_sz", "cidx"):
        getattr(pc, name)[...] = got[name]
    if s.r:
        pc.psac[..., :s.r] = got["psac"]
    return pc


def _check_sampled_tokens(orc, s, K, V, f, got, centroids, toks):
    """The oracle quantizes the sampled tokens at their own slots, given the
    library's fitted statistics; their packed fields must match."""
    ref = host_cache(s, centroids)
    for t in toks:
        orc.quantize(ref, np.ascontiguousarray(K[:, t:t + 1]), np.ascontiguousarray(V[:, t:t + 1]), int(t), s.C,
                     f["P"], f["w"], f["Wg"])
    bb, hh, tt = np.meshgrid(np.arange(s.B), np.arange(s.H_kv), toks, indexing="ij")
    sl = (bb.ravel(), hh.ravel(), tt.ravel())
    for name in ("k_code", "v_code", "cidx"):
        np.testing.assert_array_equal(got[name][sl], getattr(ref, name)[sl], err_msg=name)
    for name in ("k_sz", "v_sz"):
        for half in (0, 16):
            d = f16_ulp_diff((got[name][sl] >> half) & 0xFFFF, (getattr(ref, name)[sl] >> half) & 0xFFFF)
            assert d.max() <= 1, name
    if s.r:
        assert f16_ulp_diff(got["psac"][sl], ref.psac[sl][..., :s.r]).max() <= 1


def _library_cache(kv2, s, w, n_tok):
    dev = torch.device("cuda")
    Qh = torch.from_numpy(w.Qhist.view(np.int16)).to(dev)
    P, wt, Wg, _ = kv2.kv2_fit_psac_basis(Qh, s.H_kv, s.r)
    cache = kv2.Cache(s.B, s.H_kv, s.d, s.M, s.r, (s.capacity + 15) // 16 * 16,
                      torch.from_numpy(w.centroids.view(np.int16)))
    cache.set_fit(P, wt, Wg)
    K = torch.from_numpy(np.ascontiguousarray(w.K[:, :n_tok]).view(np.int16)).to(dev)
    V = torch.from_numpy(np.ascontiguousarray(w.V[:, :n_tok]).view(np.int16)).to(dev)
    kv2.kv2_quantize_append(cache, K, V, 0, s.C)
    torch.cuda.synchronize()
    fit = {"P": P.cpu().numpy(), "w": wt.cpu().numpy(), "Wg": Wg.cpu().numpy()}
    return cache, fit


def test_llm_decode_on_library_quantized_keys(orc):
    """LLM decode workload: batch 8, 32/8 heads, d=128, the 32,768-token
    prefix of every sequence quantized by the library (M=64, C=4, r=8); the
    workload's decode queries; the oracle recomputes sequences 0 and 7 and the
    packed fields of 16 sampled tokens of every (sequence, head)."""
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("llm_decode")
    w = wl.make("llm_decode", with_chunk=False)
    cache, fit = _library_cache(kv2, s, w, s.T)
    got = cache.to_host()
    rng = np.random.default_rng(17)
    toks = np.sort(rng.choice(s.T, 16, replace=False))
    _check_sampled_tokens(orc, s, w.K, w.V, fit, got, w.centroids, toks)
    scale = 1.0 / np.sqrt(s.d)
    out = kv2.kv2_attention_decode(cache, s.T, to_dev(w.Qdec, torch.int16), scale).cpu().numpy()
    pc = _host_view(s, got, w.centroids)
    for b in (0, s.B - 1):
        sub = wl.PackedCache(1, s.H_kv, s.d, s.M, s.r, pc.capacity, pc.k_code[b:b + 1], pc.v_code[b:b + 1],
                             pc.k_sz[b:b + 1], pc.v_sz[b:b + 1], pc.cidx[b:b + 1], pc.psac[b:b + 1],
                             pc.centroids)
        ref = orc.decode(sub, fit["P"], s.T, w.Qdec[b:b + 1], scale)
        assert_attention_close(out[b:b + 1], ref, what=f"llm decode on quantized keys, sequence {b}")


def test_video_chunk_on_library_quantized_keys(orc):
    """Video chunk workload: 40 heads, the 37,440 cached tokens (24 latent
    frames of video-law keys) quantized by the library (M=256, C=8, r=8); the
    workload's 4,680 chunk queries with the chunk's own keys and values,
    block-causal by frame; the oracle recomputes 14 sampled query rows and the
    packed fields of 8 sampled tokens of every head."""
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("video_chunk")
    w = wl.make("video_chunk")
    cache, fit = _library_cache(kv2, s, w, s.T)
    got = cache.to_host()
    rng = np.random.default_rng(19)
    toks = np.sort(rng.choice(s.T, 8, replace=False))
    _check_sampled_tokens(orc, s, w.K, w.V, fit, got, w.centroids, toks)
    scale = 1.0 / np.sqrt(s.d)
    Ks = np.ascontiguousarray(w.K_new)
    Vs = np.ascontiguousarray(w.V_new)
    out = kv2.kv2_attention_chunk(cache, s.T, to_dev(w.Qchunk, torch.int16), to_dev(Ks, torch.int16),
                                  to_dev(Vs, torch.int16), s.frame_tokens, scale)
    torch.cuda.synchronize()
    out = out.float().cpu().numpy()
    picks = [0, 1559, 1560, 3120, s.Nq - 1] + list(rng.integers(0, s.Nq, 9))
    rows = np.array([(0, int(i), int(rng.integers(0, s.H_q))) for i in picks], np.int32)
    pc = _host_view(s, got, w.centroids)
    ref = orc.chunk(pc, fit["P"], s.T, w.Qchunk, Ks, Vs, s.frame_tokens, scale, rows)
    assert_attention_close(out[rows[:, 0], rows[:, 1], rows[:, 2]], ref, what="video chunk on quantized keys")
