"""GPU parity of kv2_attention_chunk (tcgen05) against the fp64 oracle on the
same packed cache and the kernel's operand precision (fp16 keys =
fp16(code s + fp16(z + centre)), fp16 values = fp16(code s + z), fp16 q P,
self keys and values rounded to fp16): max-abs 2e-3 and relative L2 1e-3
on the fp32 output, and the bf16 output against the bf16 rounding of the
oracle. Also: the block-causal frame mask, empty cache, ragged tiles, and the
bounded device-side wait that reports a timeout instead of hanging."""
import os

import numpy as np
import pytest
import torch

import workloads as wl
from helpers import assert_attention_close, assert_bf16_attention_close, bf16_round, gpu_cache_like, host_cache, to_dev

pytestmark = pytest.mark.gpu


def _basis(s, seed):
    rng = np.random.default_rng(seed)
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    for h in range(s.H_kv):
        q, _ = np.linalg.qr(rng.standard_normal((s.d, s.d)))
        P[h] = q[:, :s.r]
    return P


def _dense(rng, shape, scale=1.0):
    return wl.bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _run(orc, pc, P, length, Q, Ks, Vs, F, rows=None, out_dtype=0, ws=None):
    import bit_kv_cache_centroid_b200 as kv2
    B, Nq, H_q, d = Q.shape
    gc = gpu_cache_like(pc)
    if pc.r:
        gc.P.copy_(torch.from_numpy(np.ascontiguousarray(P)))
    scale = 1.0 / np.sqrt(d)
    out = kv2.kv2_attention_chunk(gc, length, to_dev(Q, torch.int16), to_dev(Ks, torch.int16),
                                  to_dev(Vs, torch.int16), F, scale, out_dtype=out_dtype, ws=ws)
    torch.cuda.synchronize()
    out = out.float().cpu().numpy()
    if rows is None:
        rows = np.array([(b, i, hq) for b in range(B) for i in range(Nq) for hq in range(H_q)], np.int32)
    ref = orc.chunk(pc, P, length, Q, Ks, Vs, F, scale, rows)
    got = out[rows[:, 0], rows[:, 1], rows[:, 2]]
    return got, ref


def test_oracle_quantized_cache_all_rows(orc):
    """Cache written by the oracle's quantizer from video-law keys."""
    s = wl.spec("quant_append", H_q=2, H_kv=2, T=300, n_new=1, n_hist=128, Nq=0, frame_tokens=150, M=64)
    w = wl.make("quant_append", **{k: getattr(s, k) for k in ("H_q", "H_kv", "T", "n_new", "n_hist", "Nq",
                                                                "frame_tokens", "M")})
    f = orc.fit(w.Qhist, s.H_kv, s.r)
    pc = host_cache(s, w.centroids)
    orc.quantize(pc, w.K[:, :s.T], w.V[:, :s.T], 0, s.C, f.P, f.w, f.Wg)
    rng = np.random.default_rng(4)
    Nq, F = 200, 64
    Q = _dense(rng, (1, Nq, 2, 128))
    Ks = _dense(rng, (1, Nq, 2, 128), 2.0)
    Vs = _dense(rng, (1, Nq, 2, 128))
    got, ref = _run(orc, pc, f.P, s.T, Q, Ks, Vs, F)
    assert_attention_close(got, ref, what="oracle-quantized cache")


@pytest.mark.parametrize("H_q,H_kv,M,r,T,length,Nq,F,B", [
    (2, 2, 64, 8, 512, 512, 256, 128, 1),     # whole tiles, frames = tiles
    (4, 2, 256, 8, 700, 613, 300, 100, 1),    # GQA, ragged cache and query tiles, frames split tiles
    (2, 2, 512, 16, 400, 257, 130, 65, 2),    # u16 ids, rank 16, batch 2
    (2, 2, 64, 0, 300, 300, 129, 43, 1),      # no PSAC
    (2, 2, 64, 8, 256, 0, 200, 50, 1),        # empty cache: self attention only
    (2, 2, 32, 8, 256, 1, 64, 64, 1),         # one cached token
])
def test_random_packed_caches(orc, H_q, H_kv, M, r, T, length, Nq, F, B):
    s = wl.spec("tiny", d=128, H_q=H_q, H_kv=H_kv, M=M, r=r, T=T, B=B)
    pc = wl.random_packed_cache(s, T=T, seed=M + r + T)
    P = _basis(s, 5)
    rng = np.random.default_rng(Nq + F)
    Q = _dense(rng, (B, Nq, H_q, 128), 1.5)
    Ks = _dense(rng, (B, Nq, H_kv, 128), 1.5)
    Vs = _dense(rng, (B, Nq, H_kv, 128))
    got, ref = _run(orc, pc, P, length, Q, Ks, Vs, F)
    assert_attention_close(got, ref, what=f"chunk M{M} r{r} len{length} Nq{Nq} F{F}")


def test_bf16_output(orc):
    s = wl.spec("tiny", d=128, H_q=2, H_kv=2, M=64, r=8, T=400)
    pc = wl.random_packed_cache(s, T=400, seed=3)
    P = _basis(s, 6)
    rng = np.random.default_rng(8)
    Q = _dense(rng, (1, 160, 2, 128))
    Ks = _dense(rng, (1, 160, 2, 128))
    Vs = _dense(rng, (1, 160, 2, 128))
    got, ref = _run(orc, pc, P, 400, Q, Ks, Vs, 80, out_dtype=1)
    assert_bf16_attention_close(got, ref, what="bf16 out")


def test_frame_mask_is_block_causal(orc):
    """Self keys of later frames are made overwhelmingly attractive; a query
    must still ignore them (its output is the oracle's, which masks them)."""
    s = wl.spec("tiny", d=128, H_q=2, H_kv=2, M=16, r=8, T=128)
    pc = wl.random_packed_cache(s, T=128, seed=1)
    P = _basis(s, 1)
    rng = np.random.default_rng(2)
    Nq, F = 256, 64
    Qf = np.abs(rng.standard_normal((1, Nq, 2, 128))).astype(np.float32)
    Kf = rng.standard_normal((1, Nq, 2, 128)).astype(np.float32) * 0.1
    Kf[:, 128:] = 3.0                        # frames 2, 3: huge logits for every query
    Vf = rng.standard_normal((1, Nq, 2, 128)).astype(np.float32)
    got, ref = _run(orc, pc, P, 128, wl.bf16_bits(Qf), wl.bf16_bits(Kf), wl.bf16_bits(Vf), F)
    assert_attention_close(got, ref, what="frame mask")


@pytest.mark.slow
def test_video_chunk_full_size_sampled(orc):
    """Video world-model chunk: 40 heads, 37,440 cached tokens (24 latent
    frames of 30x52), 4,680 queries (3 frames) block-causal over themselves,
    M=256, r=8; the oracle recomputes 24 sampled query rows."""
    s = wl.spec("video_chunk")
    pc = wl.random_packed_cache(s, T=s.T)
    P = _basis(s, 7)
    rng = np.random.default_rng(12)
    Q = _dense(rng, (1, s.Nq, s.H_q, 128))
    Ks = _dense(rng, (1, s.Nq, s.H_kv, 128))
    Vs = _dense(rng, (1, s.Nq, s.H_kv, 128))
    picks = [0, 127, 128, 1559, 1560, 3119, 3120, 4600, s.Nq - 1] + list(rng.integers(0, s.Nq, 15))
    rows = np.array([(0, int(i), int(rng.integers(0, s.H_q))) for i in picks], np.int32)
    # the last heads' units run as key-range pieces on a 148-SM GPU: sample them too
    rows = np.concatenate([rows, np.array([(0, int(i), s.H_q - 1) for i in (0, 2000, 4607, s.Nq - 1)] +
                                          [(0, 4620, s.H_q - 2)], np.int32)])
    got, ref = _run(orc, pc, P, s.T, Q, Ks, Vs, s.frame_tokens, rows=rows)
    assert_attention_close(got, ref, what="video chunk full size")


@pytest.mark.slow
def test_long_horizon_chunk_full_size_sampled(orc):
    """Long-horizon memory: 187,200 cached tokens (frames 30/60/90 revisit
    frame 0), 4,680-query chunk, M=512 (u16 ids), r=16; 8 sampled rows."""
    s = wl.spec("long_horizon")
    pc = wl.random_packed_cache(s, T=s.T, revisit_every=30)
    P = _basis(s, 8)
    rng = np.random.default_rng(13)
    Q = _dense(rng, (1, s.Nq, s.H_q, 128))
    Ks = _dense(rng, (1, s.Nq, s.H_kv, 128))
    Vs = _dense(rng, (1, s.Nq, s.H_kv, 128))
    picks = [0, 1560, 3119, s.Nq - 1, 777, 2000, 4000, 4500]
    rows = np.array([(0, i, (7 * k) % s.H_q) for k, i in enumerate(picks)], np.int32)
    got, ref = _run(orc, pc, P, s.T, Q, Ks, Vs, s.frame_tokens, rows=rows)
    assert_attention_close(got, ref, what="long-horizon chunk full size")


def test_last_wave_split_into_key_ranges(orc):
    """150 units (75 heads x 2 query-tile pairs) on a 148-SM GPU: the last
    wave's 2 units run as ranges of key tiles whose partial results are merged;
    every row of the split head and rows of whole units match the oracle."""
    s = wl.spec("tiny", d=128, H_q=75, H_kv=75, M=32, r=8, T=1024, B=1)
    pc = wl.random_packed_cache(s, T=1024, seed=11)
    P = _basis(s, 9)
    rng = np.random.default_rng(21)
    Nq, F = 300, 100
    Q = _dense(rng, (1, Nq, 75, 128))
    Ks = _dense(rng, (1, Nq, 75, 128))
    Vs = _dense(rng, (1, Nq, 75, 128))
    rows = [(0, i, 74) for i in range(Nq)] + [(0, i, h) for i, h in ((0, 0), (299, 3), (150, 40), (257, 73))]
    got, ref = _run(orc, pc, P, 1024, Q, Ks, Vs, F, rows=np.array(rows, np.int32))
    assert_attention_close(got, ref, what="split last wave")


def test_bounded_wait_reports_timeout_and_context_survives(orc):
    """A wait on a barrier that nothing completes runs out of its budget: the
    kernel records 1 in the workspace's first word, frees its TMEM and returns;
    the next normal call on the same context is correct."""
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=128, H_q=2, H_kv=2, M=16, r=8, T=128)
    pc = wl.random_packed_cache(s, T=128, seed=4)
    P = _basis(s, 4)
    rng = np.random.default_rng(3)
    Q = _dense(rng, (1, 128, 2, 128))
    Ks = _dense(rng, (1, 128, 2, 128))
    Vs = _dense(rng, (1, 128, 2, 128))
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    os.environ["KV2_FORCE_WAIT_TIMEOUT"] = "1"
    try:
        _run(orc, pc, P, 128, Q, Ks, Vs, 64, ws=ws)
    finally:
        del os.environ["KV2_FORCE_WAIT_TIMEOUT"]
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 1
    got, ref = _run(orc, pc, P, 128, Q, Ks, Vs, 64, ws=ws)
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert_attention_close(got, ref, what="after timeout")


@pytest.mark.parametrize("M,r,T,length,Nq,F", [
    (256, 8, 700, 613, 300, 100),
    (512, 16, 400, 257, 130, 65),
])
def test_int8_psac_caches(orc, M, r, T, length, Nq, F):
    """Int8 PSAC coefficients with per-token fp16 scales; the kernel's PSAC
    operand is fp16(code * scale), as the oracle takes it."""
    s = wl.spec("tiny", d=128, H_q=4, H_kv=2, M=M, r=r, T=T, B=1)
    pc = wl.random_packed_cache(s, T=T, seed=M + r + 11, psac_fmt=1)
    P = _basis(s, 7)
    rng = np.random.default_rng(Nq + F + 1)
    Q = _dense(rng, (1, Nq, 4, 128), 1.5)
    Ks = _dense(rng, (1, Nq, 2, 128), 1.5)
    Vs = _dense(rng, (1, Nq, 2, 128))
    got, ref = _run(orc, pc, P, length, Q, Ks, Vs, F)
    assert_attention_close(got, ref, what=f"chunk int8 psac M{M} r{r}")
