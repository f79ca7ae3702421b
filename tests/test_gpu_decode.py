"""GPU parity of kv2_attention_decode against the fp64 oracle on the same
packed cache: max-abs 2e-3 and relative L2 1e-3 (fp32 output), and the bf16
output against the bf16 rounding of the oracle at the same thresholds."""
import numpy as np
import pytest
import torch

import workloads as wl
from helpers import assert_attention_close, assert_bf16_attention_close, bf16_round, gpu_cache_like, host_cache, to_dev

pytestmark = pytest.mark.gpu


def _decode_both(orc, pc, P, length, Q, scale, out_dtype=0):
    import bit_kv_cache_centroid_b200 as kv2
    ref = orc.decode(pc, P, length, Q, scale)
    gc = gpu_cache_like(pc)
    if pc.r:
        gc.P.copy_(torch.from_numpy(np.ascontiguousarray(P)))
    out = kv2.kv2_attention_decode(gc, length, to_dev(Q, torch.int16), scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), ref


def _basis(s, seed):
    rng = np.random.default_rng(seed)
    P = np.zeros((s.H_kv, s.d, max(s.r, 0)), np.float32)
    for h in range(s.H_kv):
        q, _ = np.linalg.qr(rng.standard_normal((s.d, s.d)))
        P[h] = q[:, :s.r]
    return P


def test_tiny_oracle_quantized_cache(orc):
    w = wl.make("tiny")
    s = w.spec
    f = orc.fit(w.Qhist, s.H_kv, s.r)
    pc = host_cache(s, w.centroids)
    orc.quantize(pc, w.K[:, :s.T], w.V[:, :s.T], 0, s.C, f.P, f.w, f.Wg)
    scale = 1.0 / np.sqrt(s.d)
    got, ref = _decode_both(orc, pc, f.P, s.T, w.Qdec, scale)
    assert_attention_close(got, ref, what="tiny f32")
    got16, _ = _decode_both(orc, pc, f.P, s.T, w.Qdec, scale, out_dtype=1)
    assert_bf16_attention_close(got16, ref, what="tiny bf16")


@pytest.mark.parametrize("d,G,M,r,T,length", [
    (128, 4, 64, 8, 1200, 1),          # one token
    (128, 4, 64, 8, 1200, 127),        # under one tile
    (128, 4, 64, 8, 1200, 129),        # one tile + 1
    (128, 1, 512, 16, 5200, 5137),     # MHA, u16 ids, rank 16, many tiles + ragged tail
    (128, 2, 256, 0, 3000, 2999),      # no PSAC
    (128, 8, 64, 8, 2100, 2049),       # 8 query heads per KV head
    (64, 4, 16, 8, 900, 899),          # d = 64
])
def test_random_packed_caches(orc, d, G, M, r, T, length):
    s = wl.spec("tiny", d=d, H_kv=2, H_q=2 * G, M=M, r=r, T=T, B=2)
    pc = wl.random_packed_cache(s, T=T, seed=d + G + M + r)
    P = _basis(s, 3)
    rng = np.random.default_rng(T)
    Q = wl.bf16_bits(rng.standard_normal((s.B, s.H_q, d)).astype(np.float32) * 1.5)
    got, ref = _decode_both(orc, pc, P, length, Q, 1.0 / np.sqrt(d))
    assert_attention_close(got, ref, what=f"d{d} G{G} M{M} r{r} len{length}")


def test_empty_cache_gives_zeros(orc):
    s = wl.spec("tiny", T=64)
    pc = wl.random_packed_cache(s, T=64)
    Q = wl.bf16_bits(np.ones((1, s.H_q, s.d), np.float32))
    got, ref = _decode_both(orc, pc, _basis(s, 1), 0, Q, 0.125)
    assert np.all(got == 0.0) and np.all(ref == 0.0)


def test_peaked_attention(orc):
    """A query aligned with one cached key: the softmax is nearly one-hot, so
    errors in the logits would show directly in the output."""
    s = wl.spec("tiny", d=128, H_q=4, H_kv=4, M=64, r=8, T=600)
    pc = wl.random_packed_cache(s, T=600, seed=5)
    P = _basis(s, 2)
    rng = np.random.default_rng(1)
    Q = wl.bf16_bits(rng.standard_normal((1, 4, 128)).astype(np.float32) * 6.0)
    got, ref = _decode_both(orc, pc, P, 600, Q, 1.0 / np.sqrt(128))
    assert_attention_close(got, ref, what="peaked")


@pytest.mark.slow
def test_llm_decode_full_size_sampled(orc):
    """The LLM decode workload (batch 8, 32/8 heads, d=128, 32,768 cached
    tokens, M=64, r=8) in the launch configuration the benchmark times; the
    oracle recomputes the outputs of two sequences."""
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("llm_decode")
    pc = wl.random_packed_cache(s, T=s.T)
    P = _basis(s, 7)
    rng = np.random.default_rng(2)
    Q = wl.bf16_bits(rng.standard_normal((s.B, s.H_q, s.d)).astype(np.float32))
    gc = gpu_cache_like(pc)
    gc.P.copy_(torch.from_numpy(P))
    scale = 1.0 / np.sqrt(s.d)
    out = kv2.kv2_attention_decode(gc, s.T, to_dev(Q, torch.int16), scale, out_dtype=kv2.KV2_OUT_BF16)
    out32 = kv2.kv2_attention_decode(gc, s.T, to_dev(Q, torch.int16), scale)
    torch.cuda.synchronize()
    for b in (0, s.B - 1):
        sub = wl.PackedCache(1, s.H_kv, s.d, s.M, s.r, pc.capacity, pc.k_code[b:b + 1], pc.v_code[b:b + 1],
                             pc.k_sz[b:b + 1], pc.v_sz[b:b + 1], pc.cidx[b:b + 1], pc.psac[b:b + 1],
                             pc.centroids)
        ref = orc.decode(sub, P, s.T, Q[b:b + 1], scale)
        assert_attention_close(out32[b:b + 1].cpu().numpy(), ref, what=f"llm f32 b{b}")
        assert_bf16_attention_close(out[b:b + 1].float().cpu().numpy(), ref, what=f"llm bf16 b{b}")


@pytest.mark.slow
def test_long_horizon_decode_full_size_sampled(orc):
    """Long-horizon memory: 187,200 cached tokens (120 latent frames, frames
    30/60/90 revisiting frame 0), 40 heads, M=512, r=16, one query per head;
    the oracle recomputes 4 heads."""
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("long_horizon")
    pc = wl.random_packed_cache(s, T=s.T, revisit_every=30)
    P = _basis(s, 9)
    rng = np.random.default_rng(3)
    Q = wl.bf16_bits(rng.standard_normal((1, s.H_q, s.d)).astype(np.float32))
    gc = gpu_cache_like(pc)
    gc.P.copy_(torch.from_numpy(P))
    scale = 1.0 / np.sqrt(s.d)
    out = kv2.kv2_attention_decode(gc, s.T, to_dev(Q, torch.int16), scale).cpu().numpy()
    heads = [0, 13, 27, 39]
    sub = wl.PackedCache(1, len(heads), s.d, s.M, s.r, pc.capacity, pc.k_code[:, heads], pc.v_code[:, heads],
                         pc.k_sz[:, heads], pc.v_sz[:, heads], pc.cidx[:, heads], pc.psac[:, heads],
                         pc.centroids[heads])
    ref = orc.decode(sub, P[heads], s.T, Q[:, heads], scale)
    assert_attention_close(out[:, heads], ref, what="long-horizon decode")


def test_bounded_wait_reports_timeout_and_context_survives(orc):
    """Copies that are never issued: every wait on a tile runs out of its
    budget, the kernel sets the workspace's error word, writes NaN for the
    affected heads and returns; the next normal call on the same context is
    correct (the error word stays set until the caller clears it)."""
    import os
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=128, H_q=8, H_kv=2, M=64, r=8, T=600, B=1)
    pc = wl.random_packed_cache(s, T=600, seed=9)
    P = _basis(s, 4)
    rng = np.random.default_rng(5)
    Q = to_dev(wl.bf16_bits(rng.standard_normal((1, s.H_q, s.d)).astype(np.float32)), torch.int16)
    gc = gpu_cache_like(pc)
    gc.P.copy_(torch.from_numpy(P))
    ws = torch.zeros(kv2.kv2_decode_workspace_size(gc, s.H_q, 600), dtype=torch.uint8, device="cuda")
    os.environ["KV2_FORCE_WAIT_TIMEOUT"] = "1"
    try:
        bad = kv2.kv2_attention_decode(gc, 600, Q, 0.1, ws=ws)
    finally:
        del os.environ["KV2_FORCE_WAIT_TIMEOUT"]
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 1
    assert torch.isnan(bad).all()
    ws.zero_()
    good = kv2.kv2_attention_decode(gc, 600, Q, 0.1, ws=ws).cpu().numpy()
    assert int(ws[:4].view(torch.int32).item()) == 0
    ref = orc.decode(pc, P, 600, Q.cpu().numpy().view(np.uint16), 0.1)
    assert_attention_close(good, ref, what="after timeout")


@pytest.mark.parametrize("B,H_q,H_kv,M,r,T,n_new", [
    (8, 32, 8, 64, 8, 3000, 1),       # decode step: one token per sequence, tile boundary inside a split
    (2, 8, 2, 512, 16, 700, 5),       # several tokens, u16 ids, rank 16
    (1, 4, 4, 64, 8, 127, 1),         # appended token in the first (only) tile
    (2, 8, 2, 64, 8, 700, 100),       # a long append: key kernel, value kernel, then decode
])
def test_append_attention_decode_equals_the_two_calls(orc, B, H_q, H_kv, M, r, T, n_new):
    """kv2_append_attention_decode (append kernel, then the decode kernel as its
    programmatic dependent) leaves the same packed bytes and returns the same
    outputs, bit for bit, as kv2_quantize_append followed by
    kv2_attention_decode; the outputs also match the oracle."""
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=128, H_q=H_q, H_kv=H_kv, M=M, r=r, T=T + n_new, B=B)
    pc = wl.random_packed_cache(s, T=T + n_new, seed=T)
    P = _basis(s, 6)
    rng = np.random.default_rng(T + 1)
    Kn = wl.bf16_bits(rng.standard_normal((B, n_new, H_kv, 128)).astype(np.float32))
    Vn = wl.bf16_bits(rng.standard_normal((B, n_new, H_kv, 128)).astype(np.float32))
    Q = to_dev(wl.bf16_bits(rng.standard_normal((B, H_q, 128)).astype(np.float32)), torch.int16)
    w = np.abs(rng.standard_normal((H_kv, 128))).astype(np.float32) + 0.1
    Wg = w.reshape(H_kv, 4, 32).sum(-1).astype(np.float32)
    scale = 1.0 / np.sqrt(128)
    outs, caches = [], []
    for fused in (False, True):
        gc = gpu_cache_like(pc)
        gc.set_fit(torch.from_numpy(P), torch.from_numpy(w), torch.from_numpy(Wg))
        Kd, Vd = to_dev(Kn, torch.int16), to_dev(Vn, torch.int16)
        if fused:
            o = kv2.kv2_append_attention_decode(gc, Kd, Vd, T, 4, Q, scale)
        else:
            kv2.kv2_quantize_append(gc, Kd, Vd, T, 4)
            o = kv2.kv2_attention_decode(gc, T + n_new, Q, scale)
        torch.cuda.synchronize()
        outs.append(o.cpu().numpy())
        caches.append(gc.to_host())
    for name in ("k_code", "v_code", "k_sz", "v_sz", "cidx", "psac"):
        np.testing.assert_array_equal(caches[0][name], caches[1][name], err_msg=name)
    np.testing.assert_array_equal(outs[0], outs[1])
    host = wl.PackedCache(B, H_kv, 128, M, r, pc.capacity,
                          caches[1]["k_code"], caches[1]["v_code"], caches[1]["k_sz"], caches[1]["v_sz"],
                          caches[1]["cidx"], caches[1]["psac"], pc.centroids)
    ref = orc.decode(host, P, T + n_new, Q.cpu().numpy().view(np.uint16), scale)
    assert_attention_close(outs[1], ref, what=f"append+decode B{B} T{T} n{n_new}")


@pytest.mark.parametrize("d,G,M,r,T,length", [
    (128, 4, 64, 8, 1200, 1100),       # LLM-like table, rank 8
    (128, 1, 512, 16, 2100, 2049),     # MHA, u16 ids, rank 16
    (64, 4, 16, 8, 900, 899),          # d = 64
])
def test_int8_psac_caches(orc, d, G, M, r, T, length):
    """Int8 PSAC coefficients with per-token fp16 scales (the oracle reads
    them back exactly as code * scale)."""
    s = wl.spec("tiny", d=d, H_kv=2, H_q=2 * G, M=M, r=r, T=T, B=2)
    pc = wl.random_packed_cache(s, T=T, seed=d + G + M + r + 7, psac_fmt=1)
    P = _basis(s, 4)
    rng = np.random.default_rng(T + 1)
    Q = wl.bf16_bits(rng.standard_normal((s.B, s.H_q, d)).astype(np.float32) * 1.5)
    got, ref = _decode_both(orc, pc, P, length, Q, 1.0 / np.sqrt(d))
    assert_attention_close(got, ref, what=f"int8 psac d{d} G{G} M{M} r{r} len{length}")


def test_int8_psac_oracle_quantized_cache(orc):
    """Keys appended by the oracle's quantizer in the int8 PSAC format."""
    w = wl.make("tiny")
    s = w.spec
    f = orc.fit(w.Qhist, s.H_kv, s.r)
    pc = host_cache(s, w.centroids, psac_fmt=1)
    orc.quantize(pc, w.K[:, :s.T], w.V[:, :s.T], 0, s.C, f.P, f.w, f.Wg)
    got, ref = _decode_both(orc, pc, f.P, s.T, w.Qdec, 1.0 / np.sqrt(s.d))
    assert_attention_close(got, ref, what="int8 psac oracle-quantized")
