"""kv2_attention_decode_noalloc — decode attention for callers that may not
allocate device memory (its scratch is a fixed array inside the library), and
kv2_decode_noalloc_error, which reads and clears that array's error word.

Called through the C ABI and compared with kv2_attention_decode (which takes a
caller-allocated workspace) and with the oracle on the same cache and queries.
Within one test the shapes change from call to call (many splits, then fewer
splits with other head counts and head dimension, then the first shape
again), so that each call runs over scratch another shape left behind. The
file sorts last so that a run stopping at the first failure has run every
other test.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import workloads as wl
from helpers import assert_attention_close, gpu_cache_like, to_dev

pytestmark = pytest.mark.gpu


def _setup(T, seed, **ov):
    s = wl.spec("tiny", T=T, **ov)
    pc = wl.random_packed_cache(s, T=T, seed=seed)
    rng = np.random.default_rng(seed)
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    for h in range(s.H_kv):
        q, _ = np.linalg.qr(rng.standard_normal((s.d, s.d)))
        P[h] = q[:, :s.r]
    gc = gpu_cache_like(pc)
    gc.P.copy_(torch.from_numpy(P))
    Qh = wl.bf16_bits(rng.standard_normal((s.B, s.H_q, s.d)).astype(np.float32))
    return s, pc, P, gc, Qh, to_dev(Qh, torch.int16)


def _noalloc(kv2, gc, length, Q, scale):
    B, H_q, d = Q.shape
    out = torch.zeros((B, H_q, d), dtype=torch.float32, device="cuda")
    desc = gc.desc()
    rc = kv2.lib.kv2_attention_decode_noalloc(ctypes.byref(desc), length, ctypes.c_void_p(Q.data_ptr()), H_q,
                                              ctypes.c_float(scale), ctypes.c_void_p(out.data_ptr()),
                                              kv2.KV2_OUT_F32,
                                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, kv2.lib.kv2_last_error().decode()
    return out


def _error_word(kv2, clear):
    flag = ctypes.c_int(-1)
    rc = kv2.lib.kv2_decode_noalloc_error(ctypes.byref(flag), int(clear),
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, kv2.lib.kv2_last_error().decode()
    return flag.value


CASES = [
    (5000, 4999, 21, dict(d=128, H_q=8, H_kv=2, M=64, r=8, B=2)),     # many splits per (batch, head)
    (3000, 2001, 22, dict(d=128, H_q=4, H_kv=4, M=512, r=16, B=1)),   # u16 ids, rank 16, MHA
    (700, 650, 23, dict(d=64, H_q=16, H_kv=2, M=32, r=8, B=3)),       # few splits, d = 64, 8 heads per group
]


def test_noalloc_matches_workspace_decode_and_oracle_across_shapes(orc):
    """Shapes 0, 1, 2, then 0 again, each called twice in a row: both calls
    equal the workspace decode's output and the oracle's within the attention
    tolerance."""
    import bit_kv_cache_centroid_b200 as kv2
    assert _error_word(kv2, clear=False) == 0
    setups = [_setup(T, seed, **ov) for T, _, seed, ov in CASES]
    for idx in (0, 1, 2, 0):
        s, pc, P, gc, Qh, Q = setups[idx]
        length = CASES[idx][1]
        scale = 1.0 / np.sqrt(s.d)
        ref = kv2.kv2_attention_decode(gc, length, Q, scale).cpu().numpy()
        want = orc.decode(pc, P, length, Qh, scale)
        for call in ("first", "second"):
            got = _noalloc(kv2, gc, length, Q, scale)
            torch.cuda.synchronize()
            got = got.cpu().numpy()
            assert_attention_close(got, ref, what=f"case {idx} noalloc {call} call vs workspace decode")
            assert_attention_close(got, want, what=f"case {idx} noalloc {call} call vs oracle")
    assert _error_word(kv2, clear=False) == 0


def test_noalloc_error_word_reports_a_timeout_and_clears():
    """Tile copies that are never issued (KV2_FORCE_WAIT_TIMEOUT=1): every wait
    runs out of its budget, the outputs are NaN and the fixed array's error
    word reads 1; clearing it reads 0 afterwards, and the next call is correct."""
    import bit_kv_cache_centroid_b200 as kv2
    T, length, seed, ov = CASES[0]
    s, pc, P, gc, Qh, Q = _setup(T, seed, **ov)
    scale = 1.0 / np.sqrt(s.d)
    _error_word(kv2, clear=True)
    os.environ["KV2_FORCE_WAIT_TIMEOUT"] = "1"
    try:
        bad = _noalloc(kv2, gc, length, Q, scale)
    finally:
        del os.environ["KV2_FORCE_WAIT_TIMEOUT"]
    torch.cuda.synchronize()
    assert torch.isnan(bad).all()
    assert _error_word(kv2, clear=True) == 1
    assert _error_word(kv2, clear=False) == 0
    good = _noalloc(kv2, gc, length, Q, scale)
    torch.cuda.synchronize()
    ref = kv2.kv2_attention_decode(gc, length, Q, scale).cpu().numpy()
    assert_attention_close(good.cpu().numpy(), ref, what="noalloc after a cleared timeout")
    assert _error_word(kv2, clear=False) == 0


def test_noalloc_rejects_shapes_beyond_the_array():
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=128, H_q=64, H_kv=64, M=512, r=16, B=512, T=16)
    c = kv2.Cache(s.B, s.H_kv, s.d, s.M, s.r, 32, torch.zeros(s.H_kv, s.M, s.d, dtype=torch.int16))
    Q = torch.zeros(s.B, s.H_q, s.d, dtype=torch.int16, device="cuda")
    assert kv2.kv2_decode_workspace_size(c, s.H_q, 16) > 8 << 20
    with pytest.raises(kv2.Kv2Error) as e:
        kv2.kv2_attention_decode_noalloc(c, 16, Q, 0.1)
    assert e.value.status == 6 and "fixed array" in str(e.value)
