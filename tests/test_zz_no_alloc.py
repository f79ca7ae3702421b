"""kv2_attention_decode_noalloc — decode attention for callers that may not
allocate device memory (its scratch is a fixed array inside the library).

Called through the C ABI and compared with kv2_attention_decode (which takes a
caller-allocated workspace) on the same cache and queries, twice in a row, so
that the second call also sees the scratch the first one left behind. The file
sorts last so that a run stopping at the first failure has run every other test.
"""
import ctypes

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
    Q = to_dev(wl.bf16_bits(rng.standard_normal((s.B, s.H_q, s.d)).astype(np.float32)), torch.int16)
    return s, gc, Q


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


@pytest.mark.parametrize("T,length,ov", [
    (5000, 4999, dict(d=128, H_q=8, H_kv=2, M=64, r=8, B=2)),
    (3000, 2001, dict(d=128, H_q=4, H_kv=4, M=512, r=16, B=1)),
])
def test_noalloc_matches_workspace_decode_twice(T, length, ov):
    import bit_kv_cache_centroid_b200 as kv2
    s, gc, Q = _setup(T, 21, **ov)
    scale = 1.0 / np.sqrt(s.d)
    ref = kv2.kv2_attention_decode(gc, length, Q, scale)
    first = _noalloc(kv2, gc, length, Q, scale)
    second = _noalloc(kv2, gc, length, Q, scale)
    torch.cuda.synchronize()
    r = ref.cpu().numpy()
    assert_attention_close(first.cpu().numpy(), r, what="noalloc first call")
    assert_attention_close(second.cpu().numpy(), r, what="noalloc second call")


def test_noalloc_rejects_shapes_beyond_the_array():
    import bit_kv_cache_centroid_b200 as kv2
    s = wl.spec("tiny", d=128, H_q=64, H_kv=64, M=512, r=16, B=512, T=16)
    c = kv2.Cache(s.B, s.H_kv, s.d, s.M, s.r, 32, torch.zeros(s.H_kv, s.M, s.d, dtype=torch.int16))
    Q = torch.zeros(s.B, s.H_q, s.d, dtype=torch.int16, device="cuda")
    assert kv2.kv2_decode_workspace_size(c, s.H_q, 16) > 8 << 20
    with pytest.raises(kv2.Kv2Error) as e:
        kv2.kv2_attention_decode_noalloc(c, 16, Q, 0.1)
    assert e.value.status == 6 and "fixed array" in str(e.value)
