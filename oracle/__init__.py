"""CPU oracle of the 2-bit KV-cache path — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. It wraps ``kv2_oracle.c`` (plain single-threaded C,
fp64 attention, fp32 quantizer decisions in a stated order) through ctypes and
shares no code with the CUDA library.

Method: "QuantWM: Training-Free 2-bit KV Cache Quantization for Stable Video
World Models", sections "1. Quantization Sensitivity-Aware Clustering (QSAC)"
and "2. Principal Subspace Attention Compensation (PSAC)". Every function's
reading of the pages is stated in the C source next to it.

Parity unpinned: whether the perturbation estimate E_j is the authors' exact
heuristic — the pages describe it in words and print no worked example; only its
internal consistency (brute-force argmin, closed forms) is pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kv2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
          "-fno-fast-math", "-mfma", "-lm"]

RND_NEAREST_EVEN, RND_DOWN, RND_UP = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (skipped when current)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", _SRC, "-o", tmp] + CFLAGS, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int


def _declare(L):
    L.or_f16_from_f32.argtypes = [ctypes.c_float, _I]
    L.or_f16_from_f32.restype = ctypes.c_uint16
    L.or_f32_from_f16.argtypes = [ctypes.c_uint16]
    L.or_f32_from_f16.restype = ctypes.c_float
    L.or_bf16_from_f32.argtypes = [ctypes.c_float]
    L.or_bf16_from_f32.restype = ctypes.c_uint16
    L.or_f32_from_bf16.argtypes = [ctypes.c_uint16]
    L.or_f32_from_bf16.restype = ctypes.c_float
    L.or_codec_group.argtypes = [_P, _I, _P, _P, _P, _P]
    # the last argument of each is the group size (channels per scale, zero)
    L.or_fit.argtypes = [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I]
    L.or_quantize.argtypes = ([_I] * 6 + [_P, _P, _I, _I, _I, _P, _P, _P, _P] + [_P] * 6 + [_I, _P, _P, _I]
                              + [_P] * 3 + [_I])
    L.or_decode.argtypes = ([_I] * 6 + [_P] * 6 + [_I, _P, _P, _I] + [_P] * 2
                            + [_I, _P, _I, ctypes.c_double, _P, _I])
    L.or_chunk.argtypes = ([_I] * 6 + [_P] * 6 + [_I, _P, _P, _I] + [_P] * 2 + [_I, _P, _I, _I, _P, _P, _I,
                                                  ctypes.c_double, _P, _I, _P, _I])
    L.or_decode_logits.argtypes = [_I] * 7 + [_P] * 4 + [_I, _P, _P, _I] + [_P] * 2 + [_I, _P, _P, _I]
    L.or_fit_centroids.argtypes = [_I] * 5 + [_P, _P, _P, _I, _P, _P, _I]
    for f in (L.or_codec_group, L.or_fit, L.or_quantize, L.or_decode, L.or_chunk,
              L.or_decode_logits, L.or_fit_centroids):
        f.restype = _I if f is not L.or_codec_group else None


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ----------------------------------------------------------------------------
# scalar conversions (IEEE 754 definitions)
# ----------------------------------------------------------------------------

def f16_from_f32(x: float, mode: int = RND_NEAREST_EVEN) -> int:
    return int(lib().or_f16_from_f32(float(x), mode))


def f32_from_f16(h: int) -> float:
    return float(lib().or_f32_from_f16(int(h)))


def bf16_from_f32(x: float) -> int:
    return int(lib().or_bf16_from_f32(float(x)))


def f32_from_bf16(b: int) -> float:
    return float(lib().or_f32_from_bf16(int(b)))


# ----------------------------------------------------------------------------
# codec, fit, quantize, attention
# ----------------------------------------------------------------------------

def codec_group(x: np.ndarray):
    """INT2 codec of one group: returns (scale_bits, zero_bits, codes, deq)."""
    x = _c(x, np.float32)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    codes = np.zeros(x.size, np.uint8)
    deq = np.zeros(x.size, np.float32)
    lib().or_codec_group(_ptr(x), x.size, _ptr(s), _ptr(z), _ptr(codes), _ptr(deq))
    return int(s[0]), int(z[0]), codes, deq


@dataclass
class Fit:
    P: np.ndarray       # fp32 [H_kv][d][r]
    w: np.ndarray       # fp32 [H_kv][d]
    Wg: np.ndarray      # fp32 [H_kv][d/group]
    evals: np.ndarray   # fp64 [H_kv][d], descending
    energy: np.ndarray  # fp64 [H_kv], top-r share of the energy


def fit(Qhist: np.ndarray, H_kv: int, r: int, group: int = 32) -> Fit:
    """PSAC basis + sensitivity weights from history queries bf16 [n][H_q][d];
    W sums w over groups of ``group`` channels."""
    Qhist = _c(Qhist, np.uint16)
    n, Hq, d = Qhist.shape
    P = np.zeros((H_kv, d, max(r, 1)), np.float32)[:, :, :r].copy()
    w = np.zeros((H_kv, d), np.float32)
    Wg = np.zeros((H_kv, max(d // group, 1)), np.float32)
    ev = np.zeros((H_kv, d), np.float64)
    en = np.zeros(H_kv, np.float64)
    rc = lib().or_fit(_ptr(Qhist), n, Hq, H_kv, d, r, _ptr(P), _ptr(w), _ptr(Wg), _ptr(ev), _ptr(en), group)
    if rc:
        raise ValueError("or_fit: bad arguments")
    return Fit(P, w, Wg, ev, en)


@dataclass
class QuantDebug:
    cand: np.ndarray    # int32 [B][n_new][H_kv][C]: candidates in rank order
    score: np.ndarray   # fp32 weighted distances D_j of the candidates
    E: np.ndarray       # fp32 perturbation estimates of the candidates


def quantize(pc, K: np.ndarray, V: np.ndarray, pos: int, C: int, P: np.ndarray,
             w: np.ndarray, Wg: np.ndarray, debug: bool = False):
    """Append K, V bf16 [B][n_new][H_kv][d] into packed cache ``pc`` (a
    ``workloads.PackedCache``, modified in place) at token ``pos``."""
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    B, n_new, Hkv, d = K.shape
    P = _c(P, np.float32)
    w = _c(w, np.float32)
    Wg = _c(Wg, np.float32)
    r = pc.r
    if Wg.shape[-1] != d // pc.group:
        raise ValueError(f"Wg has {Wg.shape[-1]} groups; the cache's groups of {pc.group} need {d // pc.group}")
    dbg = None
    if debug:
        dbg = QuantDebug(np.zeros((B, n_new, Hkv, C), np.int32),
                         np.zeros((B, n_new, Hkv, C), np.float32),
                         np.zeros((B, n_new, Hkv, C), np.float32))
    rc = lib().or_quantize(
        B, Hkv, d, pc.M, r, pc.capacity, _ptr(K), _ptr(V), n_new, pos, C,
        _ptr(_c(pc.centroids, np.uint16)), _ptr(P), _ptr(w), _ptr(Wg),
        _ptr(pc.k_code), _ptr(pc.v_code), _ptr(pc.k_sz), _ptr(pc.v_sz),
        _ptr(pc.cidx), *_psac_args(pc),
        _ptr(dbg.cand) if dbg else None, _ptr(dbg.score) if dbg else None,
        _ptr(dbg.E) if dbg else None, pc.group)
    if rc:
        raise ValueError("or_quantize: bad arguments")
    return dbg


def fit_centroids(X: np.ndarray, M: int, C: int, w: np.ndarray, Wg: np.ndarray,
                  centroids: np.ndarray, iters: int, group: int = 32):
    """QSAC-aware centre fitting (reading in ``kv2_oracle.c``): X bf16 bits
    [n][H_kv][d], initial centres fp16 bits [H_kv][M][d] -> (fitted centres
    fp16 bits [H_kv][M][d], last assignment int32 [n][H_kv])."""
    X = _c(X, np.uint16)
    n, Hkv, d = X.shape
    if np.shape(Wg)[-1] != d // group:
        raise ValueError("Wg does not match the group size")
    cent = np.array(_c(centroids, np.uint16), copy=True)
    assign = np.full((max(n, 1), Hkv), -1, np.int32)
    rc = lib().or_fit_centroids(n, Hkv, d, M, C, _ptr(X), _ptr(_c(w, np.float32)), _ptr(_c(Wg, np.float32)),
                                iters, _ptr(cent), _ptr(assign), group)
    if rc:
        raise ValueError("or_fit_centroids: bad arguments")
    return cent, assign[:n]


def _psac_args(pc):
    """(coefficients, format, per-token scales, block table, page tokens) of
    a packed cache: format 0 = fp16 [r], 1 = int8 [r] with one fp16 scale per
    token; a paged cache holds its streams as a pool of pages addressed
    through the block table [B][capacity / page]."""
    fmt = getattr(pc, "psac_fmt", 0)
    psac = pc.psac if pc.r else np.zeros(1, np.uint16)
    sc = pc.psac_scale if (fmt == 1 and pc.r) else np.zeros(1, np.uint16)
    table = getattr(pc, "table", None)
    return (_ptr(psac), fmt, _ptr(sc), _ptr(_c(table, np.int32)) if table is not None else None,
            int(getattr(pc, "page", 0)))


def _cache_args(pc):
    P = getattr(pc, "P", None)
    if P is None or pc.r == 0:
        P = np.zeros(1, np.float32)
    return (_ptr(pc.k_code), _ptr(pc.v_code), _ptr(pc.k_sz), _ptr(pc.v_sz),
            _ptr(pc.cidx), *_psac_args(pc), _ptr(_c(pc.centroids, np.uint16)),
            _ptr(_c(P, np.float32)))


def decode(pc, P: np.ndarray, length: int, Q: np.ndarray, sm_scale: float) -> np.ndarray:
    """fp64 decode attention: Q bf16 [B][H_q][d] -> out fp64 [B][H_q][d]."""
    Q = _c(Q, np.uint16)
    B, Hq, d = Q.shape
    pc.P = P
    out = np.zeros((B, Hq, d), np.float64)
    rc = lib().or_decode(pc.B, pc.H_kv, pc.d, pc.M, pc.r, pc.capacity, *_cache_args(pc),
                         length, _ptr(Q), Hq, float(sm_scale), _ptr(out), pc.group)
    if rc:
        raise ValueError("or_decode: bad arguments")
    return out


def chunk(pc, P: np.ndarray, length: int, Q: np.ndarray, Kself: np.ndarray,
          Vself: np.ndarray, frame_tokens: int, sm_scale: float,
          rows: np.ndarray) -> np.ndarray:
    """fp64 chunk attention for the (b, i, hq) rows listed: Q bf16
    [B][Nq][H_q][d], Kself/Vself bf16 [B][Nq][H_kv][d] -> out fp64 [nrows][d]."""
    Q = _c(Q, np.uint16)
    Kself = _c(Kself, np.uint16)
    Vself = _c(Vself, np.uint16)
    B, Nq, Hq, d = Q.shape
    rows = _c(rows, np.int32).reshape(-1, 3)
    pc.P = P
    out = np.zeros((rows.shape[0], d), np.float64)
    rc = lib().or_chunk(pc.B, pc.H_kv, pc.d, pc.M, pc.r, pc.capacity, *_cache_args(pc),
                        length, _ptr(Q), Hq, Nq, _ptr(Kself), _ptr(Vself), frame_tokens,
                        float(sm_scale), _ptr(rows), rows.shape[0], _ptr(out), pc.group)
    if rc:
        raise ValueError("or_chunk: bad arguments")
    return out


def decode_logits(pc, P: np.ndarray, b: int, h: int, length: int, q: np.ndarray) -> np.ndarray:
    """Unscaled fp64 logits of one fp64 query against (b, KV head h)."""
    q = _c(q, np.float64)
    pc.P = P
    out = np.zeros(length, np.float64)
    Pp = _c(P, np.float32) if pc.r else np.zeros(1, np.float32)
    rc = lib().or_decode_logits(pc.H_kv, pc.d, pc.M, pc.r, pc.capacity, b, h,
                                _ptr(pc.k_code), _ptr(pc.k_sz), _ptr(pc.cidx), *_psac_args(pc),
                                _ptr(_c(pc.centroids, np.uint16)), _ptr(Pp), length, _ptr(q), _ptr(out),
                                pc.group)
    if rc:
        raise ValueError("or_decode_logits: bad arguments")
    return out


def bf16_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> their exact values in fp64."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_top1(pc, P: np.ndarray, length: int, Q: np.ndarray):
    """Most-attended cached token per query: argmax over t < length of the
    fp64 logit q . khat_t + (q P) . a_t (first index among equal maxima), and
    the logits themselves. Q bf16 [B][nq][H_q][d] -> (int [B][nq][H_q],
    fp64 [B][nq][H_q][length])."""
    Q = _c(Q, np.uint16)
    B, nq, Hq, d = Q.shape
    G = Hq // pc.H_kv
    lg = np.zeros((B, nq, Hq, max(length, 1)), np.float64)
    for b in range(B):
        for i in range(nq):
            for hq in range(Hq):
                q = bf16_f64(Q[b, i, hq])
                if length:
                    lg[b, i, hq, :length] = decode_logits(pc, P, b, hq // G, length, q)
    top = np.argmax(lg[..., :length], axis=-1) if length else np.full((B, nq, Hq), -1)
    return top, lg[..., :length]


def dense_top1(K: np.ndarray, Q: np.ndarray):
    """Most-attended key per query over dense bf16 keys K [B][len][H_kv][d]:
    argmax of the fp64 q . k (first index among equal maxima), and the logits."""
    K = bf16_f64(_c(K, np.uint16))
    Qv = bf16_f64(_c(Q, np.uint16))
    B, n, Hkv, d = K.shape
    G = Qv.shape[2] // Hkv
    Kg = np.repeat(K, G, axis=2)                       # [B][len][H_q][d]
    lg = np.einsum("bihd,bthd->biht", Qv, Kg)
    return np.argmax(lg, axis=-1), lg

