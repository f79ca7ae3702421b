"""Thin Python binding of libkv2 (include/kv2.h): argument marshalling only.

Every step of the path runs in the CUDA library; this module passes device
pointers (``tensor.data_ptr()``) and the current CUDA stream. PyTorch is used
for device memory and streams only. If ``libkv2.so`` is missing or fails to
load, importing the binding raises: there is no CPU fallback.

Names follow the C ABI: ``kv2_fit_psac_basis``, ``kv2_fit_centroids``, ``kv2_quantize_append``,
``kv2_attention_decode``, ``kv2_attention_chunk`` and the workspace-size
queries. ``Cache`` owns the device buffers of one packed cache and builds the
``kv2_cache`` descriptor.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkv2.so")

KV2_OK = 0
KV2_OUT_F32 = 0
KV2_OUT_BF16 = 1
GROUP = 32          # default channels per (scale, zero) group
STATUS = {0: "KV2_OK", 1: "KV2_ERR_INVALID_ARG", 2: "KV2_ERR_UNSUPPORTED", 3: "KV2_ERR_CAPACITY",
          4: "KV2_ERR_CUDA", 5: "KV2_ERR_TIMEOUT", 6: "KV2_ERR_WORKSPACE"}


class Kv2Error(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


class kv2_cache(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H_kv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("M", ctypes.c_int32), ("r", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("k_code", ctypes.c_void_p), ("v_code", ctypes.c_void_p),
                ("k_sz", ctypes.c_void_p), ("v_sz", ctypes.c_void_p),
                ("cidx", ctypes.c_void_p), ("psac", ctypes.c_void_p),
                ("centroids", ctypes.c_void_p), ("P", ctypes.c_void_p),
                ("w", ctypes.c_void_p), ("Wg", ctypes.c_void_p),
                ("psac_fmt", ctypes.c_int32), ("psac_scale", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("page_tokens", ctypes.c_int32),
                ("group", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkv2.so not built ({LIB_PATH}); run python -m bit_kv_cache_centroid_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.kv2_status_string.restype = ctypes.c_char_p
    L.kv2_status_string.argtypes = [I]
    L.kv2_last_error.restype = ctypes.c_char_p
    L.kv2_version.restype = I
    L.kv2_fit_workspace_size.restype = S
    L.kv2_fit_workspace_size.argtypes = [I, I]
    L.kv2_fit_psac_basis.restype = I
    L.kv2_fit_psac_basis.argtypes = [P, I, I, I, I, I, I, P, P, P, P, P, S, P]
    L.kv2_fit_centroids_workspace_size.restype = S
    L.kv2_fit_centroids_workspace_size.argtypes = [I, I, I]
    L.kv2_fit_centroids.restype = I
    L.kv2_fit_centroids.argtypes = [P, I, I, I, I, I, I, P, P, I, P, P, P, S, P]
    L.kv2_top1_workspace_size.restype = S
    L.kv2_top1_workspace_size.argtypes = [I, I, I, I]
    L.kv2_decode_top1.restype = I
    L.kv2_decode_top1.argtypes = [P, I, P, I, I, P, P, S, P]
    L.kv2_dense_top1.restype = I
    L.kv2_dense_top1.argtypes = [P, I, I, I, I, P, I, I, P, P, S, P]
    L.kv2_quantize_append.restype = I
    L.kv2_quantize_append.argtypes = [ctypes.POINTER(kv2_cache), P, P, I, I, I, P]
    L.kv2_decode_workspace_size.restype = S
    L.kv2_decode_workspace_size.argtypes = [ctypes.POINTER(kv2_cache), I, I]
    L.kv2_attention_decode.restype = I
    L.kv2_attention_decode.argtypes = [ctypes.POINTER(kv2_cache), I, P, I, ctypes.c_float, P, I, P, S, P]
    L.kv2_attention_decode_noalloc.restype = I
    L.kv2_attention_decode_noalloc.argtypes = [ctypes.POINTER(kv2_cache), I, P, I, ctypes.c_float, P, I, P]
    L.kv2_decode_noalloc_error.restype = I
    L.kv2_decode_noalloc_error.argtypes = [ctypes.POINTER(ctypes.c_int), I, P]
    L.kv2_append_attention_decode.restype = I
    L.kv2_append_attention_decode.argtypes = [ctypes.POINTER(kv2_cache), P, P, I, I, I, P, I, ctypes.c_float, P, I,
                                              P, S, P]
    L.kv2_chunk_workspace_size.restype = S
    L.kv2_chunk_workspace_size.argtypes = [ctypes.POINTER(kv2_cache), I, I]
    L.kv2_attention_chunk.restype = I
    L.kv2_attention_chunk.argtypes = [ctypes.POINTER(kv2_cache), I, P, I, I, P, P, I,
                                      ctypes.c_float, P, I, P, S, P]
    L.kv2_page_bytes.restype = S
    L.kv2_page_bytes.argtypes = [ctypes.POINTER(kv2_cache)]
    L.kv2_page_store.restype = I
    L.kv2_page_store.argtypes = [ctypes.POINTER(kv2_cache), I, I, P, P]
    L.kv2_page_load.restype = I
    L.kv2_page_load.argtypes = [ctypes.POINTER(kv2_cache), I, I, P, P]
    return L


_lib = None


def _get_lib():
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def __getattr__(name):
    # ``lib`` is loaded on first use so that the build step can import this
    # package before libkv2.so exists; any use without the library raises.
    if name == "lib":
        return _get_lib()
    raise AttributeError(name)


EXPORTS = ["kv2_status_string", "kv2_last_error", "kv2_version", "kv2_fit_workspace_size",
           "kv2_fit_psac_basis", "kv2_fit_centroids_workspace_size", "kv2_fit_centroids",
           "kv2_top1_workspace_size", "kv2_decode_top1", "kv2_dense_top1",
           "kv2_quantize_append", "kv2_decode_workspace_size",
           "kv2_attention_decode", "kv2_attention_decode_noalloc", "kv2_decode_noalloc_error",
           "kv2_append_attention_decode",
           "kv2_chunk_workspace_size", "kv2_attention_chunk",
           "kv2_page_bytes", "kv2_page_store", "kv2_page_load"]


def _check(status: int):
    if status != KV2_OK:
        raise Kv2Error(status, _get_lib().kv2_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Cache:
    """Device buffers of one packed cache (layout of include/kv2.h) plus the
    read-only centroid table and fitted statistics it points to."""

    def __init__(self, B, H_kv, d, M, r, capacity, centroids, device="cuda", psac_fmt=0,
                 page_tokens=0, num_pages=0, group=GROUP):
        """page_tokens > 0: a paged cache, its streams a pool of num_pages pages
        of page_tokens tokens; block_table [B][capacity / page_tokens] (int32,
        device) maps each sequence's pages (initially pages in order). group:
        channels per (scale, zero) group."""
        if capacity % 16:
            raise ValueError("capacity must be a multiple of 16")
        if d % group:
            raise ValueError(f"group {group} does not divide d = {d}")
        self.B, self.H_kv, self.d, self.M, self.r, self.capacity = B, H_kv, d, M, r, capacity
        self.group = group
        self.psac_fmt = psac_fmt
        self.page_tokens = page_tokens
        self.num_pages = 0
        if page_tokens:
            pps = capacity // page_tokens
            num_pages = num_pages or B * pps
            self.num_pages = num_pages
            sh = (num_pages, H_kv, page_tokens)
            self.block_table = torch.arange(B * pps, dtype=torch.int32, device=device).remainder(num_pages) \
                .view(B, pps).contiguous()
        else:
            sh = (B, H_kv, capacity)
            self.block_table = None
        u32 = torch.int32
        self.k_code = torch.zeros(sh + (d // 16,), dtype=u32, device=device)
        self.v_code = torch.zeros(sh + (d // 16,), dtype=u32, device=device)
        self.k_sz = torch.zeros(sh + (d // group,), dtype=u32, device=device)
        self.v_sz = torch.zeros(sh + (d // group,), dtype=u32, device=device)
        self.cidx = torch.zeros(sh, dtype=torch.uint8 if M <= 256 else torch.int16, device=device)
        self.psac = torch.zeros(sh + (max(r, 1),), dtype=torch.int8 if psac_fmt == 1 else torch.int16,
                                device=device)
        self.psac_scale = torch.zeros(sh, dtype=torch.int16, device=device) if psac_fmt == 1 else None
        self.centroids = torch.as_tensor(centroids).to(device=device, dtype=torch.int16).contiguous()
        self.P = torch.zeros((H_kv, d, max(r, 1)), dtype=torch.float32, device=device)
        self.w = torch.ones((H_kv, d), dtype=torch.float32, device=device)
        self.Wg = torch.full((H_kv, d // group), float(group), dtype=torch.float32, device=device)
        self.energy = torch.zeros(H_kv, dtype=torch.float32, device=device)

    def desc(self) -> kv2_cache:
        return kv2_cache(self.B, self.H_kv, self.d, self.M, self.r, self.capacity,
                         self.k_code.data_ptr(), self.v_code.data_ptr(), self.k_sz.data_ptr(),
                         self.v_sz.data_ptr(), self.cidx.data_ptr(),
                         self.psac.data_ptr() if self.r else 0, self.centroids.data_ptr(),
                         self.P.data_ptr(), self.w.data_ptr(), self.Wg.data_ptr(), self.psac_fmt,
                         self.psac_scale.data_ptr() if self.psac_scale is not None else 0,
                         self.block_table.data_ptr() if self.block_table is not None else 0,
                         self.page_tokens, self.group)

    def set_fit(self, P, w, Wg):
        if self.r:
            self.P.copy_(torch.as_tensor(P).reshape(self.H_kv, self.d, self.r))
        self.w.copy_(torch.as_tensor(w).reshape(self.H_kv, self.d))
        self.Wg.copy_(torch.as_tensor(Wg).reshape(self.H_kv, self.d // self.group))

    def load_packed(self, pc):
        """Copy a host packed cache (numpy arrays, library layout) in."""
        for name in ("k_code", "v_code", "k_sz", "v_sz"):
            getattr(self, name).copy_(torch.from_numpy(getattr(pc, name).view("int32")))
        self.cidx.copy_(torch.from_numpy(pc.cidx.view("uint8" if self.M <= 256 else "int16")))
        if self.r:
            self.psac.copy_(torch.from_numpy(pc.psac.view("int8" if self.psac_fmt == 1 else "int16")))
            if self.psac_fmt == 1:
                self.psac_scale.copy_(torch.from_numpy(pc.psac_scale.view("int16")))
        if self.block_table is not None and getattr(pc, "table", None) is not None:
            self.block_table.copy_(torch.from_numpy(np.ascontiguousarray(pc.table, dtype=np.int32)))

    def to_host(self):
        """Host numpy copies of the packed streams (library layout)."""
        out = {n: getattr(self, n).cpu().numpy().view("uint32") for n in ("k_code", "v_code", "k_sz", "v_sz")}
        out["cidx"] = self.cidx.cpu().numpy().view("uint8" if self.M <= 256 else "uint16")
        if self.psac_fmt == 1:
            out["psac"] = self.psac.cpu().numpy()[..., :self.r]
            out["psac_scale"] = self.psac_scale.cpu().numpy().view("uint16")
        else:
            out["psac"] = self.psac.cpu().numpy().view("uint16")[..., :self.r]
        return out


# ----------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ----------------------------------------------------------------------------

def kv2_fit_workspace_size(H_kv: int, d: int) -> int:
    return int(_get_lib().kv2_fit_workspace_size(H_kv, d))


def kv2_fit_psac_basis(Qhist: torch.Tensor, H_kv: int, r: int, P=None, w=None, Wg=None,
                       energy=None, ws=None, stream=None, group: int = GROUP):
    """Qhist bf16 [n][H_q][d] (device) -> (P [H_kv][d][r], w [H_kv][d],
    Wg [H_kv][d/group], energy)."""
    n, H_q, d = Qhist.shape
    dev = Qhist.device
    P = torch.empty((H_kv, d, max(r, 1)), dtype=torch.float32, device=dev) if P is None else P
    w = torch.empty((H_kv, d), dtype=torch.float32, device=dev) if w is None else w
    Wg = torch.empty((H_kv, d // group), dtype=torch.float32, device=dev) if Wg is None else Wg
    energy = torch.empty(H_kv, dtype=torch.float32, device=dev) if energy is None else energy
    need = kv2_fit_workspace_size(H_kv, d)
    ws = torch.empty(need, dtype=torch.uint8, device=dev) if ws is None else ws
    _check(_get_lib().kv2_fit_psac_basis(_ptr(Qhist), n, H_q, H_kv, d, r, group, _ptr(P), _ptr(w), _ptr(Wg),
                                  _ptr(energy), _ptr(ws), ws.numel(), _stream(stream)))
    return P[:, :, :r], w, Wg, energy


def kv2_fit_centroids_workspace_size(H_kv: int, d: int, M: int) -> int:
    return int(_get_lib().kv2_fit_centroids_workspace_size(H_kv, d, M))


def kv2_fit_centroids(X: torch.Tensor, centroids: torch.Tensor, candidates: int, w: torch.Tensor,
                      Wg: torch.Tensor, iters: int, assign=None, ws=None, stream=None, group: int = GROUP):
    """X bf16 [n][H_kv][d] sample keys, centroids fp16 [H_kv][M][d] (device;
    updated in place), Wg for groups of ``group`` channels -> (centroids,
    assign int32 [n][H_kv])."""
    n, H_kv, d = X.shape
    M = centroids.shape[1]
    dev = X.device
    assign = torch.empty((max(n, 1), H_kv), dtype=torch.int32, device=dev) if assign is None else assign
    need = kv2_fit_centroids_workspace_size(H_kv, d, M)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev) if ws is None else ws
    _check(_get_lib().kv2_fit_centroids(_ptr(X), n, H_kv, d, M, candidates, group, _ptr(w), _ptr(Wg), iters,
                                        _ptr(centroids), _ptr(assign), _ptr(ws), ws.numel(), _stream(stream)))
    return centroids, assign[:n]


def kv2_top1_workspace_size(B: int, nq: int, H_q: int, length: int) -> int:
    return int(_get_lib().kv2_top1_workspace_size(B, nq, H_q, length))


def kv2_decode_top1(cache: Cache, length: int, Q: torch.Tensor, top1=None, ws=None, stream=None):
    """Q bf16 [B][nq][H_q][d] (or [B][H_q][d]) -> int32 of Q's leading shape:
    the cached token with the largest logit."""
    Q4 = Q if Q.dim() == 4 else Q.unsqueeze(1)
    B, nq, H_q, _ = Q4.shape
    top1 = torch.empty((B, nq, H_q), dtype=torch.int32, device=Q.device) if top1 is None else top1
    need = max(kv2_top1_workspace_size(B, nq, H_q, length), 16)
    ws = torch.empty(need, dtype=torch.uint8, device=Q.device) if ws is None else ws
    d = cache.desc()
    _check(_get_lib().kv2_decode_top1(ctypes.byref(d), length, _ptr(Q4), nq, H_q, _ptr(top1), _ptr(ws),
                                      ws.numel(), _stream(stream)))
    return top1 if Q.dim() == 4 else top1[:, 0]


def kv2_dense_top1(K: torch.Tensor, Q: torch.Tensor, top1=None, ws=None, stream=None):
    """K bf16 [B][len][H_kv][d], Q bf16 [B][nq][H_q][d] (or [B][H_q][d]) ->
    int32: the key with the largest q . k."""
    B, length, H_kv, d = K.shape
    Q4 = Q if Q.dim() == 4 else Q.unsqueeze(1)
    nq, H_q = Q4.shape[1], Q4.shape[2]
    top1 = torch.empty((B, nq, H_q), dtype=torch.int32, device=Q.device) if top1 is None else top1
    need = max(kv2_top1_workspace_size(B, nq, H_q, length), 16)
    ws = torch.empty(need, dtype=torch.uint8, device=Q.device) if ws is None else ws
    _check(_get_lib().kv2_dense_top1(_ptr(K), B, length, H_kv, d, _ptr(Q4), nq, H_q, _ptr(top1), _ptr(ws),
                                     ws.numel(), _stream(stream)))
    return top1 if Q.dim() == 4 else top1[:, 0]


def kv2_quantize_append(cache: Cache, K: torch.Tensor, V: torch.Tensor, pos: int,
                        candidates: int, stream=None):
    """K, V bf16 [B][n_new][H_kv][d] (device) -> written into cache slots [pos, pos+n_new)."""
    d = cache.desc()
    n_new = K.shape[1]
    _check(_get_lib().kv2_quantize_append(ctypes.byref(d), _ptr(K), _ptr(V), n_new, pos, candidates,
                                   _stream(stream)))


def kv2_decode_workspace_size(cache: Cache, H_q: int, length: int) -> int:
    d = cache.desc()
    return int(_get_lib().kv2_decode_workspace_size(ctypes.byref(d), H_q, length))


def kv2_attention_decode(cache: Cache, length: int, Q: torch.Tensor, sm_scale: float,
                         out_dtype: int = KV2_OUT_F32, out=None, ws=None, stream=None):
    """Q bf16 [B][H_q][d] -> out [B][H_q][d] (fp32 or bf16)."""
    B, H_q, dd = Q.shape
    if out is None:
        out = torch.empty((B, H_q, dd), dtype=torch.float32 if out_dtype == KV2_OUT_F32 else torch.bfloat16,
                          device=Q.device)
    if ws is None:
        # zeroed: the first word is the sticky error word of device-side waits
        ws = torch.zeros(max(kv2_decode_workspace_size(cache, H_q, length), 16), dtype=torch.uint8,
                         device=Q.device)
    d = cache.desc()
    _check(_get_lib().kv2_attention_decode(ctypes.byref(d), length, _ptr(Q), H_q, float(sm_scale), _ptr(out),
                                    out_dtype, _ptr(ws), ws.numel(), _stream(stream)))
    return out


def kv2_append_attention_decode(cache: Cache, K_new: torch.Tensor, V_new: torch.Tensor, pos: int, candidates: int,
                                Q: torch.Tensor, sm_scale: float, out_dtype: int = KV2_OUT_F32, out=None, ws=None,
                                stream=None):
    """Append K_new, V_new (bf16 [B][n_new][H_kv][d]) at slot pos, then decode Q over pos + n_new tokens."""
    B, H_q, dd = Q.shape
    n_new = K_new.shape[1]
    if out is None:
        out = torch.empty((B, H_q, dd), dtype=torch.float32 if out_dtype == KV2_OUT_F32 else torch.bfloat16,
                          device=Q.device)
    if ws is None:
        ws = torch.zeros(max(kv2_decode_workspace_size(cache, H_q, pos + n_new), 16), dtype=torch.uint8,
                         device=Q.device)
    d = cache.desc()
    _check(_get_lib().kv2_append_attention_decode(ctypes.byref(d), _ptr(K_new), _ptr(V_new), n_new, pos, candidates,
                                                  _ptr(Q), H_q, float(sm_scale), _ptr(out), out_dtype, _ptr(ws),
                                                  ws.numel(), _stream(stream)))
    return out


def kv2_attention_decode_noalloc(cache: Cache, length: int, Q: torch.Tensor, sm_scale: float,
                                 out_dtype: int = KV2_OUT_F32, out=None, stream=None):
    """Decode attention whose scratch lives in the library's fixed device array
    (no workspace argument; for callers that may not allocate device memory)."""
    B, H_q, dd = Q.shape
    if out is None:
        out = torch.empty((B, H_q, dd), dtype=torch.float32 if out_dtype == KV2_OUT_F32 else torch.bfloat16,
                          device=Q.device)
    d = cache.desc()
    _check(_get_lib().kv2_attention_decode_noalloc(ctypes.byref(d), length, _ptr(Q), H_q, float(sm_scale), _ptr(out),
                                            out_dtype, _stream(stream)))
    return out


def kv2_decode_noalloc_error(clear: bool = False, stream=None) -> int:
    """The error word of the fixed scratch array on the current device (1: a
    decode wait ran out of budget since it was last cleared); zeroes it when
    ``clear``. Waits for ``stream``."""
    flag = ctypes.c_int(0)
    _check(_get_lib().kv2_decode_noalloc_error(ctypes.byref(flag), int(bool(clear)), _stream(stream)))
    return int(flag.value)


def kv2_chunk_workspace_size(cache: Cache, H_q: int, Nq: int) -> int:
    d = cache.desc()
    return int(_get_lib().kv2_chunk_workspace_size(ctypes.byref(d), H_q, Nq))


def kv2_attention_chunk(cache: Cache, length: int, Q: torch.Tensor, Kself: torch.Tensor,
                        Vself: torch.Tensor, frame_tokens: int, sm_scale: float,
                        out_dtype: int = KV2_OUT_F32, out=None, ws=None, stream=None):
    """Q bf16 [B][Nq][H_q][d], Kself/Vself bf16 [B][Nq][H_kv][d] -> out [B][Nq][H_q][d]."""
    B, Nq, H_q, dd = Q.shape
    if out is None:
        out = torch.empty((B, Nq, H_q, dd), dtype=torch.float32 if out_dtype == KV2_OUT_F32 else torch.bfloat16,
                          device=Q.device)
    if ws is None:
        ws = torch.empty(max(kv2_chunk_workspace_size(cache, H_q, Nq), 16), dtype=torch.uint8,
                         device=Q.device)
    d = cache.desc()
    _check(_get_lib().kv2_attention_chunk(ctypes.byref(d), length, _ptr(Q), H_q, Nq, _ptr(Kself), _ptr(Vself),
                                   frame_tokens, float(sm_scale), _ptr(out), out_dtype, _ptr(ws),
                                   ws.numel(), _stream(stream)))
    return out


# ----------------------------------------------------------------------------
# pages of a paged cache out of HBM and back
# ----------------------------------------------------------------------------

def kv2_page_bytes(cache: Cache) -> int:
    """Bytes of one page's host image (0 if the cache is not paged)."""
    d = cache.desc()
    return int(_get_lib().kv2_page_bytes(ctypes.byref(d)))


def kv2_page_store(cache: Cache, page: int, host=None, stream=None):
    """Copy page ``page`` of every stream into ``host`` (a CPU uint8 tensor of
    kv2_page_bytes bytes; page-locked when allocated here) and return it. The
    copies are asynchronous on the stream: synchronize before reading it."""
    if host is None:
        host = torch.empty(kv2_page_bytes(cache), dtype=torch.uint8, pin_memory=True)
    d = cache.desc()
    _check(_get_lib().kv2_page_store(ctypes.byref(d), page, cache.num_pages, ctypes.c_void_p(host.data_ptr()),
                                     _stream(stream)))
    return host


def kv2_page_load(cache: Cache, page: int, host, stream=None):
    """Copy a page image (from kv2_page_store) into page ``page``; the caller
    points block-table entries at it."""
    if host.numel() * host.element_size() < kv2_page_bytes(cache):
        raise ValueError("host buffer smaller than kv2_page_bytes")
    d = cache.desc()
    _check(_get_lib().kv2_page_load(ctypes.byref(d), page, cache.num_pages, ctypes.c_void_p(host.data_ptr()),
                                    _stream(stream)))
