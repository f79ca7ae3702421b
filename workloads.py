"""Seeded synthetic inputs for the 2-bit KV-cache path (keys, values, queries,
centroid tables and ready-made packed caches).

This module only draws random inputs. It holds none of the quantizer's or the
attention's arithmetic, so that the CUDA path and the CPU oracle can both take
their inputs from it without sharing any of the method. Sixteen-bit floats are
returned as ``uint16`` bit patterns: bf16 for keys, values and queries, fp16 for
centroid tables and for the fp16 fields of a packed cache.

The five workloads follow the shapes of the QuantWM pages (QuantWM: Training-Free
2-bit KV Cache Quantization for Stable Video World Models — opening section on
KV-cache growth, "Experimental Validation" for 480p / 93-frame generation, and
"2. Principal Subspace Attention Compensation" for the ~71% Query energy in the
top-8 directions):

* ``tiny``         1 x 2 heads, d=64, 256 cached tokens, M=16, C=4, r=8.
* ``llm_decode``   batch 8, 32 query / 8 KV heads, d=128, 32,768 cached tokens.
* ``video_chunk``  40 heads, 24 latent frames x 1,560 tokens cached, 3-frame chunk.
* ``quant_append`` 4,680 new tokens x 40 heads appended at 37,440, M=256, C=8.
* ``long_horizon`` 120 latent frames x 1,560 = 187,200 tokens, M=512, r=16.

Centroid tables are an input of the quantizer; they are fitted here with a plain
seeded Lloyd k-means (unweighted L2) on a sample of the workload's keys.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np

GROUP = 32            # default channels per quantization group (32, 64 or 128)
GRID = (30, 52)       # latent tokens per 480p frame: 480/16 x 832/16
FRAME_TOKENS = GRID[0] * GRID[1]


@dataclass(frozen=True)
class Spec:
    name: str
    seed: int
    B: int
    H_q: int
    H_kv: int
    d: int
    M: int            # centroids per KV head
    C: int            # QSAC candidates
    r: int            # PSAC rank
    T: int            # cached tokens per (batch, KV head)
    n_new: int        # tokens appended by one quantize call
    capacity: int     # cache capacity in tokens per (batch, KV head)
    n_hist: int       # history (calibration) query tokens per query head
    Nq: int           # queries of one chunk-attention call (0: decode only)
    frame_tokens: int  # tokens per latent frame (chunk mask)
    key_law: str      # "gaussian" | "video" | "long"
    top_energy: float  # share of Query energy in the top-8 directions
    group: int = GROUP  # channels per (scale, zero) group of the packed cache

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    def with_(self, **kw) -> "Spec":
        s = dataclasses.replace(self, **kw)
        if "capacity" not in kw:
            s = dataclasses.replace(s, capacity=max(s.capacity, s.T + s.n_new))
        return s


SPECS = {
    "tiny": Spec("tiny", 0, B=1, H_q=2, H_kv=2, d=64, M=16, C=4, r=8, T=256,
                 n_new=256, capacity=256, n_hist=64, Nq=64, frame_tokens=32,
                 key_law="gaussian", top_energy=0.70),
    "llm_decode": Spec("llm_decode", 1, B=8, H_q=32, H_kv=8, d=128, M=64, C=4,
                       r=8, T=32768, n_new=1, capacity=32768 + 256, n_hist=128,
                       Nq=0, frame_tokens=1, key_law="gaussian",
                       top_energy=0.70),
    "video_chunk": Spec("video_chunk", 2, B=1, H_q=40, H_kv=40, d=128, M=256,
                        C=8, r=8, T=24 * FRAME_TOKENS, n_new=3 * FRAME_TOKENS,
                        capacity=27 * FRAME_TOKENS, n_hist=512,
                        Nq=3 * FRAME_TOKENS, frame_tokens=FRAME_TOKENS,
                        key_law="video", top_energy=0.71),
    "quant_append": Spec("quant_append", 3, B=1, H_q=40, H_kv=40, d=128, M=256,
                         C=8, r=8, T=24 * FRAME_TOKENS, n_new=3 * FRAME_TOKENS,
                         capacity=27 * FRAME_TOKENS, n_hist=512, Nq=0,
                         frame_tokens=FRAME_TOKENS, key_law="video",
                         top_energy=0.71),
    "long_horizon": Spec("long_horizon", 4, B=1, H_q=40, H_kv=40, d=128, M=512,
                         C=8, r=16, T=120 * FRAME_TOKENS,
                         n_new=3 * FRAME_TOKENS, capacity=123 * FRAME_TOKENS,
                         n_hist=512, Nq=3 * FRAME_TOKENS,
                         frame_tokens=FRAME_TOKENS, key_law="long",
                         top_energy=0.71),
}


def spec(name: str, **overrides) -> Spec:
    s = SPECS[name]
    return s.with_(**overrides) if overrides else s


# ----------------------------------------------------------------------------
# 16-bit encodings of the generated fp32 draws (input preparation only)
# ----------------------------------------------------------------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round-to-nearest-even (torch's CPU cast)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f16_bits(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def f16_values(bits: np.ndarray) -> np.ndarray:
    return bits.view(np.float16).astype(np.float32)


# ----------------------------------------------------------------------------
# random fields
# ----------------------------------------------------------------------------

def _orthonormal(rng: np.random.Generator, d: int) -> np.ndarray:
    a = rng.standard_normal((d, d))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def query_spectrum(d: int, top_energy: float, k: int = 8) -> np.ndarray:
    """Per-direction variances: the top k directions hold ``top_energy`` of the
    expected energy (graded, so the directions are distinct), the other d-k the
    rest; the total expected energy is d (unit variance per channel on average)."""
    top = 0.8 ** np.arange(k)
    rest = 0.97 ** np.arange(d - k)
    return np.concatenate([top / top.sum() * top_energy * d,
                           rest / rest.sum() * (1.0 - top_energy) * d])


def query_bases(s: Spec, rng: np.random.Generator) -> np.ndarray:
    """One orthonormal basis per KV head, shared by its group of query heads."""
    return np.stack([_orthonormal(rng, s.d) for _ in range(s.H_kv)])


def draw_queries(s: Spec, rng: np.random.Generator, n: int,
                 U: np.ndarray, batch: int = 1) -> np.ndarray:
    """fp32 queries [batch][n][H_q][d], q = U diag(sigma) z."""
    sig = np.sqrt(query_spectrum(s.d, s.top_energy))
    z = rng.standard_normal((batch, n, s.H_q, s.d)).astype(np.float32)
    z *= sig[None, None, None, :].astype(np.float32)
    out = np.empty_like(z)
    for hq in range(s.H_q):
        out[:, :, hq, :] = z[:, :, hq, :] @ U[hq // s.G].T.astype(np.float32)
    return out


def channel_scales(s: Spec, rng: np.random.Generator) -> np.ndarray:
    """Per (KV head, channel) log-normal scales (sigma=1) with 4 outlier
    channels per head multiplied by 8."""
    sc = np.exp(rng.standard_normal((s.H_kv, s.d)))
    for h in range(s.H_kv):
        sc[h, rng.choice(s.d, 4, replace=False)] *= 8.0
    return sc.astype(np.float32)


def grf(rng: np.random.Generator, n: int, grid=GRID, sigma: float = 4.0) -> np.ndarray:
    """n unit-variance Gaussian random fields on a (periodic) token grid: white
    noise convolved with a Gaussian of std ``sigma`` tokens. Returns [n][H*W]."""
    h, w = grid
    noise = rng.standard_normal((n, h, w))
    fy = np.fft.fftfreq(h)[:, None]
    fx = np.fft.fftfreq(w)[None, :]
    kern = np.exp(-2.0 * (np.pi * sigma) ** 2 * (fy ** 2 + fx ** 2))
    f = np.fft.ifft2(np.fft.fft2(noise) * kern).real
    f /= f.std(axis=(1, 2), keepdims=True) + 1e-12
    return f.reshape(n, h * w).astype(np.float32)


def video_frames(s: Spec, rng: np.random.Generator, frames, head: int,
                 scales: np.ndarray | None):
    """Keys (scales given) or values (scales None) of one head for the listed
    latent frames: base field + 0.05*f*drift + 0.3*per-frame noise, all GRFs
    with correlation length 4 tokens. Returns [len(frames)][1560][d] fp32."""
    d = s.d
    base = grf(rng, d).T          # [1560][d]
    drift = grf(rng, d).T
    out = []
    for f in frames:
        noise = grf(rng, d).T
        x = base + 0.05 * f * drift + 0.3 * noise
        out.append(x if scales is None else x * scales[None, :])
    return np.stack(out).astype(np.float32)


def long_frames(s: Spec, rng: np.random.Generator, frames, head: int,
                scales: np.ndarray | None):
    """Long-horizon keys/values of one head: frame f views a wider base canvas
    shifted by floor(0.25 f) tokens horizontally (slow camera drift) plus 0.3
    frame noise; frames 30, 60, 90 are frame 0 plus 0.1 noise (revisits)."""
    d = s.d
    gh, gw = GRID
    wide = (gh, gw + 32)
    canvas = grf(rng, d, grid=wide).reshape(d, gh, gw + 32)
    f0_noise = grf(rng, d).T
    out = []
    for f in frames:
        if f > 0 and f % 30 == 0:
            view = canvas[:, :, 0:gw].reshape(d, -1).T
            x = view + 0.3 * f0_noise + 0.1 * grf(rng, d).T
        else:
            sh = int(np.floor(0.25 * f)) % 32
            view = canvas[:, :, sh:sh + gw].reshape(d, -1).T
            x = view + 0.3 * (f0_noise if f == 0 else grf(rng, d).T)
        out.append(x if scales is None else x * scales[None, :])
    return np.stack(out).astype(np.float32)


def kmeans_centroids(x: np.ndarray, M: int, rng: np.random.Generator,
                     iters: int = 10) -> np.ndarray:
    """Plain Lloyd k-means (fp64, unweighted L2), initialised from M distinct
    sampled points; an empty cluster keeps its previous centre. Returns the
    centres as fp16 bit patterns [M][d]."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[0]
    c = x[rng.choice(n, M, replace=n < M)].copy()
    x2 = (x * x).sum(1)
    for _ in range(iters):
        dist = x2[:, None] - 2.0 * x @ c.T + (c * c).sum(1)[None, :]
        a = dist.argmin(1)
        cnt = np.bincount(a, minlength=M)
        sums = np.zeros_like(c)
        np.add.at(sums, a, x)
        nz = cnt > 0
        c[nz] = sums[nz] / cnt[nz, None]
    return f16_bits(np.clip(c, -65000, 65000))


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    spec: Spec
    K: np.ndarray          # bf16 bits [B][T + n_new][H_kv][d]: cached prefix then new tokens
    V: np.ndarray          # bf16 bits, same shape
    Qhist: np.ndarray      # bf16 bits [n_hist][H_q][d] (history / calibration queries)
    Qdec: np.ndarray       # bf16 bits [B][H_q][d] (one decode query per sequence)
    Qchunk: np.ndarray | None   # bf16 bits [B][Nq][H_q][d]
    centroids: np.ndarray  # fp16 bits [H_kv][M][d]

    @property
    def K_new(self):
        return self.K[:, self.spec.T:]

    @property
    def V_new(self):
        return self.V[:, self.spec.T:]


def _keys_values(s: Spec, rng, n_tok: int):
    sc = channel_scales(s, rng)
    if s.key_law == "gaussian":
        z = rng.standard_normal((s.B, n_tok, s.H_kv, s.d), dtype=np.float32)
        K = z * sc[None, None, :, :]
        V = rng.standard_normal((s.B, n_tok, s.H_kv, s.d), dtype=np.float32)
        return K, V
    law = video_frames if s.key_law == "video" else long_frames
    nf = -(-n_tok // s.frame_tokens)
    K = np.empty((s.B, nf * s.frame_tokens, s.H_kv, s.d), np.float32)
    V = np.empty_like(K)
    grid_tokens = FRAME_TOKENS
    for b in range(s.B):
        for h in range(s.H_kv):
            kf = law(s, rng, range(nf), h, sc[h])      # [nf][1560][d]
            vf = law(s, rng, range(nf), h, None)
            # frames of fewer tokens than a 30x52 grid take the first tokens
            K[b, :, h] = kf[:, :s.frame_tokens].reshape(-1, s.d) if s.frame_tokens <= grid_tokens \
                else np.resize(kf, (nf * s.frame_tokens, s.d))
            V[b, :, h] = vf[:, :s.frame_tokens].reshape(-1, s.d) if s.frame_tokens <= grid_tokens \
                else np.resize(vf, (nf * s.frame_tokens, s.d))
    return K[:, :n_tok], V[:, :n_tok]


def make(name: str, seed: int | None = None, *, with_chunk: bool = True,
         kmeans_sample: int = 8192, **overrides) -> Workload:
    """Draw a whole workload: cached prefix + new keys/values, history queries,
    decode queries, chunk queries and fitted centroid tables."""
    s = spec(name, **overrides)
    if seed is not None:
        s = s.with_(seed=seed)
    rng = np.random.default_rng(s.seed)
    U = query_bases(s, rng)
    K, V = _keys_values(s, rng, s.T + s.n_new)
    Qhist = draw_queries(s, rng, s.n_hist, U)[0]
    Qdec = draw_queries(s, rng, 1, U, batch=s.B)[:, 0]
    Qc = draw_queries(s, rng, s.Nq, U, batch=s.B) if (with_chunk and s.Nq) else None
    cents = np.empty((s.H_kv, s.M, s.d), np.uint16)
    for h in range(s.H_kv):
        keys = K[:, :max(s.T, 1), h].reshape(-1, s.d)
        if keys.shape[0] > kmeans_sample:
            keys = keys[rng.choice(keys.shape[0], kmeans_sample, replace=False)]
        kb = bf16_values(bf16_bits(keys))
        cents[h] = kmeans_centroids(kb, s.M, rng)
    return Workload(s, bf16_bits(K), bf16_bits(V), bf16_bits(Qhist),
                    bf16_bits(Qdec), None if Qc is None else bf16_bits(Qc), cents)


# ----------------------------------------------------------------------------
# ready-made packed caches (random bit patterns in the packed format)
# ----------------------------------------------------------------------------

@dataclass
class PackedCache:
    """Host copy of a packed cache, in the library's layout:
    k_code/v_code u32 [B][H_kv][cap][d/16], k_sz/v_sz u32
    [B][H_kv][cap][d/group] (low half fp16 scale, high half fp16 zero of each
    group of `group` consecutive channels), cidx u8/u16 [B][H_kv][cap],
    psac fp16 bits [B][H_kv][cap][r] (format 0) or int8 codes [B][H_kv][cap][r]
    with fp16 scale bits psac_scale [B][H_kv][cap] (format 1), centroids fp16
    bits [H_kv][M][d]."""
    B: int
    H_kv: int
    d: int
    M: int
    r: int
    capacity: int
    k_code: np.ndarray
    v_code: np.ndarray
    k_sz: np.ndarray
    v_sz: np.ndarray
    cidx: np.ndarray
    psac: np.ndarray
    centroids: np.ndarray
    psac_fmt: int = 0
    psac_scale: np.ndarray | None = None
    table: np.ndarray | None = None    # paged: page ids [B][capacity / page]
    page: int = 0                       # tokens per page (paged)
    group: int = GROUP                  # channels per (scale, zero) group

    @staticmethod
    def empty(B, H_kv, d, M, r, capacity, centroids, psac_fmt: int = 0, group: int = GROUP):
        cap = (capacity + 15) // 16 * 16          # the library wants capacity % 16 == 0
        assert d % group == 0
        return PackedCache(
            B, H_kv, d, M, r, cap,
            np.zeros((B, H_kv, cap, d // 16), np.uint32),
            np.zeros((B, H_kv, cap, d // 16), np.uint32),
            np.zeros((B, H_kv, cap, d // group), np.uint32),
            np.zeros((B, H_kv, cap, d // group), np.uint32),
            np.zeros((B, H_kv, cap), np.uint8 if M <= 256 else np.uint16),
            np.zeros((B, H_kv, cap, max(r, 1)), np.int8 if psac_fmt == 1 else np.uint16),
            centroids, psac_fmt,
            np.zeros((B, H_kv, cap), np.uint16) if psac_fmt == 1 else None, group=group)


def to_paged(pc: PackedCache, page: int, n_pages: int, seed: int = 0) -> PackedCache:
    """The same packed cache stored as a pool of n_pages pages of `page`
    tokens (streams [n_pages][H_kv][page][...]) in a seeded random order,
    addressed through a block table [B][capacity / page]; pages not in the
    table hold random bytes."""
    assert pc.capacity % page == 0
    pps = pc.capacity // page
    assert n_pages >= pc.B * pps
    rng = np.random.default_rng(seed)
    table = rng.permutation(n_pages)[:pc.B * pps].astype(np.int32).reshape(pc.B, pps)

    def pool(a):
        if a is None:
            return None
        out = rng.integers(0, 255, (n_pages, pc.H_kv, page) + a.shape[3:]).astype(a.dtype)
        for b in range(pc.B):
            for i in range(pps):
                out[table[b, i]] = a[b, :, i * page:(i + 1) * page]
        return out
    return PackedCache(pc.B, pc.H_kv, pc.d, pc.M, pc.r, pc.capacity, pool(pc.k_code), pool(pc.v_code),
                       pool(pc.k_sz), pool(pc.v_sz), pool(pc.cidx), pool(pc.psac), pc.centroids,
                       pc.psac_fmt, pool(pc.psac_scale), table, page, pc.group)


def random_packed_cache(s: Spec, T: int | None = None, seed: int | None = None,
                        centroids: np.ndarray | None = None,
                        revisit_every: int = 0, psac_fmt: int = 0) -> PackedCache:
    """A packed cache of T tokens filled with seeded random fields shaped like
    quantizer output: every u32 code word uniform (so each 2-bit code is
    uniform on 0..3), per-group fp16 scales log-normal around the spread of a
    unit-variance residual, zeros near -1.5 scale, centroid ids uniform, PSAC
    coefficients ~ N(0, (0.05 scale)^2) (format 1: int8 codes uniform on
    -127..127 with fp16 per-token scales of 0.15 scale / 127). With
    ``revisit_every`` = n > 0 the
    tokens of frame n, 2n, ... repeat frame 0 with 10% of code words redrawn,
    so that retrieval targets recur (long-horizon workload)."""
    T = s.T if T is None else T
    rng = np.random.default_rng((s.seed if seed is None else seed) + 1000)
    cap = (max(s.capacity, T) + 15) // 16 * 16
    if centroids is None:
        centroids = f16_bits(rng.standard_normal((s.H_kv, s.M, s.d)).astype(np.float32))
    pc = PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, cap, centroids, psac_fmt, s.group)
    sh = (s.B, s.H_kv, T)
    ng = s.d // s.group
    pc.k_code[:, :, :T] = rng.integers(0, 2 ** 32, sh + (s.d // 16,), dtype=np.uint32)
    pc.v_code[:, :, :T] = rng.integers(0, 2 ** 32, sh + (s.d // 16,), dtype=np.uint32)
    for arr, typical in ((pc.k_sz, 0.6), (pc.v_sz, 1.4)):
        sc = typical * np.exp(0.35 * rng.standard_normal(sh + (ng,)))
        ze = -1.5 * sc * (1.0 + 0.1 * rng.standard_normal(sh + (ng,)))
        arr[:, :, :T] = f16_bits(sc).astype(np.uint32) | (f16_bits(ze).astype(np.uint32) << 16)
    pc.cidx[:, :, :T] = rng.integers(0, s.M, sh).astype(pc.cidx.dtype)
    if s.r:
        sc = f16_values((pc.k_sz[:, :, :T] & 0xFFFF).astype(np.uint16)).mean(-1, keepdims=True)
        if psac_fmt == 1:
            pc.psac[:, :, :T] = rng.integers(-127, 128, sh + (s.r,)).astype(np.int8)
            pc.psac_scale[:, :, :T] = f16_bits(0.15 * sc[..., 0] / 127.0)
        else:
            pc.psac[:, :, :T] = f16_bits(0.05 * sc * rng.standard_normal(sh + (s.r,)))
    if revisit_every and s.frame_tokens > 1:
        F = s.frame_tokens
        for f in range(revisit_every, T // F, revisit_every):
            dst = slice(f * F, (f + 1) * F)
            for arr in (pc.k_code, pc.v_code, pc.k_sz, pc.v_sz, pc.cidx, pc.psac, pc.psac_scale):
                if arr is not None:
                    arr[:, :, dst] = arr[:, :, 0:F]
            redraw = rng.random((s.B, s.H_kv, F)) < 0.1
            fresh = rng.integers(0, 2 ** 32, (s.B, s.H_kv, F, s.d // 16), dtype=np.uint32)
            pc.k_code[:, :, dst] = np.where(redraw[..., None], fresh, pc.k_code[:, :, dst])
    return pc
