"""The C-ABI library loads and exports every symbol include/kv2.h declares;
status strings and argument checks that return before touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kv2.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kv2_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from bit_kv_cache_centroid_b200 import build
    return ctypes.CDLL(build.build())


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("kv2_fit_psac_basis", "kv2_quantize_append", "kv2_attention_decode",
                 "kv2_attention_chunk", "kv2_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_exports_match(lib):
    import bit_kv_cache_centroid_b200 as kv2
    assert set(kv2.EXPORTS) == set(declared_functions())
    for name in ("kv2_fit_psac_basis", "kv2_quantize_append", "kv2_attention_decode", "kv2_attention_chunk"):
        assert callable(getattr(kv2, name))


def test_status_strings_and_version(lib):
    lib.kv2_status_string.restype = ctypes.c_char_p
    assert lib.kv2_status_string(0) == b"KV2_OK"
    assert lib.kv2_status_string(3) == b"KV2_ERR_CAPACITY"
    assert lib.kv2_status_string(99) == b"KV2_ERR_UNKNOWN"
    assert lib.kv2_version() >= 100


def test_null_descriptor_is_rejected_before_any_launch(lib):
    lib.kv2_last_error.restype = ctypes.c_char_p
    rc = lib.kv2_quantize_append(None, None, None, 1, 0, 1, None)
    assert rc == 1
    assert b"NULL" in lib.kv2_last_error()
    rc = lib.kv2_attention_decode(None, 0, None, 1, ctypes.c_float(1.0), None, 0, None, 0, None)
    assert rc == 1


def test_unsupported_shapes_are_rejected(lib):
    import bit_kv_cache_centroid_b200 as kv2
    d = kv2.kv2_cache(1, 2, 96, 16, 8, 256, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16)
    assert lib.kv2_quantize_append(ctypes.byref(d), ctypes.c_void_p(16), ctypes.c_void_p(16), 1, 0, 1, None) == 2
    d = kv2.kv2_cache(1, 2, 64, 16, 8, 250, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16)
    assert lib.kv2_quantize_append(ctypes.byref(d), ctypes.c_void_p(16), ctypes.c_void_p(16), 1, 0, 1, None) == 2
    d = kv2.kv2_cache(1, 2, 64, 16, 8, 256, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16)
    # capacity overflow: slots [250, 260) of 256
    assert lib.kv2_quantize_append(ctypes.byref(d), ctypes.c_void_p(16), ctypes.c_void_p(16), 10, 250, 1, None) == 3
    # candidates outside 1..M
    assert lib.kv2_quantize_append(ctypes.byref(d), ctypes.c_void_p(16), ctypes.c_void_p(16), 1, 0, 17, None) == 1
    # misaligned K
    assert lib.kv2_quantize_append(ctypes.byref(d), ctypes.c_void_p(18), ctypes.c_void_p(16), 1, 0, 1, None) == 1
    # chunk needs d = 128
    assert lib.kv2_attention_chunk(ctypes.byref(d), 0, ctypes.c_void_p(16), 2, 4, ctypes.c_void_p(16),
                                   ctypes.c_void_p(16), 4, ctypes.c_float(1.0), ctypes.c_void_p(16), 0,
                                   ctypes.c_void_p(16), 1 << 20, None) == 2


def _desc(**kw):
    """A cache descriptor with fake (never dereferenced) aligned pointers."""
    import bit_kv_cache_centroid_b200 as kv2
    base = dict(B=1, H_kv=2, d=128, M=64, r=8, capacity=256, k_code=0x1000, v_code=0x2000, k_sz=0x3000,
                v_sz=0x4000, cidx=0x5000, psac=0x6000, centroids=0x7000, P=0x8000, w=0x9000, Wg=0xA000,
                psac_fmt=0, psac_scale=0, block_table=0, page_tokens=0, group=0)
    base.update(kw)
    return kv2.kv2_cache(**base)


def test_argument_checks_of_the_later_entry_points(lib):
    """Checks that return before any device work (no GPU needed)."""
    P = ctypes.c_void_p
    lib.kv2_last_error.restype = ctypes.c_char_p
    lib.kv2_fit_centroids_workspace_size.restype = ctypes.c_size_t
    lib.kv2_top1_workspace_size.restype = ctypes.c_size_t
    # workspace sizes: (H*M*d + H*M) 64-bit words; B*nq*H_q*ceil(len/4096) words
    assert lib.kv2_fit_centroids_workspace_size(2, 128, 64) == (2 * 64 * 128 + 2 * 64) * 8
    assert lib.kv2_fit_centroids_workspace_size(2, 96, 64) == 0
    assert lib.kv2_top1_workspace_size(2, 3, 4, 5000) == 2 * 3 * 4 * 2 * 8
    # centre fitting: candidates outside 1..M, unsupported d, a no-op call
    args = lambda C, d, iters: (P(0x1000), 16, 2, d, 64, C, 32, P(0x2000), P(0x3000), iters, P(0x4000),
                                P(0x5000), P(0x6000), ctypes.c_size_t(1 << 20), None)
    assert lib.kv2_fit_centroids(*args(65, 128, 1)) == 1              # KV2_ERR_INVALID_ARG
    assert b"candidates" in lib.kv2_last_error()
    assert lib.kv2_fit_centroids(*args(4, 96, 1)) == 2                # KV2_ERR_UNSUPPORTED
    assert lib.kv2_fit_centroids(*args(4, 128, 0)) == 0               # iters = 0: nothing to do
    # paged cache: a page size that is not a multiple of 128 is refused
    bad = _desc(block_table=0xB000, page_tokens=96)
    top1 = lib.kv2_decode_top1(ctypes.byref(bad), 10, P(0x1000), 1, 2, P(0x2000), P(0x3000),
                               ctypes.c_size_t(1 << 20), None)
    assert top1 == 2 and b"page_tokens" in lib.kv2_last_error()
    # int8 PSAC format without its scale array is refused
    noscale = _desc(psac_fmt=1)
    assert lib.kv2_quantize_append(ctypes.byref(noscale), P(0x1000), P(0x2000), 1, 0, 1, None) == 1
    assert b"psac_scale" in lib.kv2_last_error()


def test_group_argument_checks(lib):
    """Groups of 32, 64 and 128 channels (0 selects 32) pass the checks; other
    sizes, and a group wider than the head, are refused with their reason."""
    P = ctypes.c_void_p
    lib.kv2_last_error.restype = ctypes.c_char_p
    lib.kv2_version.restype = ctypes.c_int
    assert lib.kv2_version() >= 200
    for group, ok in ((0, True), (32, True), (64, True), (128, True), (48, False), (256, False)):
        d = _desc(group=group)
        # capacity overflow is reported only after the descriptor passed its checks
        rc = lib.kv2_quantize_append(ctypes.byref(d), P(0x1000), P(0x2000), 10, 250, 1, None)
        assert rc == (3 if ok else 2), (group, rc)
        if not ok:
            assert b"group" in lib.kv2_last_error()
    d64 = _desc(d=64, group=128)
    assert lib.kv2_quantize_append(ctypes.byref(d64), P(0x1000), P(0x2000), 1, 0, 1, None) == 2
    assert b"larger than d" in lib.kv2_last_error()
    # the statistics entry points take the group as an argument
    fit = lambda group: lib.kv2_fit_psac_basis(P(0x1000), 16, 4, 2, 128, 8, group, P(0x2000), P(0x3000),
                                               P(0x4000), None, P(0x5000), ctypes.c_size_t(16), None)
    assert fit(96) == 2 and b"group" in lib.kv2_last_error()
    assert fit(32) == 6 and fit(64) == 6 and fit(128) == 6                       # past the group check: the workspace is too small
    cent = lambda group: lib.kv2_fit_centroids(P(0x1000), 16, 2, 128, 64, 4, group, P(0x2000), P(0x3000), 1,
                                               P(0x4000), P(0x5000), P(0x6000), ctypes.c_size_t(16), None)
    assert cent(96) == 2 and b"group" in lib.kv2_last_error()
    assert cent(0) == 6


def test_page_image_size_and_argument_checks(lib):
    """A page's host image is H_kv * page_tokens slots of every stream back to
    back; the store/load checks return before any copy is issued."""
    P = ctypes.c_void_p
    lib.kv2_last_error.restype = ctypes.c_char_p
    lib.kv2_page_bytes.restype = ctypes.c_size_t
    paged = dict(block_table=0xB000, page_tokens=128)
    # per token slot: 2 x 8 code words, 2 x 4 scale/zero words, a u8 id, 8 fp16 coefficients
    assert lib.kv2_page_bytes(ctypes.byref(_desc(**paged))) == 2 * 128 * (32 + 32 + 16 + 16 + 1 + 16)
    # int8 coefficients with a per-token fp16 scale; u16 ids; no PSAC
    assert lib.kv2_page_bytes(ctypes.byref(_desc(psac_fmt=1, psac_scale=0xC000, **paged))) == \
        2 * 128 * (32 + 32 + 16 + 16 + 1 + 8 + 2)
    assert lib.kv2_page_bytes(ctypes.byref(_desc(M=512, r=0, **paged))) == 2 * 128 * (32 + 32 + 16 + 16 + 2)
    assert lib.kv2_page_bytes(ctypes.byref(_desc())) == 0                      # not paged
    store = lambda d, page, n, host: lib.kv2_page_store(ctypes.byref(d), page, n, host, None)
    assert store(_desc(), 0, 4, P(0x1000)) == 1 and b"not paged" in lib.kv2_last_error()
    assert store(_desc(**paged), 4, 4, P(0x1000)) == 1 and b"outside" in lib.kv2_last_error()
    assert store(_desc(**paged), -1, 4, P(0x1000)) == 1
    assert store(_desc(**paged), 0, 4, None) == 1 and b"NULL" in lib.kv2_last_error()
    assert lib.kv2_page_load(ctypes.byref(_desc(**paged)), 0, 0, P(0x1000), None) == 1


def test_plain_c_client(lib, tmp_path):
    """The header compiles as pedantic C11 and a C program linked against
    libkv2.so gets the documented results from the host-side checks."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("gcc not available")
    libdir = os.path.join(ROOT, "bit_kv_cache_centroid_b200")
    exe = str(tmp_path / "c_client")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "host", "c_client.c"), "-o", exe, "-L", libdir, "-l:libkv2.so",
                    f"-Wl,-rpath,{libdir}"], check=True, capture_output=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "c client ok" in r.stdout


def test_noalloc_checks_arguments_before_any_device_work(lib):
    """The allocation-free decode validates every argument before it looks up
    its fixed array (which would load the module on the device): on a machine
    without a GPU, bad calls still get their precise argument errors, and the
    error-word accessor refuses a NULL flag."""
    P = ctypes.c_void_p
    lib.kv2_last_error.restype = ctypes.c_char_p
    call = lambda desc, length, Q, H_q, out, dtype: lib.kv2_attention_decode_noalloc(
        ctypes.byref(desc) if desc is not None else None, length, P(Q), H_q, ctypes.c_float(0.1), P(out), dtype, None)
    assert call(None, 16, 0x1000, 2, 0x2000, 0) == 1 and b"NULL" in lib.kv2_last_error()
    assert call(_desc(), 16, 0, 2, 0x2000, 0) == 1 and b"Q / out" in lib.kv2_last_error()
    assert call(_desc(), 16, 0x1008, 2, 0x2000, 0) == 1                     # Q not 16-byte aligned
    assert call(_desc(), 16, 0x1000, 3, 0x2000, 0) == 2                     # H_q not a multiple of H_kv
    assert call(_desc(), 300, 0x1000, 2, 0x2000, 0) == 3                    # len beyond capacity
    assert call(_desc(), 16, 0x1000, 2, 0x2000, 7) == 1                     # out_dtype
    assert call(_desc(group=48), 16, 0x1000, 2, 0x2000, 0) == 2
    big = _desc(B=512, H_kv=64, M=512, r=16, capacity=32)
    assert call(big, 16, 0x1000, 64, 0x2000, 0) == 6 and b"fixed array" in lib.kv2_last_error()
    assert lib.kv2_decode_noalloc_error(None, 0, None) == 1
