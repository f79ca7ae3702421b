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
