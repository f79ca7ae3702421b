"""Shared-memory layout invariants of the split decode kernel, checked on the
host: tests/host/decode_layout_check.cu instantiates the kernel's layout
description for every head dim, query-head group, centroid id width and
quantization group size (32, 64, 128) and asserts 16-byte alignment of every
staged stream and bulk copy, that each field fits its region, that the
final reduction fits in the stages, that the auxiliary k-steps cover the
zero-point and PSAC columns, and the 227 KB shared-memory limit."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.timeout(600)
def test_decode_layout_invariants(tmp_path):
    if not (os.path.exists(NVCC) or shutil.which("nvcc")):
        pytest.skip("nvcc not available")
    exe = str(tmp_path / "decode_layout_check")
    subprocess.run([NVCC, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "bit_kv_cache_centroid_b200", "csrc"),
                    os.path.join(HERE, "host", "decode_layout_check.cu"), "-o", exe], check=True,
                   capture_output=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout[-3000:]
    assert "all layout checks passed" in r.stdout
