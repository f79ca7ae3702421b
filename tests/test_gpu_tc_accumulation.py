"""The quantizer's tensor-core ranking bound assumes that a chain of 16
mma.sync m16n8k16 steps (fp16 operands, fp32 accumulation) errs by at most
kappa = 2^-12 of the summed product magnitudes; no vendor document states
such a bound. This test builds a small standalone program
(tests/tc_accumulation_probe.cu, independent of the library) that runs that
chain on adversarial data and requires the worst measured relative error of
every data law to stay 16x below kappa."""
import json
import os
import shutil
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
KAPPA = 2.0 ** -12


def test_tensor_core_accumulation_within_the_ranking_bound(tmp_path):
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    if not os.path.exists(nvcc):
        nvcc = shutil.which("nvcc")
    assert nvcc, "nvcc is needed to build the probe"
    exe = str(tmp_path / "tc_probe")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe,
                    os.path.join(HERE, "tc_accumulation_probe.cu")], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=300).stdout
    worst = json.loads(out.strip().splitlines()[-1])["worst_rel"]
    assert len(worst) == 4
    for law, w in enumerate(worst):
        assert w < KAPPA / 16, f"data law {law}: worst relative error {w:.3e} vs kappa/16 = {KAPPA / 16:.3e}"
