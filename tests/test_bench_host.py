"""Host logic of bench.py for N > 1 processes, on the CPU (gloo): the timing
reduction every rank takes (the maximum over ranks), and the reference arm
under torchrun (rank 0 alone runs the oracle and prints one JSON line; the
other ranks exit 0 without work). The path runs replicas only: no collective
carries data."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    got = bench.max_over_ranks(10.0 + 3.5 * rank, device="cpu")
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_timing_is_the_maximum_over_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, 29617, out), nprocs=world, join=True)
    assert out[0] == out[1] == 13.5


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.25, device="cpu") == 4.25


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", "29619", "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--cpu-seconds", "0.5"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "GB/s"
    assert d["config"]["parallelism"] == "replicas x2" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_compression_closed_forms():
    """113 B per token-head on the LLM workload (4.53x against 512 B of bf16
    K+V); its per-head tables (64 fp16 centres, an 8-column fp32 basis, w, W)
    add 21,008 B over 32,769 tokens (4.505x); 128-channel groups with int8
    coefficients: 83 B (6.17x)."""
    sys.path.insert(0, ROOT)
    import bench
    c = bench.compression(128, 8, 64, 32769)
    assert c["bytes_per_token_head"] == 113 and c["ratio"] == 4.531
    tables = 64 * 128 * 2 + 128 * 8 * 4 + 128 * 4 + 4 * 4
    assert tables == 21008
    assert c["ratio_with_tables"] == round(512 / (113 + tables / 32769), 3) == 4.505
    g = bench.compression(128, 8, 256, 37440, psac_fmt=1, group=128)
    assert g["bytes_per_token_head"] == 83 and g["ratio"] == 6.169
    assert bench.compression(128, 16, 512, 187200)["bytes_per_token_head"] == 130
