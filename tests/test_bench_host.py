"""Host-side checks of bench.py: the multi-rank timing logic on gloo ranks
(CPU, world size 2), and the reference leg (the CPU oracle) end to end."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [5.0, 8.0][rank]  # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        tf = bench.whole_job_tflops(2e12, 10, world, ms)
        out[rank] = (ms, tf)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput_gloo():
    world = 2
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, tf = res[r]
        assert ms == 8.0                         # every rank sees the slowest time
        assert tf == pytest.approx(2e12 * 10 * 2 / 8e-3 / 1e12)  # all ranks' work / max time
    assert bench.max_over_ranks(3.0, 1, None) == 3.0


def test_reference_leg_prints_the_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["warmup"] >= 3  # the contract's minimum is enforced
    # a non-zero rank of a multi-rank launch does no work and prints nothing
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.parametrize("workload,word", [("sweep", "sweep"), ("blockwise", "block-wise")])
def test_quantize_reference_legs_report_gbs(workload, word):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        workload, "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["unit"] == "GB/s" and line["value"] > 0 and word in line["config"]["workload"]


def test_every_workload_is_described_and_sized():
    for name, cfg in bench.WORKLOADS.items():
        d = bench.workload_desc(name, cfg)
        assert isinstance(d, str) and len(d) > 20
        assert cfg["kind"] in ("layer", "decode", "sweep", "stack", "backward", "blockwise", "blockscaled", "blockq", "moe",
                               "moe_bf16")
    # one quantize call's algorithmic bytes: bf16 read + code write + f32 scales
    assert bench.q_bytes(4, 8, 4) == 4 * 8 * 3 + 16


def test_blockscaled_reference_leg_reports_tflops():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "blockscaled", "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert "block-scaled" in line["config"]["workload"] and "block 128" in line["cpu_baseline"]["sample"]
