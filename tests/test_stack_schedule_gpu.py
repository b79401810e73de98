"""The delayed stack step as `bench.py --workload stack` times it: one CUDA
graph per step holding the two GEMMs of step t and, on a second stream beside
the second GEMM, the batched delayed quantize of step t+1 (codes and scales
double-buffered by step parity).  Checked bit for bit against the serial
six-kernel step (`--workload stack_unfused`: quantize X, W_up -> GEMM ->
quantize h -> quantize W_down -> GEMM), itself checked against the oracle in
test_stack_gpu.py: y and the h ring after every step, and the X / W_up /
W_down rings, which the overlapped schedule has already advanced to step t+1,
against the serial rings one step later.  40 steps cross the ring length (16)
and both buffer parities.
"""
import argparse

import pytest
import torch

import bench

pytestmark = pytest.mark.gpu


def _build(name):
    dev = torch.device("cuda", 0)
    peaks, src = bench.load_peaks()
    args = argparse.Namespace(workload=name, steps=10, warmup=3, no_cpu_baseline=True, no_companions=True,
                              impl="ours")
    return bench.build(args, bench.WORKLOADS[name], 0, dev, torch.cuda.current_stream(dev), dict(peaks, _src=src))


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def test_overlapped_stack_schedule_matches_serial_steps():
    over, serial = _build("stack"), _build("stack_unfused")
    step_over, step_serial = over["calls"][0][1], serial["calls"][0][1]
    assert over["calls"][0][2] == 3 and serial["calls"][0][2] == 6
    ahead = None
    for t in range(40):
        step_over()
        step_serial()
        torch.cuda.synchronize()
        assert torch.equal(_bits(over["tensors"]["y"]), _bits(serial["tensors"]["y"])), t
        assert torch.equal(_bits(over["tensors"]["rings"]["h"]), _bits(serial["tensors"]["rings"]["h"])), t
        if ahead is not None:
            for k in ("x", "wu", "wd"):
                assert torch.equal(_bits(ahead[k]), _bits(serial["tensors"]["rings"][k])), (t, k)
        ahead = {k: over["tensors"]["rings"][k].clone() for k in ("x", "wu", "wd")}
    over.pop("graphs", None)
    serial.pop("graphs", None)
