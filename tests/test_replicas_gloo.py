"""The multi-GPU path of bench.py (one independent replica per rank, max-over-ranks timing) on CPU:
two gloo ranks on 127.0.0.1."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    from bit_quantized_mamba_b200 import replicas

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        replicas.barrier(world)
        local_ms = 10.0 * (rank + 1)            # rank 1 is the slower replica
        ms = replicas.max_over_ranks(local_ms, world, torch.device("cpu"))
        rate = replicas.whole_job_rate(64 * 5, world, ms / 1e3)
        replicas.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{ms} {rate}\n")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(world)]
    for ms, rate in got:
        assert float(ms) == 20.0                                # every rank holds the maximum
        assert float(rate) == pytest.approx(2 * 64 * 5 / 0.020)  # work of both ranks / slowest time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    from bit_quantized_mamba_b200 import replicas
    replicas.barrier(1)
    assert replicas.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert replicas.whole_job_rate(640, 1, 0.5) == 1280.0


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)

    class A:
        warmup, steps, gpus = 3, 1, 2

    assert bench.run_reference(A(), rank=1) is None  # returns at once, prints nothing
