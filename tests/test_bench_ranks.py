"""The multi-rank arithmetic of bench.py on two CPU ranks over gloo: every timing is the slowest
rank's (max over ranks), the reported value is whole-job throughput (weak scaling), and the
reference arm does its work on rank 0 only."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = load_bench()
        # rank r took 10 + 3r ms for its steps: both ranks must see the slowest, 13 ms
        t = bench.reduce_max(10.0 + 3.0 * rank, torch.device("cpu"), world)
        value = bench.job_gbs(1e9, 4, t, world)
        ref = None
        if rank != 0:  # the reference arm returns at once on every rank but 0
            class A:
                steps, warmup, workload = 1, 0, 5
            ref = bench.run_reference(A, rank, world)
        out[rank] = (t, value, ref)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_count_all_work():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(rank_main, args=(2, free_port(), out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 13.0
    # 2 ranks x 1 GB x 4 steps in 13 ms
    assert res[0][1] == pytest.approx(2 * 1e9 * 4 / 0.013 / 1e9)
    assert res[1][2] is None


def test_single_rank_is_the_identity():
    bench = load_bench()
    assert bench.reduce_max(7.5, torch.device("cpu"), 1) == 7.5
    assert bench.job_gbs(2e9, 10, 1000.0, 1) == pytest.approx(20.0)
