"""The benchmark's multi-rank plumbing on CPU: world_size 2 over gloo. Ranks are
replicas (no collective on the data path); the one reduction is the max over
ranks of the timing scalars, and only rank 0 runs the reference arm."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's "time" differs; every rank must see the slowest one
        got = [bench.max_over_ranks(1.5 + rank * 0.25 + i, world, "cpu") for i in range(3)]
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    expect = [1.75 + i for i in range(3)]
    assert out[0] == expect and out[1] == expect


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25


def test_reference_arm_runs_on_rank0_only(capsys):
    class A:
        warmup = 3
        steps = 1
    bench.run_reference(A(), rank=1, world=2)   # a non-zero rank exits without work or output
    assert capsys.readouterr().out == ""


def test_both_arms_report_the_same_config():
    """The headline is the 2-bit batch-64 workload (the largest fp16 configuration);
    both arms name it, and the lines beside it name their own workloads."""
    c = bench.bench_config(1)
    assert c["workload"] == "twobit_b64_ctx8192"
    assert c["encode"]["batch"] == 64 and c["encode"]["bits"] == 2 and c["decode"]["context"] == 8192
    assert bench.bench_config(4)["parallelism"] == "replicas x4"
    names = [sc.name for sc in bench.BESIDE]
    assert names == ["llama3_8b_gqa", "llama7b_layer_encode + decode_b16_ctx8192"]
    g = bench.scenario_config(bench.BESIDE[0], 1)
    assert g["encode"]["layers"] == 32 and g["decode"]["q_heads"] == 32 and g["decode"]["buffer"] == 20
