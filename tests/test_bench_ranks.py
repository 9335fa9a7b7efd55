"""The multi-rank host logic of bench.py on CPU: two gloo ranks report different
timed-region lengths; both must see the slowest one, and the whole-job throughput
must count the bytes of every rank over that time (weak scaling, replicas)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        out[rank] = ms
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_and_throughput():
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    # 2 ranks x 100 steps x 1e9 bytes in 50 ms -> 4000 GB/s
    assert bench.job_throughput_gbs(1e9, 100, 2, 50.0) == pytest.approx(4000.0)


def test_bench_scheme_override_parses():
    import bench
    from weight_only_additive_b200 import workloads
    a = bench.parse_args(["--workload", "llama2_7b_layer_set_2x8g8", "--scheme", "3x8g16"])
    w = bench.select_workload(a)
    assert all(l.scheme == workloads.Scheme(3, 8, 16) for l in w.layers)
    assert w.name.endswith("@3x8g16")
    import pytest
    with pytest.raises(SystemExit):
        bench.parse_scheme("3x8")
