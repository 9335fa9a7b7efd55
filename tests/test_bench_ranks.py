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


def test_reference_arm_names_the_same_config():
    """Both arms' lines carry line_config's object: for a given L2 size the reference
    arm's config equals what the library's arm prints for the same arguments."""
    for argv in ([], ["--launch", "per-layer", "--schedule", "streamk"], ["--pool", "3"],
                 ["--workload", "llama2_7b_layer_set_2x8g8", "--batch", "4"]):
        a = bench.parse_args(argv)
        w = bench.select_workload(a)
        batch = bench.workload_batch(w, a.batch)
        ref = bench.reference_config(a, w, batch, 2)
        pool = bench.pool_copies(bench.step_bytes(w, batch), bench.L2_FALLBACK, a.pool)
        assert ref == bench.line_config(w, batch, 2, a.launch, a.schedule, pool, bench.L2_FALLBACK)
        assert ref["workload"] == w.name and ref["batch"] == batch and ref["parallelism"] == "replicas x2"
        assert f"pool of {pool} copies" in ref["l2"] and f"graphs of {pool} consecutive" in ref["launch"]


def test_pool_rule():
    l2 = 126 << 20
    assert bench.pool_copies(354e6, l2) == 8            # 8 copies already exceed 3x L2
    assert bench.pool_copies(5e6, l2) == 80            # ceil(3 L2 / 5 MB)
    assert bench.pool_copies(20e9, l2) == 3            # capped at 60 GB
    assert bench.pool_copies(5e6, l2, copies=3) == 3


def test_reference_arm_names_the_same_config_for_the_input_gradient():
    a = bench.parse_args(["--op", "input-grad", "--workload", "llama2_7b_layer_set_2x8g8", "--batch", "64"])
    w = bench.select_workload(a)
    ref = bench.reference_config(a, w, 64, 1)
    pool = bench.grad_pool_copies(bench.grad_step_bytes(w, 64), bench.L2_FALLBACK, a.pool)
    assert ref == bench.grad_line_config(w, 64, 1, a.schedule, pool, bench.L2_FALLBACK)
    assert ref["op"] == "input-grad" and ref["flops_per_step"] == sum(2.0 * 64 * l.N * l.K for l in w.layers)


def test_roofline_record_names_the_bound_and_the_gather_traffic():
    from weight_only_additive_b200 import workloads
    peaks = {"hbm_gbs": 6451.2, "tc_tflops": 1650.0, "source": "measured"}
    w = workloads.get("single_4096x4096_1x16g8")
    rec = bench.roofline_record(w, 1, 14.6e-6, peaks, 148, 1965.0)
    assert rec["bound"] == "l1tex_gather" and set(rec["roofs"]) >= {"hbm", "l1tex_gather"}
    gathers = 4096 * 512  # one codeword per 8 weights of 4096 x 4096
    assert rec["roofs"]["l1tex_gather"]["achieved"] == pytest.approx(gathers / 1e9 / 14.6e-6)
    l2 = rec["l2_gather_sectors"]
    assert l2["sectors"] == gathers and l2["bytes"] == 32 * gathers
    assert l2["per_hbm_byte"] == pytest.approx(32 * gathers / bench.step_bytes(w, 1))
    # a 2x8 workload: HBM-bound at batch 1, no gathers from L2
    w2 = workloads.get("llama2_7b_layer_set_2x8g8")
    rec2 = bench.roofline_record(w2, 1, 18e-6, peaks, 148, 1965.0)
    assert rec2["bound"] == "hbm" and "l2_gather_sectors" not in rec2
    assert rec2["frac"] == pytest.approx(bench.step_bytes(w2, 1) / 18e-6 / 1e9 / 6451.2)


def test_reference_arm_prints_one_complete_line(monkeypatch, capsys):
    """`bench.py --impl reference` end to end on the CPU, with the oracle's timing
    replaced by fixed numbers: one JSON line with the contract's keys, its config
    equal to the library arm's for the same arguments."""
    import json

    calls = []

    def fake_sample(w, batch, seconds, copy=0, nthreads=0):
        calls.append(seconds)
        return 2e6, 0.5, 7, 4          # bytes credited, seconds, rows per layer, threads

    def fake_grad(w, batch, seconds, seed=5):
        calls.append(seconds)
        return 3e9, 0.25, 16, 4        # flops credited, seconds, columns per layer, threads

    monkeypatch.setattr(bench, "oracle_sample_run", fake_sample)
    monkeypatch.setattr(bench, "oracle_grad_sample_run", fake_grad)
    for argv, unit, value in ((["--impl", "reference", "--steps", "4", "--warmup", "3"], "GB/s", 2e6 / 0.5 / 1e9),
                              (["--impl", "reference", "--op", "input-grad", "--workload",
                                "llama2_7b_layer_set_2x8g8", "--steps", "4", "--warmup", "3"],
                               "TFLOP/s", 3e9 / 0.25 / 1e12)):
        calls.clear()
        assert bench.main(argv) == 0
        line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
        assert len(calls) == 7                                   # warm-up + timed steps
        assert line["impl"] == "reference" and line["unit"] == unit and line["steps"] == 4
        assert line["value"] == pytest.approx(value) and line["e2e"]["value"] == line["value"]
        assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
        assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 4
        a = bench.parse_args(argv)
        w = bench.select_workload(a)
        batch = line["config"]["batch"]
        assert line["config"] == bench.reference_config(a, w, batch, 1)
        for key in ("metric", "n_gpus", "warmup", "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                    "dtype", "data"):
            assert key in line, key


def test_cpu_kernel_leg_reports_its_method():
    """The `cpu_kernel` record of the library's arm, on a short budget: positive
    throughput over whole layers, and the method the CPU library runs at its level."""
    from weight_only_additive_b200 import cpu, workloads
    for name, batch in (("single_4096x4096_1x16g8", 1), ("llama2_7b_layer_set_2x8g8", 1)):
        w = workloads.BY_NAME[name]
        rec = bench.cpu_kernel_run(w, batch, 0.2)
        assert rec["value"] > 0 and rec["unit"] == "GB/s" and rec["simd"] == cpu.SIMD_NAMES[cpu.simd_level()]
        level, B = cpu.simd_level(), w.layers[0].scheme.B
        if B == 8:
            assert "lookup tables" in rec["sample"]
        else:
            assert ("fused decode" if level == 2 else "decode to fp32") in rec["sample"]
