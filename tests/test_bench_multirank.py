"""The multi-replica logic of bench.py on 2 gloo ranks (CPU): barrier, the max over ranks of
the timed region, and the whole-job throughput (every rank's tokens over the slowest time)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        local_ms = 100.0 + 25.0 * rank          # rank 1 is the slower replica
        total = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.job_throughput(4096, world, 10, total)
        out[rank] = (total, value)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_replicas_agree_on_the_slowest_time_and_job_throughput():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0] == res[1]
    total, value = res[0]
    assert total == 125.0
    assert value == pytest.approx(4096 * 2 * 10 / 0.125)


def test_single_process_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    bench.barrier(1)
    assert bench.job_throughput(4096, 1, 100, 250.0) == pytest.approx(4096 * 100 / 0.25)


def test_reference_arm_runs_on_rank_zero_only():
    class A:
        steps, warmup, workload, tokens, ref_budget = 1, 3, "mixtral", 0, 1.0
    assert bench.run_reference(A(), rank=1, world=2) is None     # returns without work


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    # a small Mixtral-shaped layer so that the fp64 oracle steps take well under a second
    import json
    from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, scaled
    small = scaled(WORKLOADS["mixtral"], T=64, D=128, F=128)
    monkeypatch.setattr(bench, "workload_of", lambda args: small)

    class A:
        steps, warmup, workload, tokens, ref_budget = 2, 3, "mixtral", 0, 0.5
    bench.run_reference(A(), rank=0, world=1)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    assert r["impl"] == "reference" and r["metric"] == bench.METRIC
    assert r["unit"] == "tokens/s" and r["higher_is_better"] is True
    assert r["steps"] == 2 and r["warmup"] == 3 and r["n_gpus"] == 1
    assert r["value"] > 0 and r["dtype"] == "f64"
    assert r["config"]["workload"] == small.name and "model" not in r["config"]
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["value"] == r["value"]
    assert r["cpu_baseline"]["cores"] >= 1 and r["cpu_baseline"]["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_traffic_is_null_for_shapes_other_than_the_captured_one():
    import argparse
    from sparse_mixture_experts_warp_b200.workloads import WORKLOADS
    full = bench.workload_of(argparse.Namespace(workload="mixtral", tokens=0, ffn=0))
    assert full == WORKLOADS["mixtral"]
    for tokens, ffn in ((1024, 0), (0, 3584)):
        w = bench.workload_of(argparse.Namespace(workload="mixtral", tokens=tokens, ffn=ffn))
        assert w != full and bench.load_traffic("mixtral", w) is None
