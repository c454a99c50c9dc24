"""The multi-process side of bench.py on CPU: two gloo ranks (the launcher's
environment, 127.0.0.1 rendezvous) take the max of their times and report
the whole-job aggregate; the reference arm does no work on rank 1."""
import argparse
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    pg = bench.init_group("gloo")
    got = bench.max_over_ranks(pg, times[rank], torch.device("cpu"))
    value = bench.aggregate_tflops(world, 1e12, got)
    pg.barrier()
    pg.destroy_process_group()
    q.put((rank, got, value))


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    times = [3.0, 5.0]                 # ms of each rank
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, value in res:
        assert got == 5.0
        assert value == pytest.approx(2 * 1e12 / 5e-3 / 1e12)   # 400 TFLOP/s


def test_single_process_needs_no_group():
    import bench
    assert bench.init_group("gloo") is None or int(os.environ.get("WORLD_SIZE", "1")) > 1
    assert bench.max_over_ranks(None, 2.5, torch.device("cpu")) == 2.5
    assert bench.aggregate_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)


def test_reference_arm_is_rank0_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(workload="tiny", steps=1, warmup=3, cpu_budget=1.0)
    assert bench.bench_reference(args) is None


@pytest.mark.parametrize("which", ["fwd", "bwd"])
def test_reference_arm_runs_the_oracle(which, monkeypatch):
    """Rank 0 of the reference arm times the fp64 oracle (forward, or the
    gradients with --pass bwd) on the host cores and reports the arm's
    metric; no GPU is touched."""
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = argparse.Namespace(workload="tiny", steps=1, warmup=3, cpu_budget=1.0, which=which)
    line = bench.bench_reference(args)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["metric"] == (bench.METRIC_BWD if which == "bwd" else bench.METRIC)
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    factor = 2.5 if which == "bwd" else 1.0
    assert line["config"]["flops_per_step"] == pytest.approx(
        factor * 4.0 * 256 * 256 * 64 / 2.0 * 2)


def test_forward_source_hash_ignores_the_backward():
    """The forward's traffic record stays valid when only backward sources
    change: its hash skips attn_bwd* files and attn_api.cu past the
    backward marker, and the backward's hash does not."""
    import bench
    api = os.path.join(ROOT, "exact_tiled_attention_39_b200", "csrc", "attn_api.cu")
    data = open(api, "rb").read()
    assert data.count(bench.BWD_SECTION_MARK) == 1
    assert bench.kernel_sources_sha256("fwd") != bench.kernel_sources_sha256("bwd")
