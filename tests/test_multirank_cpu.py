"""The N > 1 bench path, on CPU: two gloo ranks on 127.0.0.1.

NSA has no cross-sequence exchange, so multi-GPU runs are independent
replicas (weak scaling); the only collectives are the timing reduction
(max over ranks) and the barrier around the timed region.  These tests run
that host logic with world_size 2 on the gloo backend.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        my_ms = [2.0, 5.0][rank]
        job_ms = bench.max_over_ranks(my_ms, True, device="cpu")
        dist.barrier()
        value = bench.job_tokens_per_s(8192, world, job_ms)
        q.put((rank, job_ms, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_rank_timing_is_max_over_ranks_and_value_sums_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, job_ms, value in res:
        assert job_ms == 5.0  # the slowest rank sets the job time
        assert value == pytest.approx(2 * 8192 / 5e-3)


def test_single_rank_needs_no_collective():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, False) == 3.5
    assert bench.job_tokens_per_s(8192, 1, 0.5) == pytest.approx(8192 / 0.5e-3)


def test_fwd_flops_matches_the_counting_rule():
    """Algorithmic FLOPs at the 340M shape: 4*D per (row, attended key);
    31.29 / 16.64 / 2.13 GFLOP for selection / window / compression."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    f = bench.fwd_flops(bench.WORK)
    assert f["sel"] == 31_289_507_840
    assert f["swa"] == 16_644_046_848
    assert f["cmp"] == 2_131_230_720


def test_reference_arm_line_matches_the_gpu_arm_config(monkeypatch, capsys):
    """The reference arm (the fp64 oracle on the host cores) prints one line
    on rank 0 only, with the GPU arm's config; the oracle timing itself is
    stubbed here (bench's cpu_baseline leg runs it for real)."""
    import argparse
    import json
    import sys
    sys.path.insert(0, ROOT)
    import bench
    calls = []

    def fake(budget_s, seed=0):
        calls.append(budget_s)
        return {"value": 1000.0 + len(calls), "unit": "tokens/s", "cores": 4,
                "kind": "oracle", "sample": "stub"}

    monkeypatch.setattr(bench, "oracle_tokens_per_s", fake)
    args = argparse.Namespace(gpus=2, steps=2, warmup=3)
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == "" and not calls
    bench.run_reference(args, rank=0, world=2)
    line = json.loads(capsys.readouterr().out.strip())
    assert len(calls) == 5 and calls[:3] == [1.0] * 3
    assert line["impl"] == "reference" and line["config"] == bench.workload_config(bench.WORK, 2)
    assert line["value"] == 1004.5 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["value"] == line["value"]
