"""The multi-GPU bench path on CPU: two gloo ranks.  Each rank decodes its own
sequences (weak scaling); the ranks share only the timing barrier and the
maximum of their device times, so that is what is checked here, together
with the per-rank seeds and the whole-job throughput."""
import datetime
import os
import socket
from types import SimpleNamespace

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank reports a different device time; the job's time is the slowest
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        dist.barrier()
        q.put((rank, ms, bench.rank_seed(rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_use_distinct_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    try:
        results = sorted(q.get(timeout=120) for _ in range(2))
    finally:
        for pr in procs:
            pr.join(timeout=60)
            if pr.is_alive():
                pr.kill()
    assert [r for r, _, _ in results] == [0, 1]
    assert all(ms == 15.0 for _, ms, _ in results)
    assert results[0][2] != results[1][2]
    for pr in procs:
        assert pr.exitcode == 0


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25


def test_job_throughput_counts_every_rank_over_the_slowest_time():
    # 2 ranks x 256 sequences x 10 steps in 15 ms
    assert bench.job_tokens_per_s(2, 256, 10, 15.0) == pytest.approx(2 * 256 * 10 / 0.015)
    assert bench.job_tokens_per_s(1, 256, 10, 15.0) * 2 == pytest.approx(bench.job_tokens_per_s(2, 256, 10, 15.0))


def test_reference_arm_does_no_work_off_rank_zero(capsys):
    args = SimpleNamespace(gpus=2, steps=1, warmup=0)
    bench.reference_arm(args, rank=1)
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_the_contract_line_on_rank_zero(capsys):
    """One timed step of the oracle arm (a few seconds of CPU): one JSON line
    with the keys the bench contract asks of the reference arm."""
    import json
    args = SimpleNamespace(gpus=1, steps=1, warmup=0)
    bench.reference_arm(args, rank=0)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True and d["steps"] == 1
    assert d["config"]["workload"] == bench.WORKLOAD
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
