"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

Tokens are independent, so N GPUs run N replicas of the layer, each on its own
batch, with no collective on the data path; the only cross-rank steps are the
barriers around the timed region and the max-over-ranks of the timings.  These
tests run those steps on two gloo ranks on the CPU.
"""

import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from workloads import CONFIGS, make_tokens


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        cfg = CONFIGS["tiny_fp32"]
        # each rank times a different amount of work; the job time is the slowest rank's
        my_ms = 10.0 + 2.5 * rank
        dist.barrier()
        job_ms = bench.max_over_ranks(my_ms, dist, "cpu")
        dist.barrier()
        tok = make_tokens(cfg, cfg.N, seed=bench.replica_token_seed(rank))
        digest = float(tok.double().sum())
        q.put((rank, job_ms, bench.whole_job_tokens_per_s(cfg.N, world, 7, job_ms), digest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_count_all_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, d0), (r1, ms1, v1, d1) = out
    assert ms0 == ms1 == 12.5                       # max over ranks, on every rank
    assert v0 == v1 == pytest.approx(64 * 2 * 7 / 0.0125)
    assert d0 != d1                                  # replicas draw their own batches


def test_single_rank_helpers_without_a_process_group():
    assert bench.max_over_ranks(3.0, None, "cpu") == 3.0
    assert bench.whole_job_tokens_per_s(32, 1, 100, 50.0) == pytest.approx(64000.0)
    assert bench.replica_token_seed(0) == 0 and bench.replica_token_seed(3) == 1003


def test_reference_arm_prints_nothing_on_other_ranks(capsys, monkeypatch):
    import argparse
    monkeypatch.setenv("RANK", "1")
    ns = argparse.Namespace(impl="reference", workload="tiny_fp32", steps=1, warmup=0, gpus=2,
                            set=[], no_cpu_baseline=True, cpu_seconds=1.0)
    bench.run_reference(ns)
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(capsys, monkeypatch):
    import argparse
    import json
    monkeypatch.setenv("RANK", "0")
    ns = argparse.Namespace(impl="reference", workload="tiny_fp32", steps=2, warmup=1, gpus=1,
                            set=[], no_cpu_baseline=True, cpu_seconds=1.0)
    bench.run_reference(ns)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True
