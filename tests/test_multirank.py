"""Replicas-only multi-rank plumbing of bench.py on CPU ranks (gloo, world size 2).

The layer is not sharded: every rank runs the whole workload and the bench
reports all ranks' work over the slowest rank's time.  These tests run the
same helpers bench.py uses under torchrun, with two gloo ranks on the host.
"""
import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench

    os.environ["RANK"] = str(rank)
    os.environ["WORLD_SIZE"] = str(world)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    dist.barrier()
    local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
    total = bench.max_over_ranks(local_ms, world)
    local_e2e = 3.0 - rank                  # rank 0 is the slow one here
    e2e = bench.max_over_ranks(local_e2e, world)
    value = bench.whole_job_value(world, 2.0e12, 10, total)

    class A:  # arguments of the reference arm
        workload = "tiny_fwd"
        steps = 1
        warmup = 0
        reference_budget = 1.0
    ref = bench.run_reference(A) if rank != 0 else "skipped"
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
        json.dump({"total": total, "e2e": e2e, "value": value, "ref_is_none": ref is None}, f)


def test_two_gloo_ranks_take_the_slowest_time(tmp_path):
    mp = pytest.importorskip("torch.multiprocessing")
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r in res:
        assert r["total"] == 15.0          # max over ranks, identical on every rank
        assert r["e2e"] == 3.0
        # two replicas x 10 steps x 2 TFLOP in 15 ms
        assert r["value"] == pytest.approx(2 * 2.0e12 * 10 / 15e-3 / 1e12)
    assert res[1]["ref_is_none"]           # only rank 0 runs the reference arm


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.whole_job_value(1, 1.0e12, 4, 2.0) == pytest.approx(1.0e12 * 4 / 2e-3 / 1e12)
