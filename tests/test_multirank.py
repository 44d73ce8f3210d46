"""The N > 1 path of bench.py on CPU: two gloo ranks on 127.0.0.1.  The path
runs replicas (no exchange on the data path), so what crosses ranks is only the
timing: every rank's times are replaced by the slowest rank's, and the
whole-job figure counts the bytes all ranks moved in that time."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # rank r: step time 1 + r ms, kernel time 5 - r ms
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank], "cpu")
        out[rank] = (got, bench.whole_job_gbs(world, 2e9, got[0]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_slowest_rank_sets_every_time(world):
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        times, gbs = res[r]
        assert times == [float(world), 5.0]              # max of 1 + r; max of 5 - r
        assert gbs == pytest.approx(world * 2e9 / (world * 1e-3) / 1e9)


def test_single_process_is_identity():
    assert bench.max_over_ranks([0.25, 3.0], "cpu") == [0.25, 3.0]
    assert bench.whole_job_gbs(1, 1e9, 1.0) == pytest.approx(1000.0)


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    """Under torchrun the reference arm runs on rank 0 only."""
    import argparse
    monkeypatch.setenv("RANK", "1")
    ns = argparse.Namespace(gpus=2, steps=1, warmup=3, impl="reference", workload="70b", seed=0,
                            no_cpu_baseline=True, no_e2e=True, math="auto", merge="kernel", num_seqs=0,
                            swap_mb=0, verify_kernel="auto", partition_size=0, profile_all=False, queries=1)
    assert bench.run_reference(ns) == 0
