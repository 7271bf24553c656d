"""The N > 1 host logic of bench.py on CPU: two gloo ranks.

The GPU path runs one independent replica per rank; the only collectives
are the barriers around the timed region and the max-over-ranks reduction
of the device times, which these tests exercise with the gloo backend.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = bench.max_over_ranks(local_ms[rank], world, "cpu")
        dist.barrier()
        out[rank] = ms
    finally:
        dist.destroy_process_group()


def _run(world, local_ms):
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, local_ms, out), nprocs=world, join=True)
    return [out[r] for r in range(world)]


def test_max_over_ranks_two_gloo_ranks():
    got = _run(2, [3.25, 7.5])
    assert got == [7.5, 7.5]  # every rank sees the slowest rank's time


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(4.0, 1, "cpu") == 4.0


def test_job_throughput_counts_every_rank():
    # 2 ranks x 8 tokens x 10 steps in 5 ms of the slowest rank
    assert bench.job_tokens_per_s(2, 8, 10, 5.0) == pytest.approx(32000.0)
    assert bench.job_tokens_per_s(1, 8, 10, 5.0) == pytest.approx(16000.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    # ranks other than 0 exit without work and print nothing
    assert bench.run_reference(None, None, 1, rank=1, world=2) is None
    assert capsys.readouterr().out == ""
