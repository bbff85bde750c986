"""Host plumbing of `bench.py --gpus N`: the linear shards along tokens with no exchange,
so N ranks run independent replicas; their per-rank times are reduced with MAX and the
job's throughput counts every rank's work.  Two gloo ranks on the CPU stand in for two
GPUs (no GPU is touched)."""
import argparse
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        local_ms = [3.0, 5.0][rank]                    # rank 1 is the slow one
        slowest = bench.max_over_ranks(local_ms, "cpu")
        out.put((rank, slowest, bench.replica_tflops(1.0e12, slowest, world)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest_and_count_both_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, tflops in got:
        assert slowest == 5.0                          # MAX over ranks, on every rank
        assert tflops == pytest.approx(2 * 1.0e12 / 5.0e-3 / 1e12)   # both replicas' work


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(4.25, "cpu") == 4.25
    assert bench.replica_tflops(2.0e12, 1.0, 1) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(gpus=2, steps=3, warmup=3, impl="reference",
                              workload="nvfp4_attn_1mp", m=0)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
