"""Host logic of the N-GPU benchmark path, on CPU with two gloo ranks: every
rank runs its own layer (no collective on the data path); the job time is the
slowest rank's and the value sums all ranks' kept-pair flops."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        elapsed = 10.0 + 5.0 * rank  # the second rank is slower
        flops = 1e12 * (rank + 1)
        t = bench.max_over_ranks(elapsed, "cpu", world)
        f = bench.sum_over_ranks(flops, "cpu", world)
        out[rank] = (t, f, bench.whole_job_tflops(f, 4, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_value():
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for r in range(2):
        t, f, v = out[r]
        assert t == 15.0  # max over ranks
        assert f == 3e12  # sum of both ranks' flops
        assert v == pytest.approx(4 * 3e12 / 15e-3 / 1e12)


def test_reference_arm_other_ranks_do_nothing(capsys):
    import argparse

    import bench

    bench.run_reference(argparse.Namespace(steps=1, warmup=0, gpus=2), rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_single_rank_helpers_need_no_process_group():
    import bench

    assert bench.max_over_ranks(3.5, "cpu", 1) == 3.5
    assert bench.sum_over_ranks(2.0, "cpu", 1) == 2.0
    assert not dist.is_initialized()
    assert torch.tensor(1.0).item() == 1.0
