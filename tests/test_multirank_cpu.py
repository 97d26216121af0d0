"""The N > 1 path of bench.py on CPU: two gloo ranks (one process each, the
way torchrun starts them) run the host logic the GPU bench uses between
ranks. That is the max-over-ranks step time, the whole-job throughput over all
replicas, and each rank's own seeded token stream. bench.py shards the work
into independent replicas (no data-path collective), so these are the only
exchanges there are. Rendezvous on 127.0.0.1."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                    # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, world, device="cpu")
        toks = bench.replica_tokens(rank, 2, 16, 50257)
        again = bench.replica_tokens(rank, 2, 16, 50257)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), ms_max=ms_max,
                 thr=bench.job_throughput(ms_max, 2, 16, world),
                 idx0=toks[0][0], tgt0=toks[0][1], same=all(np.array_equal(a[0], b[0]) for a, b in zip(toks, again)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_time_and_throughput(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    r = [np.load(tmp_path / f"r{k}.npz") for k in range(world)]
    for k in range(world):
        assert float(r[k]["ms_max"]) == 15.0           # the slowest rank's time, on every rank
        assert float(r[k]["thr"]) == pytest.approx(2 * 16 * world / 0.015)
        assert bool(r[k]["same"])                       # a rank's stream is reproducible
    # ... and the replicas see different data
    assert not np.array_equal(r[0]["idx0"], r[1]["idx0"])
    # targets are the ids shifted by one within each rank's stream
    assert np.array_equal(r[0]["idx0"][:, 1:], r[0]["tgt0"][:, :-1])


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(20.0, 16, 1024, 1) == pytest.approx(16 * 1024 / 0.02)
