"""Multi-rank host logic of bench.py, on two gloo ranks on the CPU: the step
time every rank reports is the max over ranks, the whole-job throughput
counts every rank's batch, and each rank draws its own inputs."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [10.0 + 5.0 * rank, 3.0 - rank]            # per-rank timings
        mx = bench.max_over_ranks(ms, device="cpu")
        cfg = synth.CsaDecode("t", B=2, N=4096, H=4, d=128, H_I=2, c_I=64, m=4, k=8, W=4, lam=0.1,
                              seed=1 + bench.rank_seed_offset(rank))
        q = synth.csa_decode_inputs(cfg)["q"].float()
        qs = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(qs, q)
        out[rank] = (mx, bench.job_throughput(64, world, mx[0]), bool(torch.equal(qs[0], qs[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        mx, value, same_inputs = res[rank]
        assert mx == [15.0, 3.0]                        # max over ranks, element-wise
        assert value == pytest.approx(64 * 2 / 0.015)   # both ranks' units / slowest time
        assert not same_inputs                          # ranks draw different batches
