"""Multi-rank plumbing of bench.py on CPU with gloo (world size 2): every rank runs its own,
equally shaped batch (weak scaling by request), timings reduce to the slowest rank, and the
job's throughput counts every rank's rows."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sparse_attention_12_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synth.custom("ranks", [300, 500], [1, 1], n_heads_index=16, topk=64, n_heads=16)
        hb = synth.make_batch(wl, seed=bench.rank_seed(rank))
        step_ms = 2.0 + 3.0 * rank            # this rank's (fake) step time
        ms = bench.max_over_ranks(step_ms, dist, "cpu")
        digest = float(hb.kI_scale.sum())
        out_q.put((rank, ms, bench.job_throughput(hb.total_q, world, ms), digest, hb.qI.shape, hb.q.shape))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, d0, qi0, q0), (r1, ms1, v1, d1, qi1, q1) = res
    assert ms0 == ms1 == 5.0                  # both ranks report the slowest rank
    assert v0 == v1 == 2 * 2 / (5.0 / 1e3)    # 2 ranks x 2 query rows over 5 ms
    assert qi0 == qi1 and q0 == q1            # same shapes on every rank
    assert d0 != d1                           # different data on every rank
