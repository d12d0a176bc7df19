"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on CPU.

Batch rows are independent, so `bench.py --gpus N` gives every rank its own
rows (weak scaling) and uses no collective on the data path: only a barrier
and a maximum over ranks of the step timings.  These tests check that logic
(per-rank seeds, the max-over-ranks reduction, the whole-job throughput)
through a real two-process group."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from fsq_latent_decode_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank times its own rows; the job takes the slowest rank's time
        ms, kern = bench.max_over_ranks(torch, dist, [10.0 + rank, 5.0 - rank], torch.device("cpu"))
        seed = bench.rank_seed(synth, rank, 16, 131072, 256)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        dist.barrier()
        out.put((rank, ms, kern, seeds))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_reduce_timings_and_draw_distinct_rows():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, ms, kern, seeds in res:
        assert ms == 11.0 and kern == 5.0  # element-wise maximum over the two ranks
        assert len(set(seeds)) == world    # every rank draws its own batch rows
    assert res[0][3] == res[1][3]


def test_single_process_path_and_job_throughput():
    assert bench.max_over_ranks(torch, None, [1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]
    # weak scaling: N ranks of B rows x T tokens in the slowest rank's step time
    assert bench.job_throughput(1, 16, 131072, 0.125) == pytest.approx(16 * 131072 / 0.125e-3)
    assert bench.job_throughput(8, 16, 131072, 0.125) == pytest.approx(8 * bench.job_throughput(1, 16, 131072, 0.125))
