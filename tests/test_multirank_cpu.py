"""Host logic of the multi-GPU benchmark path, on CPU with gloo (world size 2):
every rank decodes its own batch (distinct seeds, same shape), the step time is
the maximum over ranks, and the job throughput counts every rank's bytes."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    case = synth.make_config(2, seed=bench.rank_seed(2, rank), values=False)
    t = bench.max_over_ranks(10.0 + rank, world, "cpu")      # ranks report 10 ms and 11 ms
    out[rank] = (t, int(case.context_lens.sum()), case.B, case.Hq)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_replicas_and_max_time():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 11.0                    # every rank sees the slowest rank
    assert out[0][1] != out[1][1]                            # distinct batches
    assert out[0][2:] == out[1][2:] == (32, 16)              # same shape
    assert bench.job_throughput_gbs(10**9, world, 11.0) == 2 * 10**9 / 0.011 / 1e9


def test_rank_zero_runs_the_workload_seed():
    assert bench.rank_seed(2, 0) is None
    a = synth.make_config(2, seed=bench.rank_seed(2, 0), values=False)
    b = synth.make_config(2, values=False)
    assert np.array_equal(a.context_lens, b.context_lens)
