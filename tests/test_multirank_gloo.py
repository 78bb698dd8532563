"""The multi-rank host logic of the benchmark on CPU, world size 2 over gloo:
every rank gets its own problem, timings are reduced with max over ranks and
the job throughput counts the units of all ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import gen


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as tdist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p, d = bench.rank_workloads(gen.PREFILL_128K, gen.DECODE_B64, rank, world)
        # each rank draws its own inputs: first indexer-key bytes differ
        first = gen.prefill_kI(p, 0, 4).tobytes()
        times = bench.max_over_ranks([10.0 + rank, 5.0 - rank], world)
        out[rank] = dict(seed_p=p.seed_, seed_d=d.seed_, first=first, times=times.tolist(),
                         tput=bench.job_throughput(p.L, world, times[0] / 1e3))
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    assert r0["seed_p"] != r1["seed_p"] and r0["seed_d"] != r1["seed_d"]
    assert r0["first"] != r1["first"]
    assert r0["times"] == r1["times"] == [11.0, 5.0]          # elementwise max
    assert r0["tput"] == pytest.approx(2 * 131072 / 0.011)   # both ranks' tokens / slowest time


def test_single_rank_is_identity():
    import bench
    p, d = bench.rank_workloads(gen.PREFILL_128K, gen.DECODE_B64, 0, 1)
    assert p is gen.PREFILL_128K and d is gen.DECODE_B64
    assert np.array_equal(bench.max_over_ranks([1.0, 2.0], 1), [1.0, 2.0])
