"""The multi-GPU exchange logic on CPU, world sizes 2 and 3 over gloo (the
same torch.distributed calls run over NCCL on GPUs):

* gather_zigzag assembles every rank's zig-zag blocks of k_I / K / V into
  the full arrays on every rank;
* with the keys gathered, every rank's own rows of the oracle's selection
  equal those rows of the one-process selection (the query-shard plan is
  exact);
* deal_sequences gives each decode sequence to exactly one rank.

Source: the openi.cn product page's deployment list (two or more GPUs) and
the Keye-VL-2.0 technical-report summary, section 1 (the selection)."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

import gen
from sparse_long_context_02_b200 import dist, shards


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as tdist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = gen.custom(L=600, H_I=4, d_I=64, k=48, seed=81)
        full = gen.prefill_inputs(cfg)
        # this rank holds only its own blocks of the key tensors (gloo moves
        # them as int32 words; NCCL takes the bytes and bf16 as they are)
        blk = shards.zigzag_blocks(cfg.L, world)[0][1]
        res = {}
        gathered = {}
        for name in ("k_I", "K"):
            a = np.ascontiguousarray(full[name]).reshape(cfg.L, -1)
            t = torch.from_numpy(a.view(np.int32))
            got = torch.empty((2 * world * blk, t.shape[1]), dtype=torch.int32)
            dist.gather_zigzag(dist.own_blocks(t, cfg.L, world, rank), got, cfg.L, world)
            res[name] = bool(torch.equal(got[:cfg.L], t))
            gathered[name] = got[:cfg.L].numpy().view(a.dtype).reshape(full[name].shape)
        kI = gathered["k_I"]
        sel_ok = True
        for a, b in shards.zigzag_rows(cfg.L, world, rank):
            rows = np.arange(a, b, dtype=np.int64)
            # the rank's query rows and the gathered keys only
            q_rows = np.zeros_like(full["q_I"])
            q_rows[a:b] = full["q_I"][a:b]
            w_rows = np.zeros_like(full["w"])
            w_rows[a:b] = full["w"][a:b]
            mine = oracle.index_topk(q_rows, kI, w_rows, cfg.k, rows=rows)
            ref = oracle.index_topk(full["q_I"], full["k_I"], full["w"], cfg.k, rows=rows)
            sel_ok = sel_ok and np.array_equal(mine, ref)
        res["selection"] = sel_ok
        res["rows"] = shards.zigzag_rows(cfg.L, world, rank)
        out[rank] = res
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


def _run(world):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    return [out[r] for r in range(world)]


def test_zigzag_gather_and_selection_two_ranks():
    res = _run(2)
    for r in res:
        assert r["k_I"] and r["K"] and r["selection"]
    rows = sorted(x for r in res for x in r["rows"])
    assert rows[0][0] == 0 and rows[-1][1] == 600


def test_zigzag_gather_and_selection_three_ranks():
    res = _run(3)
    for r in res:
        assert r["k_I"] and r["K"] and r["selection"]


def test_deal_sequences_is_a_partition_and_balanced():
    lens = gen.decode_lengths(gen.DECODE_B64)
    for P in (2, 4, 8):
        own = dist.deal_sequences(lens, P)
        flat = sorted(b for o in own for b in o)
        assert flat == list(range(len(lens)))
        load = [int(sum(lens[o])) for o in own]
        assert max(load) / min(load) < 1.15
