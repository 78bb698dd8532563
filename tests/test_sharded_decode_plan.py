"""The planned cache-sharded decode (one long sequence's cache rows split over
ranks), checked on the oracle with two gloo ranks on CPU: each rank selects
its local top-k by the total order (score descending, key ascending), the
candidates are all-gathered and merged by the same order, and the result
equals the single-rank top-k bit for bit; the attention over the merged keys,
computed as per-rank partials (unnormalised O, running max, sum) and combined
by log-sum-exp, equals the single-rank attention.  No GPU code runs here: this
pins the decomposition the multi-GPU decode is to implement."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import gen
import oracle

K_SEL = 256
LENS = [3001, 1700]  # two sequences, each split in two ragged halves over the ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    cfg = gen.Config(0, "sharded decode check", "decode", k=K_SEL, H_I=4, d_I=64, Hq=8, Hkv=2,
                     d=64, B=len(LENS), seed=61)
    off = np.concatenate([[0], np.cumsum(LENS)]).astype(np.int64)
    N = int(off[-1])
    q = gen.decode_queries(cfg)
    return (cfg, off, q, gen.decode_kI_rows(cfg, 0, N), gen.decode_K_rows(cfg, 0, N),
            gen.decode_V_rows(cfg, 0, N))


def _bf16(a):
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _shard(n, rank, world):
    lo = n * rank // world
    return lo, n * (rank + 1) // world


def _local_candidates(cfg, q, kI, b, lo, hi, off):
    """(score, key) of this rank's keys [lo, hi) of sequence b, its top-k by the
    total order.  The decode query's scores are the last row of a prefill
    problem whose keys are the local rows (decode = last prefill row)."""
    m = hi - lo
    if m <= 0:
        return []
    q_pre = np.zeros((m + 1, cfg.H_I, cfg.d_I), np.uint8)
    q_pre[m] = q["q_I"][b]
    w_pre = np.zeros((m + 1, cfg.H_I), np.float32)
    w_pre[m] = q["w"][b]
    k_pre = np.zeros((m + 1, cfg.d_I), np.uint8)
    k_pre[:m] = kI[off[b] + lo:off[b] + hi]
    scores = oracle.index_scores(q_pre, k_pre, w_pre, rows=[m])[0, :m]
    order = np.lexsort((np.arange(m), -scores))[:K_SEL]
    return [(float(scores[i]), int(lo + i)) for i in order]


def _partials(cfg, q, K, V, b, keys, off):
    """Unnormalised O, running max and sum per query head over `keys`."""
    G = cfg.Hq // cfg.Hkv
    Qf = _bf16(q["Q"][b])                     # [Hq][d]
    o = np.zeros((cfg.Hq, cfg.d))
    mx = np.full(cfg.Hq, -np.inf)
    sm = np.zeros(cfg.Hq)
    if len(keys):
        rows = off[b] + np.asarray(keys)
        Kf, Vf = _bf16(K[rows]), _bf16(V[rows])   # [n][Hkv][d]
        for h in range(cfg.Hq):
            x = cfg.scale * (Kf[:, h // G, :] @ Qf[h])
            mx[h] = x.max()
            e = np.exp(x - mx[h])
            sm[h] = e.sum()
            o[h] = e @ Vf[:, h // G, :]
    return o, mx, sm


def _worker(rank, world, port, out):
    import torch.distributed as tdist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, off, q, kI, K, V = _problem()
        res = []
        for b, n in enumerate(LENS):
            lo, hi = _shard(n, rank, world)
            local = _local_candidates(cfg, q, kI, b, lo, hi, off)
            gathered = [None] * world
            tdist.all_gather_object(gathered, local)
            cand = [c for part in gathered for c in part]
            merged = sorted(cand, key=lambda c: (-c[0], c[1]))[:K_SEL]
            sel = sorted(c[1] for c in merged)
            mine = [s for s in sel if lo <= s < hi]
            parts = [None] * world
            tdist.all_gather_object(parts, _partials(cfg, q, K, V, b, mine, off))
            m = np.maximum.reduce([p[1] for p in parts])  # per head
            num = sum(p[0] * np.exp(p[1] - m)[:, None] for p in parts)
            den = sum(p[2] * np.exp(p[1] - m) for p in parts)
            res.append((sel, num / den[:, None]))
        out[rank] = res
    finally:
        tdist.destroy_process_group()


def test_sharded_decode_decomposition_matches_single_rank():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    cfg, off, q, kI, K, V = _problem()
    ref_idx, ref_O = oracle.decode(q["q_I"], q["w"], q["Q"], kI, K, V, off, cfg.k, cfg.scale)
    for rank in range(world):
        for b, n in enumerate(LENS):
            sel, O = out[rank][b]
            want = ref_idx[b][ref_idx[b] >= 0]
            assert np.array_equal(np.asarray(sel, np.int64), want.astype(np.int64)), (rank, b)
            assert np.abs(O - ref_O[b]).max() < 1e-12, (rank, b)
