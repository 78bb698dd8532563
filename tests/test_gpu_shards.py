"""The multi-GPU decompositions, validated on one GPU: every rank's share
runs here one after the other, and the exchanges are concatenations.

* Prefill query shards (zig-zag blocks): each rank's index rows and
  attention rows, computed from its own query rows and the keys up to its
  last row, equal the one-call results bit for bit.
* Decode cache shards: per-rank top-k pairs, their merge, per-rank attention
  partials and their log-sum-exp merge give the same index rows as the
  one-GPU decode (bit for bit; also against the oracle) and outputs within
  the attention tolerance of the oracle.

Kwai Keye-VL-2.0 technical-report summary, section 1 (the selection and
attention these shards reproduce) and section 8 (decode); the deployment
list of the openi.cn product page runs the model on two or more GPUs."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sparse_long_context_02_b200 as dsa
from sparse_long_context_02_b200 import shards

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def dev(a, dt=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dt) if dt is not None else t).cuda()


@pytest.mark.parametrize("P", [2, 3, 4])
def test_prefill_query_shards_equal_the_whole_prefill(P):
    cfg = gen.custom(L=5000, H_I=64, d_I=128, k=2048, Hq=32, Hkv=4, d=128, seed=71)
    h = gen.prefill_inputs(cfg)
    q, kI, w = dev(h["q_I"]), dev(h["k_I"]), dev(h["w"])
    Q, K, V = (dev(h[n], torch.bfloat16) for n in ("Q", "K", "V"))
    idx = dsa.index_topk(q, kI, w, cfg.k)
    O = dsa.sparse_attn_prefill(Q, K, V, idx, cfg.scale)
    covered = np.zeros(cfg.L, bool)
    for r in range(P):
        for a, b in shards.zigzag_rows(cfg.L, P, r):
            covered[a:b] = True
            # what rank r holds: its query rows, and keys 0 .. b-1
            i_r = dsa.index_topk_rows(q[a:b].contiguous(), kI[:b].contiguous(),
                                      w[a:b].contiguous(), a, cfg.k)
            assert torch.equal(i_r, idx[a:b]), (r, a, b)
            O_r = dsa.sparse_attn_rows(Q[a:b].contiguous(), K[:b].contiguous(),
                                       V[:b].contiguous(), i_r, cfg.scale)
            assert torch.equal(O_r, O[a:b]), (r, a, b)
    assert covered.all()
    assert dsa.device_error() == dsa.DEVERR_NONE


def test_zigzag_blocks_balance_the_causal_work():
    L, P = 131072, 8
    work = [shards.causal_pairs(shards.zigzag_rows(L, P, r)) for r in range(P)]
    assert max(work) / min(work) < 1.001
    rows = sorted(x for r in range(P) for x in shards.zigzag_rows(L, P, r))
    assert rows[0][0] == 0 and rows[-1][1] == L
    assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))


def _decode_case(lens, seed, k):
    cfg = gen.Config(0, "sharded decode", "decode", k=k, H_I=64, d_I=128, Hq=32, Hkv=4, d=128,
                     B=len(lens), seed=seed)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = int(off[-1])
    q = gen.decode_queries(cfg)
    return cfg, off, q, gen.decode_kI_rows(cfg, 0, N), gen.decode_K_rows(cfg, 0, N), \
        gen.decode_V_rows(cfg, 0, N)


@pytest.mark.parametrize("P,lens,k", [(2, [5000, 70000, 2048, 3], 2048),
                                      (3, [40001, 2, 9000, 100000, 2049], 2048),
                                      (4, [30000, 1, 7, 65536], 512),
                                      (8, [300000, 12345], 2048)])
def test_decode_cache_shards_equal_the_one_gpu_decode(P, lens, k):
    cfg, off, q, kI_h, K_h, V_h = _decode_case(np.array(lens), seed=72 + P, k=k)
    B = cfg.B
    qI, w, Q = dev(q["q_I"]), dev(q["w"]), dev(q["Q"], torch.bfloat16)
    kI, K, V = dev(kI_h), dev(K_h, torch.bfloat16), dev(V_h, torch.bfloat16)
    idx1 = torch.empty((B, k), dtype=torch.int32, device="cuda")
    O1, _ = dsa.sparse_attn_decode(qI, w, Q, kI, K, V, dev(off), k, cfg.scale, idx_out=idx1)

    parts = shards.cache_parts(np.array(lens), P)
    packed = []
    for pr in parts:  # each rank's packed cache: its rows of every sequence
        rows = np.concatenate([np.arange(s, s + n) for s, n in zip(pr["src"], pr["lens"])])
        rows = torch.from_numpy(rows.astype(np.int64)).cuda()
        packed.append((kI[rows].contiguous(), K[rows].contiguous(), V[rows].contiguous(),
                       dev(pr["off"]), dev(pr["base"])))
    ords, keys = [], []
    for kI_r, _, _, off_r, base_r in packed:
        o, kk = dsa.decode_select_shard(qI, w, kI_r, off_r, k, key_base=base_r)
        ords.append(o)
        keys.append(kk)
    idx = dsa.decode_merge_shards(torch.stack(ords), torch.stack(keys))
    assert torch.equal(idx, idx1)
    po, pml = [], []
    for kI_r, K_r, V_r, off_r, base_r in packed:
        o, m = dsa.decode_attn_shard(Q, K_r, V_r, off_r, base_r, idx, cfg.scale)
        po.append(o)
        pml.append(m)
    O = dsa.decode_combine_shards(torch.stack(po), torch.stack(pml))
    assert dsa.device_error() == dsa.DEVERR_NONE
    r_idx, r_O = oracle.decode(q["q_I"], q["w"], q["Q"], kI_h, K_h, V_h, off, k, cfg.scale)
    assert np.array_equal(idx.cpu().numpy(), r_idx)
    for got in (O, O1):
        err = np.abs(got.float().cpu().numpy() - r_O)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
