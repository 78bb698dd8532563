"""Adjacent-query dedup attention (dsa_sparse_attn_prefill_dedup) against the
fp64 oracle: same bars as the per-query kernel (max-abs 2e-2, mean-abs
2e-3), on index rows from the GPU indexer (bit-exact with the oracle's),
with -1 holes, a ragged last block of queries and an out-of-range entry."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sparse_long_context_02_b200 as dsa

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def check(O_gpu, ref):
    got = O_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS, err.max()
    assert err.mean() <= MEAN_ABS, err.mean()


@pytest.mark.parametrize("L,k,H_I,d_I,Hq,Hkv,d", [(3001, 256, 64, 128, 32, 4, 128),
                                                  (2500, 2048, 64, 128, 32, 4, 128),
                                                  (1999, 256, 4, 64, 8, 2, 64)])
def test_dedup_attention_matches_oracle(L, k, H_I, d_I, Hq, Hkv, d):
    cfg = gen.custom(L=L, H_I=H_I, d_I=d_I, k=k, Hq=Hq, Hkv=Hkv, d=d, seed=21)
    inp = gen.prefill_inputs(cfg)
    idx = dsa.index_topk(dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"]), k)
    Q, K, V = (dev(inp[n], torch.bfloat16) for n in ("Q", "K", "V"))
    O = dsa.sparse_attn_prefill_dedup(Q, K, V, idx, cfg.scale)
    assert dsa.device_error() == dsa.DEVERR_NONE
    rows = np.unique(np.concatenate([np.arange(0, 13), np.arange(L - 13, L),
                                     np.linspace(13, L - 14, 40).astype(np.int64)]))
    ref = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], idx.cpu().numpy(), cfg.scale, rows=rows)
    check(O[torch.from_numpy(rows).cuda()], ref)
    # and close to the per-query kernel everywhere
    O1 = dsa.sparse_attn_prefill(Q, K, V, idx, cfg.scale)
    diff = (O.float() - O1.float()).abs()
    assert diff.max().item() <= 2 * MAX_ABS and diff.mean().item() <= MEAN_ABS


def test_dedup_attention_holes_empty_rows_and_bad_index():
    cfg = gen.custom(L=700, H_I=4, d_I=64, k=64, Hq=8, Hkv=2, d=64, seed=22)
    inp = gen.prefill_inputs(cfg)
    rng = np.random.default_rng(5)
    idx = np.full((cfg.L, cfg.k), -1, dtype=np.int32)
    for t in range(cfg.L):
        n = min(cfg.k, t + 1)
        sel = np.sort(rng.choice(t + 1, size=n, replace=False)).astype(np.int32)
        holes = rng.random(n) < 0.2
        sel[holes] = -1
        idx[t, :n] = sel
    idx[5, :] = -1                      # a row with no key: zeros
    idx_bad = idx.copy()
    idx_bad[300, 3] = cfg.L + 7         # out of range: skipped and flagged
    Q, K, V = (dev(inp[n], torch.bfloat16) for n in ("Q", "K", "V"))
    O = dsa.sparse_attn_prefill_dedup(Q, K, V, dev(idx_bad), cfg.scale)
    assert dsa.device_error() == dsa.DEVERR_INDEX
    rows = np.array([0, 1, 5, 6, 299, 300, 301, 697, 698, 699])
    idx_ref = idx_bad.copy()
    idx_ref[idx_ref >= cfg.L] = -1
    ref = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], idx_ref, cfg.scale, rows=rows)
    check(O[torch.from_numpy(rows).cuda()], ref)
    assert float(O[5].float().abs().max()) == 0.0
    assert dsa.device_error() == dsa.DEVERR_NONE
