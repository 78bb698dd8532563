"""Adjacent-query dedup attention (dsa_sparse_attn_prefill_dedup) against the
fp64 oracle: same bars as the per-query kernel (max-abs 2e-2, mean-abs
2e-3), on index rows from the GPU indexer (bit-exact with the oracle's),
with -1 holes, a ragged last block of queries, an out-of-range entry, a
repeated key, clustered (video) rows whose blocks share most keys, scores
that grow along the key order (the running maximum moves many times, so the
accumulator is rescaled in TMEM), and both block shapes (16 queries x 8
heads, 32 queries x 4 heads).

Kwai Keye-VL-2.0 technical-report summary, section 8, item 2 (the dedup) and
section 1 (the attention it reproduces)."""
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


def test_dedup_attention_on_clustered_video_rows():
    cfg = gen.custom(L=9000, H_I=64, d_I=128, k=2048, Hq=32, Hkv=4, d=128, video=True, seed=24)
    inp = gen.prefill_inputs(cfg)
    idx = dsa.index_topk(dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"]), cfg.k)
    Q, K, V = (dev(inp[n], torch.bfloat16) for n in ("Q", "K", "V"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O = dsa.sparse_attn_prefill_dedup(Q, K, V, idx, cfg.scale, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == dsa.DEVERR_NONE
    rows = np.unique(np.concatenate([np.arange(0, 20), np.arange(cfg.L - 20, cfg.L),
                                     np.linspace(20, cfg.L - 21, 60).astype(np.int64)]))
    ref = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], idx.cpu().numpy(), cfg.scale, rows=rows)
    check(O[torch.from_numpy(rows).cuda()], ref)
    O1 = dsa.sparse_attn_prefill(Q, K, V, idx, cfg.scale)
    diff = (O.float() - O1.float()).abs()
    assert diff.max().item() <= 2 * MAX_ABS and diff.mean().item() <= MEAN_ABS


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 4, 128), (8, 2, 64), (16, 4, 128), (16, 2, 64)])
def test_dedup_attention_with_a_moving_maximum(Hq, Hkv, d):
    """Key u's K row grows with u and every query has a positive bias along
    it, so the scores of later (larger) keys are larger by up to ~40 in
    log2 units: the running maximum moves past the rescale threshold many
    times while a block walks its keys in ascending order."""
    L, k = 2300, 512
    rng = np.random.default_rng(31)
    Qf = rng.standard_normal((L, Hq, d)) * 0.5 + 1.0
    grow = 3.0 * np.arange(L, dtype=np.float64)[:, None, None] / L
    Kf = (rng.standard_normal((L, Hkv, d)) * 0.5 + 1.0) * grow
    Vf = rng.standard_normal((L, Hkv, d))
    Qh, Kh, Vh = gen.encode_bf16(Qf), gen.encode_bf16(Kf), gen.encode_bf16(Vf)
    idx = np.full((L, k), -1, dtype=np.int32)
    for t in range(L):
        n = min(k, t + 1)
        idx[t, :n] = rng.permutation(rng.choice(t + 1, size=n, replace=False)).astype(np.int32)
    scale = 1.0 / np.sqrt(d)
    Q, K, V = (dev(a, torch.bfloat16) for a in (Qh, Kh, Vh))
    O = dsa.sparse_attn_prefill_dedup(Q, K, V, dev(idx), scale)
    assert dsa.device_error() == dsa.DEVERR_NONE
    rows = np.unique(np.concatenate([np.arange(0, 40), np.arange(L - 40, L),
                                     np.linspace(40, L - 41, 60).astype(np.int64)]))
    ref = oracle.sparse_attn(Qh, Kh, Vh, idx, scale, rows=rows)
    check(O[torch.from_numpy(rows).cuda()], ref)


def test_dedup_attention_counts_a_repeated_key_once():
    cfg = gen.custom(L=600, H_I=4, d_I=64, k=64, Hq=32, Hkv=4, d=128, seed=25)
    inp = gen.prefill_inputs(cfg)
    rng = np.random.default_rng(6)
    idx = np.full((cfg.L, cfg.k), -1, dtype=np.int32)
    for t in range(cfg.L):
        n = min(cfg.k, t + 1)
        idx[t, :n] = rng.choice(t + 1, size=n, replace=False).astype(np.int32)
    idx_rep = idx.copy()
    idx_rep[500, 10] = idx_rep[500, 3]       # key repeated in one row
    idx_rep[501, :] = idx_rep[501, 0]        # one key, k times
    Q, K, V = (dev(inp[n], torch.bfloat16) for n in ("Q", "K", "V"))
    O = dsa.sparse_attn_prefill_dedup(Q, K, V, dev(idx_rep), cfg.scale)
    assert dsa.device_error() == dsa.DEVERR_NONE
    once = idx_rep.copy()
    once[500, 10] = -1
    once[501, 1:] = -1
    rows = np.array([0, 1, 499, 500, 501, 502, 599])
    ref = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], once, cfg.scale, rows=rows)
    check(O[torch.from_numpy(rows).cuda()], ref)


def _random_rows(L, k, rng, hole_frac=0.0):
    idx = np.full((L, k), -1, dtype=np.int32)
    for t in range(L):
        n = min(k, t + 1)
        sel = rng.choice(t + 1, size=n, replace=False).astype(np.int32)
        if hole_frac:
            sel[rng.random(n) < hole_frac] = -1
        idx[t, :n] = sel
    return idx


def test_dedup_attention_across_two_waves():
    """4096 blocks of 16 rows form one wave: L = 66 536 needs two, so rows on
    both sides of the wave boundary (65 535 / 65 536) and the ragged last
    block are compared with the oracle."""
    L, k = 4096 * 16 + 1000, 16
    rng = np.random.default_rng(41)
    cfg = gen.custom(L=L, H_I=4, d_I=64, k=k, Hq=32, Hkv=4, d=128, seed=42)
    Qh, Kh, Vh = gen.prefill_Q(cfg), gen.prefill_K(cfg), gen.prefill_V(cfg)
    idx = _random_rows(L, k, rng)
    Q, K, V = (dev(a, torch.bfloat16) for a in (Qh, Kh, Vh))
    O = dsa.sparse_attn_prefill_dedup(Q, K, V, dev(idx), cfg.scale)
    assert dsa.device_error() == dsa.DEVERR_NONE
    rows = np.unique(np.concatenate([np.arange(0, 20), np.arange(65520, 65552),
                                     np.arange(L - 20, L),
                                     np.linspace(20, L - 21, 60).astype(np.int64)]))
    ref = oracle.sparse_attn(Qh, Kh, Vh, idx, cfg.scale, rows=rows)
    check(O[torch.from_numpy(rows).cuda()], ref)


@pytest.mark.parametrize("L,k", [(1, 1), (17, 4), (40, 64)])
def test_dedup_attention_degenerate_shapes(L, k):
    """One row; one full block plus one row; k above L; and a block whose
    rows select nothing (rows 16..31 all holes: zeros)."""
    rng = np.random.default_rng(43 + L)
    cfg = gen.custom(L=L, H_I=4, d_I=64, k=k, Hq=32, Hkv=4, d=128, seed=44)
    Qh, Kh, Vh = gen.prefill_Q(cfg), gen.prefill_K(cfg), gen.prefill_V(cfg)
    idx = _random_rows(L, k, rng)
    if L >= 32:
        idx[16:32] = -1
    Q, K, V = (dev(a, torch.bfloat16) for a in (Qh, Kh, Vh))
    O = dsa.sparse_attn_prefill_dedup(Q, K, V, dev(idx), cfg.scale)
    assert dsa.device_error() == dsa.DEVERR_NONE
    rows = np.arange(L)
    ref = oracle.sparse_attn(Qh, Kh, Vh, idx, cfg.scale, rows=rows)
    check(O, ref)
    if L >= 32:
        assert float(O[16:32].float().abs().max()) == 0.0
