"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against what the definition and mathematics fix:
library decoders, a hand-derived worked example, brute force in Python
integers on tiny inputs, closed forms and invariants, and a separately
written dense causal attention.  Definitions: Kwai Keye-VL-2.0
technical-report summary, section 1 (indexer, top-2048 selection, sparse GQA
attention) and section 8 (decode)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import gen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def e4m3_ints(byte_arr):
    """Library decode of e4m3 bytes (torch's float8_e4m3fn), to exact ints."""
    t = torch.from_numpy(np.ascontiguousarray(byte_arr)).view(torch.float8_e4m3fn).float()
    return t.numpy().astype(np.int64)


def bf16_vals(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.double().numpy()


# ---------------------------------------------------------------- decoding

def test_e4m3_decode_matches_library_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_value(c) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decode_matches_library():
    bits = np.array([0x0000, 0x8000, 0x3F80, 0xBF80, 0x4049, 0x0001, 0x7F7F, 0x3C23, 0xC2F7],
                    dtype=np.uint16)
    got = np.array([oracle.bf16_value(b) for b in bits])
    assert np.array_equal(got, bf16_vals(bits))


# ---------------------------------------------------------------- worked examples

def _example_topk():
    with open(os.path.join(GOLDEN, "worked_example_topk.json")) as f:
        ex = json.load(f)
    q = gen.encode_e4m3(np.array(ex["q"], np.float64))
    kI = gen.encode_e4m3(np.array(ex["k_I"], np.float64))
    w = np.array(ex["w"], np.float32)
    return ex, q, kI, w


def test_worked_example_topk():
    ex, q, kI, w = _example_topk()
    idx = oracle.index_topk(q, kI, w, ex["k"])
    assert idx.tolist() == ex["idx"]


def test_worked_example_scores():
    ex, q, kI, w = _example_topk()
    sc = oracle.index_scores(q, kI, w)
    for t, row in enumerate(ex["scores"]):
        assert sc[t, :t + 1].tolist() == row
        assert np.all(np.isneginf(sc[t, t + 1:]))


def test_worked_example_attn():
    with open(os.path.join(GOLDEN, "worked_example_attn.json")) as f:
        ex = json.load(f)
    Q = gen.encode_bf16(np.array(ex["Q"]))
    K = gen.encode_bf16(np.array(ex["K"]))
    V = gen.encode_bf16(np.array(ex["V"]))
    idx = np.array(ex["idx"], np.int32)
    O = oracle.sparse_attn(Q, K, V, idx, ex["scale"])
    assert np.allclose(O, np.array(ex["O"]), atol=1e-15, rtol=0)


# ---------------------------------------------------------------- brute force

def brute_topk(q_b, kI_b, w, k):
    """Python-integer scores and a full sort of every (score, s) pair."""
    qi, ki = e4m3_ints(q_b), e4m3_ints(kI_b)
    L, H, d = qi.shape
    out = []
    for t in range(L):
        cands = []
        for s in range(t + 1):
            sc = 0
            for j in range(H):
                dot = sum(int(qi[t, j, c]) * int(ki[s, c]) for c in range(d))
                sc += int(w[t, j]) * max(0, dot)
            cands.append((-sc, s))
        cands.sort()
        sel = sorted(s for _, s in cands[:k])
        out.append(sel + [-1] * (k - len(sel)))
    return np.array(out, np.int32)


@pytest.mark.parametrize("L,H,d,k,seed", [
    (16, 1, 2, 1, 1), (33, 2, 4, 4, 2), (64, 2, 3, 7, 3), (48, 1, 4, 48, 4),
    (40, 2, 4, 16, 5), (64, 1, 1, 5, 6),
])
def test_topk_matches_brute_force(L, H, d, k, seed):
    cfg = gen.custom(L=L, H_I=H, d_I=d, k=k, seed=seed)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    assert np.array_equal(oracle.index_topk(q, kI, w, k), brute_topk(q, kI, w, k))


def test_topk_ties_small_range_brute_force():
    # values in {-1,0,1} and weights in {0,1} make many exact ties
    L, H, d, k = 50, 2, 3, 6
    cfg = gen.custom(L=L, H_I=H, d_I=d, k=k, seed=11)
    q = gen.int_e4m3(cfg.seed_, 1, 0, L * H * d, -1, 1).reshape(L, H, d)
    kI = gen.int_e4m3(cfg.seed_, 2, 0, L * d, -1, 1).reshape(L, d)
    w = gen.int_f32(cfg.seed_, 3, 0, L * H, 0, 1).reshape(L, H)
    assert np.array_equal(oracle.index_topk(q, kI, w, k), brute_topk(q, kI, w, k))


def test_scores_match_brute_force():
    cfg = gen.custom(L=24, H_I=2, d_I=4, seed=7)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    qi, ki = e4m3_ints(q), e4m3_ints(kI)
    sc = oracle.index_scores(q, kI, w)
    for t in range(cfg.L):
        for s in range(cfg.L):
            if s > t:
                assert sc[t, s] == -math.inf
            else:
                ref = sum(int(w[t, j]) * max(0, int(np.dot(qi[t, j], ki[s]))) for j in range(2))
                assert sc[t, s] == ref


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("mode", ["w0", "q0", "neg"])
def test_all_zero_scores_select_lowest_indices(mode):
    L, H, d, k = 40, 4, 8, 9
    cfg = gen.custom(L=L, H_I=H, d_I=d, k=k, seed=21)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    if mode == "w0":
        w = np.zeros_like(w)
    elif mode == "q0":
        q = gen.encode_e4m3(np.zeros((L, H, d)))
    else:  # every dot product negative: q <= -1 elementwise, k >= 1
        q = gen.encode_e4m3(-np.abs(e4m3_ints(q)) - 1)
        kI = gen.encode_e4m3(np.abs(e4m3_ints(kI)) + 1)
    idx = oracle.index_topk(q, kI, w, k)
    for t in range(L):
        m = min(k, t + 1)
        assert idx[t].tolist() == list(range(m)) + [-1] * (k - m)


def test_weight_scaling_and_head_permutation_invariance():
    cfg = gen.custom(L=96, H_I=4, d_I=16, k=12, seed=31)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    base = oracle.index_topk(q, kI, w, cfg.k)
    assert np.array_equal(base, oracle.index_topk(q, kI, w * 2, cfg.k))
    perm = np.array([2, 0, 3, 1])
    assert np.array_equal(base, oracle.index_topk(q[:, perm], kI, w[:, perm], cfg.k))
    s1 = oracle.index_scores(q, kI, w)
    s2 = oracle.index_scores(q, kI, w * 2)
    fin = np.isfinite(s1)
    assert np.array_equal(s2[fin], 2 * s1[fin])


def test_selection_invariants():
    cfg = gen.custom(L=200, H_I=4, d_I=16, k=20, seed=41)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    idx = oracle.index_topk(q, kI, w, cfg.k)
    sc = oracle.index_scores(q, kI, w)
    for t in range(cfg.L):
        m = min(cfg.k, t + 1)
        sel = idx[t, :m]
        assert np.all(idx[t, m:] == -1)
        assert np.all(np.diff(sel) > 0) and sel[0] >= 0 and sel[-1] <= t
        unsel = np.setdiff1d(np.arange(t + 1), sel)
        if unsel.size:
            worst_sel = min((sc[t, s], -s) for s in sel)
            best_uns = max((sc[t, s], -s) for s in unsel)
            assert worst_sel > best_uns


def _attn_inputs(L=64, Hq=8, Hkv=2, d=32, seed=51):
    cfg = gen.custom(L=L, Hq=Hq, Hkv=Hkv, d=d, seed=seed)
    return cfg, gen.prefill_Q(cfg), gen.prefill_K(cfg), gen.prefill_V(cfg)


def test_equal_keys_give_mean_of_selected_values():
    cfg, Q, K, V = _attn_inputs()
    K = np.broadcast_to(K[:1], K.shape).copy()
    rng = np.random.default_rng(0)
    idx = np.stack([np.sort(rng.choice(cfg.L, 10, replace=False)) for _ in range(cfg.L)])
    idx = idx.astype(np.int32)
    O = oracle.sparse_attn(Q, K, V, idx, cfg.scale)
    Vd = bf16_vals(V)
    G = cfg.Hq // cfg.Hkv
    for t in range(cfg.L):
        for h in range(cfg.Hq):
            ref = Vd[idx[t], h // G].mean(axis=0)
            assert np.allclose(O[t, h], ref, atol=1e-12, rtol=0)


def test_group_constant_values_pin_gqa_mapping():
    cfg, Q, K, V = _attn_inputs(Hq=8, Hkv=4)
    Vc = np.zeros((cfg.L, cfg.Hkv, cfg.d))
    for g in range(cfg.Hkv):
        Vc[:, g, :] = g + 1
    V = gen.encode_bf16(Vc)
    idx = np.tile(np.arange(16, dtype=np.int32), (cfg.L, 1))
    O = oracle.sparse_attn(Q, K, V, idx, cfg.scale)
    G = cfg.Hq // cfg.Hkv
    for h in range(cfg.Hq):
        assert np.allclose(O[:, h], h // G + 1, atol=1e-12, rtol=0)


def test_softmax_weights_sum_to_one():
    cfg, Q, K, V = _attn_inputs(L=128)
    rng = np.random.default_rng(1)
    idx = np.full((cfg.L, 24), -1, np.int32)
    for t in range(cfg.L):
        m = min(24, t + 1)
        idx[t, :m] = np.sort(rng.choice(t + 1, m, replace=False))
    for t in (0, 5, 23, 24, 77, 127):
        for h in range(cfg.Hq):
            p = oracle.attn_weights(Q, K, idx, cfg.scale, t, h)
            assert np.all(p >= 0)
            assert abs(p.sum() - 1.0) < 1e-12
            assert np.all(p[idx[t] < 0] == 0)


def test_sparse_with_k_at_least_t_plus_1_is_dense_causal():
    cfg = gen.custom(L=96, H_I=4, d_I=16, k=96, Hq=8, Hkv=2, d=32, seed=61)
    inp = gen.prefill_inputs(cfg)
    idx = oracle.index_topk(inp["q_I"], inp["k_I"], inp["w"], cfg.k)
    sparse = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], idx, cfg.scale)
    dense = oracle.dense_causal_attn(inp["Q"], inp["K"], inp["V"], cfg.scale)
    assert np.max(np.abs(sparse - dense)) < 1e-12


def test_sparse_rows_below_k_are_dense_causal_at_workload_shape():
    # rows t < k of the tiny prefill workload select every visible key
    cfg = gen.TINY_PREFILL.with_(L=300)
    inp = gen.prefill_inputs(cfg)
    rows = np.array([0, 1, 17, 128, 255], np.int64)
    idx = oracle.index_topk(inp["q_I"], inp["k_I"], inp["w"], cfg.k, rows=rows)
    full = np.full((cfg.L, cfg.k), -1, np.int32)
    full[rows] = idx
    sparse = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], full, cfg.scale, rows=rows)
    dense = oracle.dense_causal_attn(inp["Q"], inp["K"], inp["V"], cfg.scale, rows=rows)
    assert np.max(np.abs(sparse - dense)) < 1e-12


def test_constant_values_give_constant_output():
    cfg, Q, K, V = _attn_inputs()
    V = gen.encode_bf16(np.full(V.shape, 0.375))
    idx = np.tile(np.arange(0, 64, 3, dtype=np.int32), (cfg.L, 1))
    O = oracle.sparse_attn(Q, K, V, idx, cfg.scale)
    assert np.allclose(O, 0.375, atol=1e-14, rtol=0)


def test_two_key_softmax_closed_form_pins_scale_and_sign():
    cfg, Q, K, V = _attn_inputs(L=8, Hq=2, Hkv=1, d=4)
    Qd = np.zeros((8, 2, 4)); Qd[:, :, 0] = 2.0
    Kd = np.zeros((8, 1, 4)); Kd[3, 0, 0] = 1.5; Kd[5, 0, 0] = -0.5
    Vd = np.zeros((8, 1, 4)); Vd[3, 0, 1] = 1.0; Vd[5, 0, 2] = 1.0
    idx = np.tile(np.array([3, 5], np.int32), (8, 1))
    scale = 0.25
    O = oracle.sparse_attn(gen.encode_bf16(Qd), gen.encode_bf16(Kd), gen.encode_bf16(Vd), idx,
                           scale)
    x3, x5 = scale * 2.0 * 1.5, scale * 2.0 * -0.5
    p3 = math.exp(x3) / (math.exp(x3) + math.exp(x5))
    assert np.allclose(O[:, :, 1], p3, atol=1e-15)
    assert np.allclose(O[:, :, 2], 1 - p3, atol=1e-15)


def test_invalid_entries_are_skipped_and_empty_rows_are_zero():
    cfg, Q, K, V = _attn_inputs(L=16)
    idx = np.full((16, 4), -1, np.int32)
    idx[3] = [2, -1, 99, 1]
    O = oracle.sparse_attn(Q, K, V, idx, cfg.scale)
    assert np.all(O[0] == 0)
    ref_idx = idx.copy(); ref_idx[3] = [2, 1, -1, -1]
    O2 = oracle.sparse_attn(Q, K, V, ref_idx, cfg.scale)
    assert np.array_equal(O[3], O2[3])


# ---------------------------------------------------------------- decode

def test_decode_equals_last_prefill_row():
    cfg = gen.custom(L=160, H_I=4, d_I=16, k=24, Hq=8, Hkv=2, d=32, seed=71)
    inp = gen.prefill_inputs(cfg)
    lens = np.array([1, 23, 24, 25, 100, 160], np.int64)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    kI_c = np.concatenate([inp["k_I"][:n] for n in lens])
    K_c = np.concatenate([inp["K"][:n] for n in lens])
    V_c = np.concatenate([inp["V"][:n] for n in lens])
    t = lens - 1
    idx_d, O_d = oracle.decode(inp["q_I"][t], inp["w"][t], inp["Q"][t], kI_c, K_c, V_c, off,
                               cfg.k, cfg.scale)
    idx_p = oracle.index_topk(inp["q_I"], inp["k_I"], inp["w"], cfg.k, rows=t)
    full = np.full((cfg.L, cfg.k), -1, np.int32)
    full[t] = idx_p
    O_p = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], full, cfg.scale, rows=t)
    assert np.array_equal(idx_d, idx_p)
    assert np.array_equal(O_d, O_p)
