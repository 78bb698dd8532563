"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars: indexer scores and top-k index sets bit-exact (integer-valued inputs
make every fp32 score exact); bf16 attention outputs within max-abs 2e-2 and
mean-abs 2e-3 of the fp64 oracle."""
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


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def check_attn(O_gpu: torch.Tensor, O_ref: np.ndarray):
    got = bf16_to_f64(O_gpu)
    err = np.abs(got - O_ref)
    assert err.max() <= MAX_ABS, err.max()
    assert err.mean() <= MEAN_ABS, err.mean()
    return err.max(), err.mean()


def no_device_error():
    assert dsa.device_error() == dsa.DEVERR_NONE


# ------------------------------------------------------------------ indexer

@pytest.mark.parametrize("L,H,d", [(300, 4, 64), (260, 64, 128), (129, 64, 64), (200, 4, 128)])
def test_index_scores_exact(L, H, d):
    cfg = gen.custom(L=L, H_I=H, d_I=d, seed=100 + L)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    ref = oracle.index_scores(q, kI, w)
    got = dsa.index_scores(dev(q), dev(kI), dev(w)).cpu().numpy().astype(np.float64)
    no_device_error()
    assert np.array_equal(got, ref)


def test_index_scores_worst_case_magnitude_is_exact():
    # every product +-64, alternating signs per head: dots reach +-8192
    L, H, d = 256, 64, 128
    q = np.full((L, H, d), 8.0)
    q[:, 1::2, :] = -8.0
    kI = np.full((L, d), 8.0)
    kI[1::3] = -8.0
    w = np.full((L, H), 3.0, np.float32)
    qb, kb = gen.encode_e4m3(q), gen.encode_e4m3(kI)
    ref = oracle.index_scores(qb, kb, w)
    got = dsa.index_scores(dev(qb), dev(kb), dev(w)).cpu().numpy().astype(np.float64)
    assert np.array_equal(got, ref)
    assert np.nanmax(ref[np.isfinite(ref)]) == 32 * 3 * 8192


def test_index_topk_tiny_workload_bit_exact():
    cfg = gen.TINY_PREFILL
    inp = gen.prefill_inputs(cfg)
    ref = oracle.index_topk(inp["q_I"], inp["k_I"], inp["w"], cfg.k)
    got = dsa.index_topk(dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"]), cfg.k).cpu().numpy()
    no_device_error()
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("L,k,seed", [(1000, 64, 1), (777, 128, 2), (2600, 2048, 3),
                                      (1500, 1, 4), (513, 300, 5)])
def test_index_topk_64x128_bit_exact(L, k, seed):
    cfg = gen.custom(L=L, H_I=64, d_I=128, k=k, seed=seed)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    ref = oracle.index_topk(q, kI, w, k)
    got = dsa.index_topk(dev(q), dev(kI), dev(w), k).cpu().numpy()
    no_device_error()
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("mode", ["w0", "ties"])
def test_index_topk_ties_bit_exact(mode):
    L, H, d, k = 1200, 64, 128, 100
    cfg = gen.custom(L=L, H_I=H, d_I=d, k=k, seed=9)
    if mode == "w0":
        q, kI = gen.prefill_qI(cfg), gen.prefill_kI(cfg)
        w = np.zeros((L, H), np.float32)
    else:  # values in {-1, 0, 1}, weights in {0, 1}: many equal scores
        q = gen.int_e4m3(cfg.seed_, 1, 0, L * H * d, -1, 1).reshape(L, H, d)
        kI = gen.int_e4m3(cfg.seed_, 2, 0, L * d, -1, 1).reshape(L, d)
        w = gen.int_f32(cfg.seed_, 3, 0, L * H, 0, 1).reshape(L, H)
    ref = oracle.index_topk(q, kI, w, k)
    got = dsa.index_topk(dev(q), dev(kI), dev(w), k).cpu().numpy()
    assert np.array_equal(got, ref)
    if mode == "w0":
        for t in (0, 5, 99, 100, 1199):
            m = min(k, t + 1)
            assert got[t].tolist() == list(range(m)) + [-1] * (k - m)


def test_index_topk_is_deterministic():
    cfg = gen.custom(L=3000, H_I=64, d_I=128, k=512, seed=13)
    q, kI, w = dev(gen.prefill_qI(cfg)), dev(gen.prefill_kI(cfg)), dev(gen.prefill_w(cfg))
    a = dsa.index_topk(q, kI, w, cfg.k)
    b = dsa.index_topk(q, kI, w, cfg.k)
    assert torch.equal(a, b)


# ------------------------------------------------------------------ attention

def test_attention_tiny_workload():
    cfg = gen.TINY_PREFILL
    inp = gen.prefill_inputs(cfg)
    idx = oracle.index_topk(inp["q_I"], inp["k_I"], inp["w"], cfg.k)
    ref = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], idx, cfg.scale)
    O = dsa.sparse_attn_prefill(dev(inp["Q"], torch.bfloat16), dev(inp["K"], torch.bfloat16),
                                dev(inp["V"], torch.bfloat16), dev(idx), cfg.scale)
    no_device_error()
    check_attn(O, ref)


@pytest.mark.parametrize("d,Hkv,G", [(128, 4, 8), (64, 2, 4), (128, 2, 4), (64, 4, 8)])
def test_attention_shapes_with_padding_and_holes(d, Hkv, G):
    L, k = 700, 200
    cfg = gen.custom(L=L, Hq=Hkv * G, Hkv=Hkv, d=d, seed=21 + d + Hkv)
    Q, K, V = gen.prefill_Q(cfg), gen.prefill_K(cfg), gen.prefill_V(cfg)
    rng = np.random.default_rng(5)
    idx = np.full((L, k), -1, np.int32)
    for t in range(L):
        m = min(k, t + 1)
        sel = np.sort(rng.choice(t + 1, m, replace=False)).astype(np.int32)
        if t % 7 == 3:
            sel[rng.integers(0, m)] = -1          # a hole inside the row
        if t % 11 == 5:
            sel = sel[::-1].copy()                # any order is allowed
        idx[t, :m] = sel
    ref = oracle.sparse_attn(Q, K, V, idx, cfg.scale)
    O = dsa.sparse_attn_prefill(dev(Q, torch.bfloat16), dev(K, torch.bfloat16),
                                dev(V, torch.bfloat16), dev(idx), cfg.scale)
    no_device_error()
    check_attn(O, ref)


@pytest.mark.parametrize("d,Hkv,G,L", [(128, 4, 8, 50000), (64, 4, 8, 98400)])
def test_attention_with_keys_beyond_l2(d, Hkv, G, L):
    """K and V above 96 MB: the kernel runs with one producer warp per CTA
    (the smaller cases above run with two); sampled rows against the oracle."""
    k = 64
    cfg = gen.custom(L=L, Hq=Hkv * G, Hkv=Hkv, d=d, seed=31 + d)
    Q, K, V = gen.prefill_Q(cfg), gen.prefill_K(cfg), gen.prefill_V(cfg)
    rng = np.random.default_rng(6)
    idx = np.full((L, k), -1, np.int32)
    for t in range(L):
        m = min(k, t + 1)
        idx[t, :m] = rng.choice(t + 1, m, replace=False).astype(np.int32)
    rows = np.unique(np.concatenate([np.arange(0, 70), np.arange(L - 10, L),
                                     np.linspace(70, L - 11, 50).astype(np.int64)]))
    ref = oracle.sparse_attn(Q, K, V, idx, cfg.scale, rows=rows)
    O = dsa.sparse_attn_prefill(dev(Q, torch.bfloat16), dev(K, torch.bfloat16),
                                dev(V, torch.bfloat16), dev(idx), cfg.scale)
    no_device_error()
    check_attn(O[torch.from_numpy(rows).cuda()], ref)


def test_attention_empty_rows_are_zero_and_out_of_range_is_flagged():
    cfg = gen.custom(L=64, Hq=32, Hkv=4, d=128, seed=31)
    Q, K, V = gen.prefill_Q(cfg), gen.prefill_K(cfg), gen.prefill_V(cfg)
    idx = np.full((64, 32), -1, np.int32)
    idx[10, :3] = [1, 2, 3]
    O = dsa.sparse_attn_prefill(dev(Q, torch.bfloat16), dev(K, torch.bfloat16),
                                dev(V, torch.bfloat16), dev(idx), cfg.scale)
    no_device_error()
    got = bf16_to_f64(O)
    assert np.all(got[0] == 0) and np.all(got[63] == 0)
    ref = oracle.sparse_attn(Q, K, V, idx, cfg.scale, rows=[10])
    assert np.abs(got[10] - ref[0]).max() < MAX_ABS
    idx[20, 0] = 64  # one past the last key
    dsa.sparse_attn_prefill(dev(Q, torch.bfloat16), dev(K, torch.bfloat16),
                            dev(V, torch.bfloat16), dev(idx), cfg.scale)
    assert dsa.device_error() == dsa.DEVERR_INDEX
    no_device_error()


def test_error_words_of_concurrent_calls_are_separate():
    """Two calls on two streams, each with its own device error word: the
    call whose index row holds a key past the end flags DSA_DEVERR_INDEX in
    its own word only; the clean call's word and the library's per-device
    word stay 0."""
    cfg = gen.custom(L=64, Hq=32, Hkv=4, d=128, seed=32)
    Q, K, V = (dev(gen.prefill_Q(cfg), torch.bfloat16), dev(gen.prefill_K(cfg), torch.bfloat16),
               dev(gen.prefill_V(cfg), torch.bfloat16))
    good = np.full((64, 32), -1, np.int32)
    good[:, 0] = np.arange(64)
    bad = good.copy()
    bad[20, 1] = 64  # one past the last key: skipped and flagged
    good_d, bad_d = dev(good), dev(bad)
    e_good, e_bad = dsa.error_word(), dsa.error_word()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for _ in range(3):
        dsa.sparse_attn_prefill(Q, K, V, bad_d, cfg.scale, stream=s1, err=e_bad)
        dsa.sparse_attn_prefill(Q, K, V, good_d, cfg.scale, stream=s2, err=e_good)
    assert dsa.device_error(stream=s2, err=e_good) == dsa.DEVERR_NONE
    assert dsa.device_error(stream=s1, err=e_bad) == dsa.DEVERR_INDEX
    assert dsa.device_error(stream=s1, err=e_bad) == dsa.DEVERR_NONE  # read clears it
    no_device_error()


def test_prefill_end_to_end_tiny_workload():
    cfg = gen.TINY_PREFILL
    inp = gen.prefill_inputs(cfg)
    idx = dsa.index_topk(dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"]), cfg.k)
    O = dsa.sparse_attn_prefill(dev(inp["Q"], torch.bfloat16), dev(inp["K"], torch.bfloat16),
                                dev(inp["V"], torch.bfloat16), idx, cfg.scale)
    rows = np.array([0, 1, 255, 256, 1000, 2047])
    ref_idx = oracle.index_topk(inp["q_I"], inp["k_I"], inp["w"], cfg.k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    ref = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], ref_idx, cfg.scale, rows=rows)
    check_attn(O[torch.from_numpy(rows).cuda()], ref)


# ------------------------------------------------------------------ decode

def _decode_case(lens, seed, k=2048):
    cfg = gen.Config(0, "decode case", "decode", k=k, H_I=64, d_I=128, Hq=32, Hkv=4, d=128,
                     B=len(lens), seed=seed)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = int(off[-1])
    qs = gen.decode_queries(cfg)
    return cfg, off, qs, gen.decode_kI_rows(cfg, 0, N), gen.decode_K_rows(cfg, 0, N), \
        gen.decode_V_rows(cfg, 0, N)


def test_decode_small_batch():
    lens = [1, 5, 2047, 2048, 2049, 5000, 13000, 40001]
    cfg, off, qs, kI, K, V = _decode_case(lens, seed=41)
    ref_idx, ref_O = oracle.decode(qs["q_I"], qs["w"], qs["Q"], kI, K, V, off, cfg.k, cfg.scale)
    idx_out = torch.empty((len(lens), cfg.k), dtype=torch.int32, device="cuda")
    O, _ = dsa.sparse_attn_decode(dev(qs["q_I"]), dev(qs["w"]), dev(qs["Q"], torch.bfloat16),
                                  dev(kI), dev(K, torch.bfloat16), dev(V, torch.bfloat16),
                                  dev(off), cfg.k, cfg.scale, idx_out=idx_out)
    no_device_error()
    assert np.array_equal(idx_out.cpu().numpy(), ref_idx)
    check_attn(O, ref_O)


def test_decode_from_host_buffers():
    """The host-input decode step (queries copied in, outputs copied out, the
    caches resident) gives the device-input decode's index rows and outputs
    bit for bit, and the oracle's rows."""
    lens = [3, 2048, 9000, 40001]
    cfg, off, qs, kI, K, V = _decode_case(lens, seed=43)
    B = len(lens)
    ref_idx, _ = oracle.decode(qs["q_I"], qs["w"], qs["Q"], kI, K, V, off, cfg.k, cfg.scale)
    caches = dict(kI_cache=dev(kI), K_cache=dev(K, torch.bfloat16), V_cache=dev(V, torch.bfloat16))
    d_off = dev(off)
    idx1 = torch.empty((B, cfg.k), dtype=torch.int32, device="cuda")
    O1, _ = dsa.sparse_attn_decode(dev(qs["q_I"]), dev(qs["w"]), dev(qs["Q"], torch.bfloat16),
                                   caches["kI_cache"], caches["K_cache"], caches["V_cache"], d_off,
                                   cfg.k, cfg.scale, idx_out=idx1)
    pin = lambda a, dt=None: (torch.from_numpy(np.ascontiguousarray(a)).view(dt) if dt else  # noqa: E731
                              torch.from_numpy(np.ascontiguousarray(a))).pin_memory()
    host = dict(q_I=pin(qs["q_I"]), w=pin(qs["w"]), Q=pin(qs["Q"].view(np.int16), torch.bfloat16),
                O=torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16).pin_memory(),
                idx=torch.empty((B, cfg.k), dtype=torch.int32).pin_memory())
    need = dsa.decode_workspace_size(B, int(off[-1]), 64, 128, cfg.k, 32, 4, 128)
    devb = dict(q_I=torch.empty((B, 64, 128), dtype=torch.uint8, device="cuda"),
                w=torch.empty((B, 64), dtype=torch.float32, device="cuda"),
                Q=torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda"),
                O=torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda"),
                idx=torch.empty((B, cfg.k), dtype=torch.int32, device="cuda"),
                workspace=torch.empty(need, dtype=torch.uint8, device="cuda"), **caches)
    dsa.decode_from_host(host, devb, d_off, cfg.k, cfg.scale)
    torch.cuda.synchronize()
    no_device_error()
    assert torch.equal(host["idx"], idx1.cpu())
    assert np.array_equal(host["idx"].numpy(), ref_idx)
    assert torch.equal(host["O"], O1.cpu())


def test_decode_equals_prefill_last_row():
    cfg = gen.custom(L=6000, H_I=64, d_I=128, k=2048, Hq=32, Hkv=4, d=128, seed=51)
    inp = gen.prefill_inputs(cfg)
    lens = np.array([1, 700, 2048, 2049, 6000], np.int64)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    t = lens - 1
    kI_c = np.concatenate([inp["k_I"][:n] for n in lens])
    K_c = np.concatenate([inp["K"][:n] for n in lens])
    V_c = np.concatenate([inp["V"][:n] for n in lens])
    idx_p = dsa.index_topk(dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"]), cfg.k)
    O_p = dsa.sparse_attn_prefill(dev(inp["Q"], torch.bfloat16), dev(inp["K"], torch.bfloat16),
                                  dev(inp["V"], torch.bfloat16), idx_p, cfg.scale)
    idx_d = torch.empty((len(lens), cfg.k), dtype=torch.int32, device="cuda")
    O_d, _ = dsa.sparse_attn_decode(dev(inp["q_I"][t]), dev(inp["w"][t]),
                                    dev(inp["Q"][t], torch.bfloat16), dev(kI_c),
                                    dev(K_c, torch.bfloat16), dev(V_c, torch.bfloat16), dev(off),
                                    cfg.k, cfg.scale, idx_out=idx_d)
    tt = torch.from_numpy(t).cuda()
    assert torch.equal(idx_d, idx_p[tt])
    diff = (O_d.float() - O_p[tt].float()).abs()
    assert diff.max().item() <= 2 ** -7  # same keys, split vs one-pass softmax order


def _ascending_case(L, H, d, seed):
    """Indexer inputs whose scores rise with the key index (with ties): q = 1
    everywhere, key s holds a count of +1 entries that grows with s."""
    rng = np.random.default_rng(seed)
    q = np.ones((L, H, d))
    kI = -np.ones((L, d))
    ones = np.minimum((np.arange(L) * d) // L + rng.integers(0, 2, L), d)
    for s in range(L):
        kI[s, :ones[s]] = 1.0
    w = rng.integers(0, 4, (L, H)).astype(np.float32)
    return gen.encode_e4m3(q), gen.encode_e4m3(kI), w


@pytest.mark.parametrize("L,k", [(4000, 256), (5000, 2048), (3001, 64)])
def test_index_topk_ascending_scores_stress(L, k):
    q, kI, w = _ascending_case(L, 64, 128, seed=L + k)
    rows = np.array(sorted({0, k - 1, k, L // 2, L - 2, L - 1} | set(range(0, L, 97))), np.int64)
    ref = oracle.index_topk(q, kI, w, k, rows=rows)
    got = dsa.index_topk(dev(q), dev(kI), dev(w), k).cpu().numpy()[rows]
    no_device_error()
    assert np.array_equal(got, ref)


def test_decode_ascending_scores_stress():
    L = 70000
    q, kI, w = _ascending_case(L, 64, 128, seed=3)
    lens = np.array([L, 30000, 5], np.int64)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    kI_c = np.concatenate([kI[:n] for n in lens])
    cfg = gen.Config(0, "stress", "decode", k=2048, H_I=64, d_I=128, Hq=32, Hkv=4, d=128, B=3,
                     seed=5)
    Q = gen.normal_bf16(5, 4, 0, 3 * 32 * 128).reshape(3, 32, 128)
    N = int(off[-1])
    K = gen.normal_bf16(5, 5, 0, N * 512).reshape(N, 4, 128)
    V = gen.normal_bf16(5, 6, 0, N * 512).reshape(N, 4, 128)
    qd, wd = q[lens - 1], w[lens - 1]
    r_idx, r_O = oracle.decode(qd, wd, Q, kI_c, K, V, off, cfg.k, cfg.scale)
    idx = torch.empty((3, cfg.k), dtype=torch.int32, device="cuda")
    O, _ = dsa.sparse_attn_decode(dev(qd), dev(wd), dev(Q, torch.bfloat16), dev(kI_c),
                                  dev(K, torch.bfloat16), dev(V, torch.bfloat16), dev(off), cfg.k,
                                  cfg.scale, idx_out=idx)
    no_device_error()
    assert np.array_equal(idx.cpu().numpy(), r_idx)
    check_attn(O, r_O)
