"""GPU parity of the sparse attention backward (dsa_sparse_attn_backward)
and of the forward's log-sum-exp output, through the C ABI, against the
float64 oracle (oracle/attn_bwd.py, pinned by finite differences and
autograd in tests/test_oracle_attn_bwd.py).

Tolerance, derived from what the kernel rounds: dS and P are rounded to bf16
for their products (relative 2^-9 each), D = dO . O uses the bf16 forward
output (an error of 2^-9 sum |dO| |O|), and everything else is fp32.  Each
output element must lie within 2^-7 of the oracle's magnitude of its terms
(sum of |dS| |K| for dQ, and so on; a margin of 4 over the rounding), plus
1e-5 for fp32 accumulation, and the Frobenius error must stay under 1 %.

Source: Kwai Keye-VL-2.0 technical-report summary, section 1 (sparse
adaptation: training through the truly sparse attention)."""
import numpy as np
import pytest
import torch

import gen
import oracle.attn_bwd as AB
import sparse_long_context_02_b200 as dsa

pytestmark = pytest.mark.gpu


def dev(a, dt=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dt) if dt is not None else t).cuda()


def _rows(L, k, seed, holes=True):
    rng = np.random.default_rng(seed)
    idx = np.full((L, k), -1, np.int32)
    for t in range(L):
        m = min(k, t + 1)
        sel = rng.choice(t + 1, m, replace=False).astype(np.int32)
        if holes and t % 7 == 3:
            sel[rng.integers(0, m)] = -1         # a hole inside the row
        if holes and t % 11 == 5 and m > 1:
            sel[1] = sel[0]                      # a key listed twice counts twice
        idx[t, :m] = sel
    if holes:
        idx[L // 2, :] = -1                       # an empty row
    return idx


def _run(cfg, idx, seed):
    Qb, Kb, Vb = gen.prefill_Q(cfg), gen.prefill_K(cfg), gen.prefill_V(cfg)
    rng = np.random.default_rng(seed)
    dOb = gen.encode_bf16(rng.normal(size=Qb.shape))
    Q, K, V, dO = (dev(a, torch.bfloat16) for a in (Qb, Kb, Vb, dOb))
    idx_d = dev(idx)
    lse = torch.empty((cfg.L, cfg.Hq), dtype=torch.float32, device="cuda")
    O = dsa.sparse_attn_prefill(Q, K, V, idx_d, cfg.scale, lse=lse)
    dQ, dK, dV = dsa.sparse_attn_backward(Q, K, V, idx_d, O, lse, dO, cfg.scale)
    assert dsa.device_error() == dsa.DEVERR_NONE
    f64 = [AB.decode_bf16(a) for a in (Qb, Kb, Vb, dOb)]
    ref = AB.backward(*f64[:3], idx, f64[3], cfg.scale, magnitudes=True)
    ref_lse = AB.lse(f64[0], f64[1], idx, cfg.scale)
    return dict(dQ=dQ, dK=dK, dV=dV, lse=lse), ref, ref_lse


def _check(got, ref, ref_lse):
    lse = got["lse"].cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.abs(lse[fin] - ref_lse[fin]).max() <= 1e-4
    for n, m in (("dQ", "mQ"), ("dK", "mK"), ("dV", "mV")):
        g = got[n].cpu().numpy().astype(np.float64)
        err = np.abs(g - ref[n])
        bound = 2.0 ** -7 * ref[m] + 1e-5
        worst = np.unravel_index(np.argmax(err - bound), err.shape)
        assert np.all(err <= bound), (n, worst, g[worst], ref[n][worst], ref[m][worst])
        assert np.linalg.norm(g - ref[n]) <= 1e-2 * np.linalg.norm(ref[n]) + 1e-6, n


@pytest.mark.parametrize("d,Hkv,G", [(128, 4, 8), (64, 2, 4), (128, 2, 4), (64, 4, 8)])
def test_backward_shapes_with_holes_repeats_and_empty_rows(d, Hkv, G):
    cfg = gen.custom(L=300, Hq=Hkv * G, Hkv=Hkv, d=d, k=40, seed=61 + d + Hkv)
    idx = _rows(cfg.L, cfg.k, seed=d + G)
    got, ref, ref_lse = _run(cfg, idx, seed=1)
    _check(got, ref, ref_lse)


def test_backward_dense_rows_equal_dense_attention_gradient():
    """k >= t + 1 for every row: the sparse attention is the dense causal one
    (the oracle's own pin against autograd), over several 16-key chunks with
    a ragged last chunk."""
    cfg = gen.custom(L=150, Hq=32, Hkv=4, d=128, k=150, seed=62)
    idx = np.full((cfg.L, cfg.k), -1, np.int32)
    for t in range(cfg.L):
        idx[t, :t + 1] = np.arange(t + 1)
    got, ref, ref_lse = _run(cfg, idx, seed=2)
    _check(got, ref, ref_lse)


def test_backward_at_the_prefill_shape_k2048():
    """The prefill workloads' shapes (32/4 heads, d = 128, k = 2048) on a
    short sequence whose late rows hold the full 2048 keys, in random order."""
    cfg = gen.custom(L=2600, Hq=32, Hkv=4, d=128, k=2048, seed=63)
    idx = _rows(cfg.L, cfg.k, seed=9, holes=False)
    got, ref, ref_lse = _run(cfg, idx, seed=3)
    _check(got, ref, ref_lse)


def test_backward_out_of_range_entry_is_skipped_and_flagged():
    cfg = gen.custom(L=64, Hq=32, Hkv=4, d=128, k=8, seed=64)
    idx = _rows(cfg.L, cfg.k, seed=4, holes=False)
    Qb, Kb, Vb = gen.prefill_Q(cfg), gen.prefill_K(cfg), gen.prefill_V(cfg)
    Q, K, V = (dev(a, torch.bfloat16) for a in (Qb, Kb, Vb))
    lse = torch.empty((cfg.L, cfg.Hq), dtype=torch.float32, device="cuda")
    O = dsa.sparse_attn_prefill(Q, K, V, dev(idx), cfg.scale, lse=lse)
    assert dsa.device_error() == dsa.DEVERR_NONE
    bad = idx.copy()
    bad[40, 3] = cfg.L + 100
    err = dsa.error_word()
    dQ, dK, dV = dsa.sparse_attn_backward(Q, K, V, dev(bad), O, lse, torch.ones_like(Q),
                                          cfg.scale, err=err)
    assert dsa.device_error(err=err) == dsa.DEVERR_INDEX
    for t_ in (dQ, dK, dV):
        assert torch.isfinite(t_).all()
