"""Indexer warm-up KL loss (dsa_indexer_kl_forward / _backward) against the
float64 oracle in oracle/kl.py, on the generator's integer-valued e4m3
indexer inputs (so S = q_I . k_I is exact on both sides and the ReLU's
[S > 0] decisions agree) and N(0, 1) bf16 attention inputs.

Tolerances, from the arithmetic:
* kl and G: fp32 logits and exponentials (ex2/lg2 approximations, relative
  error ~1e-7 each) -> |dkl| <= 1e-4 (1 + |kl|), |dG| <= 1e-5 scale_I.
* dw: fp32 products of exact S with G, fp32 sums -> 1e-5 of max |dw|.
* dq_I, dk_I: dS = G w [S > 0] is rounded to bf16 (relative 2^-9) before
  its product with the exact e4m3 values; every term's error is at most
  2^-9 |dS| |x|, so |d dq[t,j,:]| <= 2^-8 w[t,j] sum_s |G[t,s]| max|k_I| and
  |d dk[s,:]| <= 2^-8 sum_t |G[t,s]| sum_j w[t,j] max|q_I| (a factor 2 over
  the rounding for the fp32 sums), plus a 1 % bound on the relative
  Frobenius error.
The backward is checked on the oracle's own G (rounded to fp32) so that its
arithmetic is measured alone; the chained forward -> backward is checked on
the Frobenius bound."""
import numpy as np
import pytest
import torch

import gen
import oracle.kl as KL
import sparse_long_context_02_b200 as dsa

pytestmark = pytest.mark.gpu


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


CASES = [
    # L spanning several 64-row tiles with a ragged tail; full heads
    dict(L=700, H_I=64, d_I=128, Hq=32, Hkv=4, d=128, scale_I=1.0 / 2048, seed=41),
    # small heads
    dict(L=1000, H_I=4, d_I=64, Hq=8, Hkv=2, d=64, scale_I=1.0 / 128, seed=42),
    # L % 8 == 0 (32-byte G row loads in the tensor-core dq kernel), ragged 128-row tail
    dict(L=1032, H_I=64, d_I=128, Hq=32, Hkv=4, d=128, scale_I=1.0 / 2048, seed=45),
    # Hkv = 8 (the mma.sync forward), H_I = 4 with d_I = 128 (tensor-core dq/dk,
    # one head per dk group)
    dict(L=300, H_I=4, d_I=128, Hq=16, Hkv=8, d=128, scale_I=1.0 / 512, seed=46),
    # Hkv = 2 on the tensor-core forward, d_I = 64 backward
    dict(L=450, H_I=64, d_I=64, Hq=8, Hkv=2, d=128, scale_I=1.0 / 1024, seed=47),
    # exactly one tile, and one row
    dict(L=64, H_I=64, d_I=128, Hq=32, Hkv=4, d=128, scale_I=1.0 / 2048, seed=43),
    dict(L=1, H_I=4, d_I=64, Hq=8, Hkv=2, d=64, scale_I=1.0 / 128, seed=44),
]


def _inputs(c):
    cfg = gen.custom(L=c["L"], H_I=c["H_I"], d_I=c["d_I"], k=8, Hq=c["Hq"], Hkv=c["Hkv"],
                     d=c["d"], seed=c["seed"])
    return cfg, gen.prefill_inputs(cfg)


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"L{c['L']}_HI{c['H_I']}_d{c['d']}")
def test_kl_forward_and_backward_match_oracle(c):
    cfg, inp = _inputs(c)
    sI = c["scale_I"]
    ref = KL.indexer_kl(inp["q_I"], inp["k_I"], inp["w"], inp["Q"], inp["K"], cfg.scale, sI)
    q, kI, w = dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"])
    Q, K = dev(inp["Q"], torch.bfloat16), dev(inp["K"], torch.bfloat16)

    kl, G = dsa.indexer_kl_forward(q, kI, w, Q, K, cfg.scale, sI)
    kl_g = kl.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(kl_g - ref["kl"]) <= 1e-4 * (1 + np.abs(ref["kl"]))), \
        np.abs(kl_g - ref["kl"]).max()
    G_g = G.cpu().numpy().astype(np.float64)
    assert np.abs(G_g - ref["G"]).max() <= 1e-5 * sI, np.abs(G_g - ref["G"]).max()

    # backward on the oracle's G
    dq, dk, dw = dsa.indexer_kl_backward(q, kI, w, dev(ref["G"].astype(np.float32)))
    assert dsa.device_error() == dsa.DEVERR_NONE
    dq, dk, dw = (x.cpu().numpy().astype(np.float64) for x in (dq, dk, dw))
    assert np.abs(dw - ref["dw"]).max() <= 1e-5 * max(np.abs(ref["dw"]).max(), 1e-30)
    aG = np.abs(ref["G"])
    wf = inp["w"].astype(np.float64)
    qmax = np.abs(KL.decode_e4m3(inp["q_I"])).max()
    kmax = np.abs(KL.decode_e4m3(inp["k_I"])).max()
    bound_dq = 2.0 ** -8 * wf * aG.sum(axis=1)[:, None] * kmax                 # [L][H_I]
    bound_dk = 2.0 ** -8 * (aG * wf.sum(axis=1)[:, None]).sum(axis=0) * qmax  # [L]
    assert np.all(np.abs(dq - ref["dq_I"]) <= bound_dq[:, :, None] + 1e-12)
    assert np.all(np.abs(dk - ref["dk_I"]) <= bound_dk[:, None] + 1e-12)
    for got, r in ((dq, ref["dq_I"]), (dk, ref["dk_I"])):
        n = np.linalg.norm(r)
        assert np.linalg.norm(got - r) <= 1e-2 * n + 1e-12

    # chained: the GPU's own G into the GPU backward
    dq2, dk2, dw2 = (x.cpu().numpy().astype(np.float64) for x in dsa.indexer_kl_backward(q, kI, w, G))
    for got, r in ((dq2, ref["dq_I"]), (dk2, ref["dk_I"]), (dw2, ref["dw"])):
        assert np.linalg.norm(got - r) <= 1e-2 * np.linalg.norm(r) + 1e-12


def test_kl_is_bit_identical_run_to_run():
    cfg, inp = _inputs(CASES[0])
    q, kI, w = dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"])
    Q, K = dev(inp["Q"], torch.bfloat16), dev(inp["K"], torch.bfloat16)
    a = dsa.indexer_kl_forward(q, kI, w, Q, K, cfg.scale, 1.0 / 2048)
    b = dsa.indexer_kl_forward(q, kI, w, Q, K, cfg.scale, 1.0 / 2048)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    ga = dsa.indexer_kl_backward(q, kI, w, a[1])
    gb = dsa.indexer_kl_backward(q, kI, w, b[1])
    assert all(torch.equal(x, y) for x, y in zip(ga, gb))


def test_kl_rejects_bad_arguments():
    cfg, inp = _inputs(CASES[3])
    q, kI, w = dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"])
    Q, K = dev(inp["Q"], torch.bfloat16), dev(inp["K"], torch.bfloat16)
    with pytest.raises(dsa.DSAError):  # Hq not a multiple of Hkv
        dsa.indexer_kl_forward(q, kI, w, Q[:, :7].contiguous(), K, cfg.scale, 1.0)
    with pytest.raises(dsa.DSAError):  # workspace too small
        dsa.indexer_kl_forward(q, kI, w, Q, K, cfg.scale, 1.0,
                               workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
    cfg2, inp2 = _inputs(CASES[0])
    q2, k2, w2 = dev(inp2["q_I"]), dev(inp2["k_I"]), dev(inp2["w"])
    G2 = torch.zeros((cfg2.L, cfg2.L), dtype=torch.float32, device="cuda")
    with pytest.raises(dsa.DSAError):  # backward workspace too small (8 head groups here)
        dsa.indexer_kl_backward(q2, k2, w2, G2,
                                workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
