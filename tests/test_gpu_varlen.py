"""Packed variable-length prefill (dsa_index_topk_varlen) against the oracle
run sequence by sequence: every sequence restarts the causal mask, so its
index rows must equal the single-sequence oracle's on its own rows, shifted
to packed positions.  Integer-valued inputs keep the comparison bit-exact;
the attention runs unchanged on the packed rows."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sparse_long_context_02_b200 as dsa

pytestmark = pytest.mark.gpu


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def packed_reference(q, kI, w, cu, k):
    """Oracle per sequence, keys shifted to packed positions."""
    ref = np.full((q.shape[0], k), -1, dtype=np.int32)
    for b in range(len(cu) - 1):
        lo, hi = int(cu[b]), int(cu[b + 1])
        r = oracle.index_topk(q[lo:hi], kI[lo:hi], w[lo:hi], k)
        ref[lo:hi] = np.where(r >= 0, r + lo, -1)
    return ref


# boundaries off the 4-token blocks and the 128-key tiles; a one-token
# sequence; a sequence shorter than k and one longer
LENS = [700, 1, 1300, 129, 2100, 3]


@pytest.mark.parametrize("k", [64, 256, 2048])
def test_index_topk_varlen_bit_exact(k):
    cu = np.concatenate([[0], np.cumsum(LENS)]).astype(np.int32)
    cfg = gen.custom(L=int(cu[-1]), H_I=64, d_I=128, k=k, seed=11)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    got = dsa.index_topk_varlen(dev(q), dev(kI), dev(w), dev(cu), k).cpu().numpy()
    assert dsa.device_error() == dsa.DEVERR_NONE
    assert np.array_equal(got, packed_reference(q, kI, w, cu, k))


def test_index_topk_varlen_one_sequence_equals_plain():
    cfg = gen.custom(L=1500, H_I=64, d_I=128, k=256, seed=12)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    cu = np.array([0, cfg.L], dtype=np.int32)
    a = dsa.index_topk_varlen(dev(q), dev(kI), dev(w), dev(cu), cfg.k).cpu().numpy()
    b = dsa.index_topk(dev(q), dev(kI), dev(w), cfg.k).cpu().numpy()
    assert np.array_equal(a, b)


def test_varlen_prefill_end_to_end_small_heads():
    lens = [300, 517, 5, 1200]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cfg = gen.custom(L=int(cu[-1]), H_I=4, d_I=64, k=256, Hq=8, Hkv=2, d=64, seed=13)
    inp = gen.prefill_inputs(cfg)
    idx = dsa.index_topk_varlen(dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"]), dev(cu), cfg.k)
    ref_idx = packed_reference(inp["q_I"], inp["k_I"], inp["w"], cu, cfg.k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    O = dsa.sparse_attn_prefill(dev(inp["Q"], torch.bfloat16), dev(inp["K"], torch.bfloat16),
                                dev(inp["V"], torch.bfloat16), idx, cfg.scale)
    rows = np.array([0, 299, 300, 301, 816, 817, 821, 822, 2021])
    ref = oracle.sparse_attn(inp["Q"], inp["K"], inp["V"], ref_idx, cfg.scale, rows=rows)
    got = O[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    assert dsa.device_error() == dsa.DEVERR_NONE


def test_index_topk_varlen_flags_bad_ends():
    cfg = gen.custom(L=600, H_I=64, d_I=128, k=64, seed=14)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    cu = np.array([0, 300, 599], dtype=np.int32)  # does not end at L
    dsa.index_topk_varlen(dev(q), dev(kI), dev(w), dev(cu), cfg.k)
    assert dsa.device_error() == dsa.DEVERR_INDEX
    assert dsa.device_error() == dsa.DEVERR_NONE  # read and cleared


def test_prefill_from_host_matches_device_path():
    """The chunked host-to-device prefill computes exactly what the device
    calls compute (same kernels on the same rows), with a ragged last chunk."""
    cfg = gen.custom(L=3000, H_I=64, d_I=128, k=256, Hq=32, Hkv=4, d=128, seed=15)
    inp = gen.prefill_inputs(cfg)
    host = {"q_I": torch.from_numpy(inp["q_I"]).pin_memory(),
            "k_I": torch.from_numpy(inp["k_I"]).pin_memory(),
            "w": torch.from_numpy(inp["w"]).pin_memory(),
            "Q": torch.from_numpy(inp["Q"].view(np.int16)).view(torch.bfloat16).pin_memory(),
            "K": torch.from_numpy(inp["K"].view(np.int16)).view(torch.bfloat16).pin_memory(),
            "V": torch.from_numpy(inp["V"].view(np.int16)).view(torch.bfloat16).pin_memory()}
    host["O"] = torch.empty_like(host["Q"]).pin_memory()
    devb = {n: torch.empty_like(host[n], device="cuda") for n in ("q_I", "k_I", "w", "Q", "K", "V", "O")}
    devb["idx"] = torch.empty((cfg.L, cfg.k), dtype=torch.int32, device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    dsa.prefill_from_host(host, devb, cfg.k, cfg.scale, chunk_rows=1000, h2d_stream=s1,
                          d2h_stream=s2)
    torch.cuda.synchronize()
    idx = dsa.index_topk(dev(inp["q_I"]), dev(inp["k_I"]), dev(inp["w"]), cfg.k)
    O = dsa.sparse_attn_prefill(dev(inp["Q"], torch.bfloat16), dev(inp["K"], torch.bfloat16),
                                dev(inp["V"], torch.bfloat16), idx, cfg.scale)
    assert torch.equal(devb["idx"], idx)
    assert torch.equal(host["O"], O.cpu())
    assert dsa.device_error() == dsa.DEVERR_NONE
