"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (the same C-ABI calls on the same shapes).

Every row is checked for the properties that hold at any size (count =
min(k, t+1), ascending, inside [0, t], padding last); sampled rows, which
the oracle computes one by one, are compared bit-exactly (index sets) and
within max-abs 2e-2 / mean-abs 2e-3 (attention outputs)."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sparse_long_context_02_b200 as dsa

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def dev(a, dt=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dt) if dt is not None else t).cuda()


def check_rows_valid(idx: torch.Tensor, n_visible: torch.Tensor, k: int):
    """idx [R][k] on the GPU; n_visible [R] = number of visible keys per row."""
    valid = idx >= 0
    cnt = valid.sum(1)
    assert torch.equal(cnt, torch.clamp(n_visible, max=k).to(cnt.dtype))
    assert not (valid[:, 1:] & ~valid[:, :-1]).any(), "padding must come last"
    both = valid[:, 1:] & valid[:, :-1]
    assert bool(((idx[:, 1:] > idx[:, :-1]) | ~both).all()), "rows must ascend"
    assert bool(((idx < n_visible[:, None]) | ~valid).all()), "keys must be visible"


def sample_rows(L, k, n=16, seed=0, extra=()):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, k - 2, k - 1, k, k + 1, L - 1]
    strat = [int((i + rng.random()) * L / n) for i in range(n)]
    return np.array(sorted(set(r for r in fixed + strat + list(extra) if 0 <= r < L)), np.int64)


@pytest.mark.parametrize("cfg", [gen.PREFILL_32K, gen.PREFILL_128K, gen.VIDEO_256K],
                         ids=lambda c: c.name)
def test_prefill_full_size(cfg):
    host = gen.prefill_inputs(cfg)
    idx = dsa.index_topk(dev(host["q_I"]), dev(host["k_I"]), dev(host["w"]), cfg.k)
    O = dsa.sparse_attn_prefill(dev(host["Q"], torch.bfloat16), dev(host["K"], torch.bfloat16),
                                dev(host["V"], torch.bfloat16), idx, cfg.scale)
    assert dsa.device_error() == dsa.DEVERR_NONE
    t = torch.arange(cfg.L, device="cuda")
    check_rows_valid(idx, t + 1, cfg.k)
    extra = ()
    if cfg.video:
        ft = cfg.frame_text + cfg.frame_vision
        extra = [f * ft + o for f in (1, 117, 239) for o in (0, 15, 16, ft - 1)]
    rows = sample_rows(cfg.L, cfg.k, seed=cfg.id, extra=extra)
    ref_idx = oracle.index_topk(host["q_I"], host["k_I"], host["w"], cfg.k, rows=rows)
    got_idx = idx[torch.from_numpy(rows).cuda()].cpu().numpy()
    bad = [int(r) for r, a, b in zip(rows, got_idx, ref_idx) if not np.array_equal(a, b)]
    assert not bad, f"index rows differ from the oracle: {bad}"
    ref_O = oracle.sparse_attn(host["Q"], host["K"], host["V"], ref_idx, cfg.scale, rows=rows,
                               idx_by_row=True)
    got_O = O[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    err = np.abs(got_O - ref_O)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert torch.isfinite(O.float()).all()


def test_decode_full_size():
    cfg = gen.DECODE_B64
    off = gen.decode_offsets(cfg)
    lens = np.diff(off)
    N = int(off[-1])
    q = gen.decode_queries(cfg)
    kI = torch.empty((N, cfg.d_I), dtype=torch.uint8, device="cuda")
    K = torch.empty((N, cfg.Hkv, cfg.d), dtype=torch.bfloat16, device="cuda")
    V = torch.empty((N, cfg.Hkv, cfg.d), dtype=torch.bfloat16, device="cuda")
    step = 1 << 19
    for r0 in range(0, N, step):
        r1 = min(N, r0 + step)
        kI[r0:r1].copy_(torch.from_numpy(gen.decode_kI_rows(cfg, r0, r1)))
        K[r0:r1].copy_(torch.from_numpy(gen.decode_K_rows(cfg, r0, r1).view(np.int16)).view(
            torch.bfloat16))
        V[r0:r1].copy_(torch.from_numpy(gen.decode_V_rows(cfg, r0, r1).view(np.int16)).view(
            torch.bfloat16))
    idx = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device="cuda")
    O, _ = dsa.sparse_attn_decode(dev(q["q_I"]), dev(q["w"]), dev(q["Q"], torch.bfloat16), kI, K,
                                  V, dev(off), cfg.k, cfg.scale, idx_out=idx)
    assert dsa.device_error() == dsa.DEVERR_NONE
    check_rows_valid(idx, torch.from_numpy(lens).cuda(), cfg.k)
    # oracle on four sequences: the shortest, the longest and two others
    seqs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 7, 40})
    sub_lens = lens[seqs]
    sub_off = np.concatenate([[0], np.cumsum(sub_lens)]).astype(np.int64)
    kI_h = np.concatenate([gen.decode_kI_rows(cfg, off[b], off[b + 1]) for b in seqs])
    K_h = np.concatenate([gen.decode_K_rows(cfg, off[b], off[b + 1]) for b in seqs])
    V_h = np.concatenate([gen.decode_V_rows(cfg, off[b], off[b + 1]) for b in seqs])
    r_idx, r_O = oracle.decode(q["q_I"][seqs], q["w"][seqs], q["Q"][seqs], kI_h, K_h, V_h, sub_off,
                               cfg.k, cfg.scale)
    assert np.array_equal(idx.cpu().numpy()[seqs], r_idx)
    err = np.abs(O.float().cpu().numpy()[seqs] - r_O)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
