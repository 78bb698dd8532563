"""The allocation-free decode entry point against the workspace one.

dsa_sparse_attn_decode_noalloc serves callers that cannot allocate device
memory at call time (a host framework that owns all device memory, a decode
loop that must not call cudaMalloc); its scratch is a fixed array inside the
library.  This test calls it through the C ABI twice in a row, on two
different batches, and checks each result against dsa_sparse_attn_decode with
a caller workspace: index rows identical, outputs within the attention
tolerance.  It lives in a file of its own that is collected last."""
import numpy as np
import pytest
import torch

import gen
import sparse_long_context_02_b200 as dsa

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _case(lens, seed):
    cfg = gen.Config(0, "no-alloc decode", "decode", k=2048, H_I=64, d_I=128, Hq=32, Hkv=4, d=128,
                     B=len(lens), seed=seed)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = int(off[-1])
    q = gen.decode_queries(cfg)

    def dev(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(dt) if dt is not None else t).cuda()

    args = (dev(q["q_I"]), dev(q["w"]), dev(q["Q"], torch.bfloat16),
            dev(gen.decode_kI_rows(cfg, 0, N)), dev(gen.decode_K_rows(cfg, 0, N), torch.bfloat16),
            dev(gen.decode_V_rows(cfg, 0, N), torch.bfloat16), dev(off))
    return cfg, args


@pytest.mark.parametrize("calls", [[[3, 2048, 9000, 30001], 1], [[70000, 5, 2049], 2]])
def test_noalloc_decode_matches_workspace_decode(calls):
    lens, seed = calls
    cfg, args = _case(lens, seed)
    B = len(lens)
    ref_idx = torch.empty((B, cfg.k), dtype=torch.int32, device="cuda")
    ref_O, _ = dsa.sparse_attn_decode(*args, cfg.k, cfg.scale, idx_out=ref_idx)
    for _ in range(2):  # two calls in a row share the library's scratch
        idx = torch.full((B, cfg.k), -7, dtype=torch.int32, device="cuda")
        O, _ = dsa.sparse_attn_decode_noalloc(*args, cfg.k, cfg.scale, idx_out=idx)
        torch.cuda.synchronize()
        assert dsa.device_error() == dsa.DEVERR_NONE
        assert torch.equal(idx, ref_idx)
        err = (O.float() - ref_O.float()).abs()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS


def test_noalloc_decode_without_index_output_and_changing_shapes():
    """Calls whose index rows stay inside the shared scratch (idx_out None),
    back to back with calls of another batch and another k: stale counts or
    rows left by the previous call would show up as a difference from the
    workspace decode."""
    plan = [([40000, 7, 2048, 12345, 3], 3, 2048, False),
            ([9000, 300000], 4, 512, True),
            ([40000, 7, 2048, 12345, 3], 3, 2048, True),
            ([65, 64, 63], 5, 64, False)]
    for lens, seed, k, with_idx in plan:
        cfg, args = _case(lens, seed)
        B = len(lens)
        ref_idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
        ref_O, _ = dsa.sparse_attn_decode(*args, k, cfg.scale, idx_out=ref_idx)
        idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda") if with_idx else None
        O, _ = dsa.sparse_attn_decode_noalloc(*args, k, cfg.scale, idx_out=idx)
        torch.cuda.synchronize()
        assert dsa.device_error() == dsa.DEVERR_NONE
        if with_idx:
            assert torch.equal(idx, ref_idx)
        err = (O.float() - ref_O.float()).abs()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (lens, k)


def test_noalloc_decode_rejects_sizes_beyond_its_scratch():
    L = dsa.lib()
    need = L.dsa_decode_workspace_size(4096, 1 << 30, 64, 128, 2048, 32, 4, 128)
    assert need > 64 << 20
    fake = 0x10000
    st = L.dsa_sparse_attn_decode_noalloc(fake, fake, fake, fake, fake, fake, fake, 4096, 1 << 30,
                                          64, 128, 32, 4, 128, 2048, 0.088, fake, None, None,
                                          None)
    assert st == 3  # DSA_ERR_WORKSPACE, before any launch
    assert b"built-in array" in L.dsa_last_error()
