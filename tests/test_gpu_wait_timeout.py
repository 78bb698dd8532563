"""The bounded waits every kernel relies on (an mbarrier wait that gives up
after 2 s of %globaltimer, records DSA_DEVERR_TIMEOUT in the call's error
word and lets the kernel finish) exercised on the GPU: a test kernel waits
on a barrier that nothing arrives at.  The host reads the status and the
context stays usable for the next call.  No fault, trap or unbounded wait is
involved (the benchmark's probe library holds the test kernel)."""
import ctypes

import numpy as np
import pytest
import torch

import gen
import oracle
import sparse_long_context_02_b200 as dsa
from sparse_long_context_02_b200 import build as dsa_build

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_records_the_timeout_and_the_context_survives():
    L = ctypes.CDLL(dsa_build.build_probe())
    L.dsa_probe_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream()
    assert L.dsa_probe_wait_timeout(err.data_ptr(), st.cuda_stream) == 0
    torch.cuda.synchronize()
    assert int(err.item()) == dsa.DEVERR_TIMEOUT
    # the next call on the same context runs and is exact
    cfg = gen.custom(L=300, H_I=4, d_I=64, k=32, seed=91)
    h = gen.prefill_inputs(cfg)
    idx = dsa.index_topk(torch.from_numpy(h["q_I"]).cuda(), torch.from_numpy(h["k_I"]).cuda(),
                         torch.from_numpy(h["w"]).cuda(), cfg.k)
    ref = oracle.index_topk(h["q_I"], h["k_I"], h["w"], cfg.k)
    assert np.array_equal(idx.cpu().numpy(), ref)
    assert dsa.device_error() == dsa.DEVERR_NONE
