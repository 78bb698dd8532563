"""Host-side checks of the C ABI (no GPU needed): the library builds and
loads, exports every entry point include/dsa.h declares, and rejects bad
arguments with a status before it touches the device."""
import ctypes
import os
import re
import subprocess

import pytest

import sparse_long_context_02_b200 as dsa
from sparse_long_context_02_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")

INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3


@pytest.fixture(scope="module")
def L():
    dsa_build.build()
    return dsa.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("dsa_index_topk", "dsa_sparse_attn_prefill", "dsa_sparse_attn_decode",
                 "dsa_index_scores", "dsa_decode_workspace_size", "dsa_check_device_error",
                 "dsa_last_error", "dsa_status_string", "dsa_version"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)


def test_status_strings_and_version(L):
    assert L.dsa_version() >= 100
    assert L.dsa_status_string(0) == b"DSA_OK"
    assert L.dsa_status_string(3) == b"DSA_ERR_WORKSPACE"
    assert L.dsa_status_string(99) == b"DSA_ERR_UNKNOWN"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation


def test_index_topk_rejects_bad_arguments(L):
    f = L.dsa_index_topk
    assert f(None, FAKE, FAKE, 64, 4, 64, 8, FAKE, None, None) == INVALID
    assert b"q_I is NULL" in L.dsa_last_error()
    assert f(FAKE + 4, FAKE, FAKE, 64, 4, 64, 8, FAKE, None, None) == INVALID
    assert b"aligned" in L.dsa_last_error()
    assert f(FAKE, FAKE, FAKE, 0, 4, 64, 8, FAKE, None, None) == INVALID
    assert f(FAKE, FAKE, FAKE, 64, 4, 64, 0, FAKE, None, None) == INVALID
    assert f(FAKE, FAKE, FAKE, 64, 4, 64, 4096, FAKE, None, None) == UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 64, 8, 64, 8, FAKE, None, None) == UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 64, 64, 96, 8, FAKE, None, None) == UNSUPPORTED


def test_index_scores_rejects_bad_arguments(L):
    f = L.dsa_index_scores
    assert f(FAKE, FAKE, None, 64, 4, 64, FAKE, None, None) == INVALID
    assert f(FAKE, FAKE, FAKE, 1 << 16, 4, 64, FAKE, None, None) == INVALID
    assert f(FAKE, FAKE, FAKE, 64, 16, 64, FAKE, None, None) == UNSUPPORTED


def test_prefill_attention_rejects_bad_arguments(L):
    f = L.dsa_sparse_attn_prefill
    sc = ctypes.c_float(0.125)
    assert f(FAKE, FAKE, FAKE, None, 64, 8, 2, 64, 16, sc, FAKE, None, None, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, 64, 8, 3, 64, 16, sc, FAKE, None, None, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, 64, 8, 2, 64, 16, ctypes.c_float(-1.0), FAKE, None, None, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, 64, 8, 2, 96, 16, sc, FAKE, None, None, None) == UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, 64, 16, 1, 64, 16, sc, FAKE, None, None, None) == UNSUPPORTED


def test_decode_from_host_rejects_bad_arguments(L):
    f = L.dsa_decode_from_host
    sc = ctypes.c_float(0.088)
    args = [FAKE] * 12 + [4, 40000, 64, 128, 32, 4, 128, 2048, sc, FAKE, FAKE, FAKE, 1 << 30,
                          None, None]
    bad = list(args)
    bad[0] = None  # q_I_host
    assert f(*bad) == INVALID
    bad = list(args)
    bad[22] = None  # idx_out NULL while idx_host is given
    assert f(*bad) == INVALID
    assert b"idx_host needs idx_out" in L.dsa_last_error()
    bad = list(args)
    bad[16] = 16  # Hq
    assert f(*bad) == UNSUPPORTED
    bad = list(args)
    bad[24] = 100  # workspace too small
    assert f(*bad) == WORKSPACE


def test_attention_backward_rejects_bad_arguments(L):
    f = L.dsa_sparse_attn_backward
    sc = ctypes.c_float(0.125)
    args = [FAKE] * 7 + [64, 8, 2, 64, 16, sc, FAKE, FAKE, FAKE, None, None]
    bad = list(args)
    bad[5] = None  # lse
    assert f(*bad) == INVALID
    assert b"lse is NULL" in L.dsa_last_error()
    bad = list(args)
    bad[9] = 3  # Hkv does not divide Hq
    assert f(*bad) == INVALID
    bad = list(args)
    bad[10] = 96  # d
    assert f(*bad) == UNSUPPORTED
    bad = list(args)
    bad[12] = ctypes.c_float(0.0)
    assert f(*bad) == INVALID
    assert f(*(args[:7] + [64, 16, 1, 64, 16, sc] + args[13:])) == UNSUPPORTED


def test_decode_rejects_bad_arguments_and_small_workspace(L):
    f = L.dsa_sparse_attn_decode
    sc = ctypes.c_float(0.088)
    args = [FAKE] * 7 + [4, 40000, 64, 128, 32, 4, 128, 2048, sc, FAKE, None, FAKE]
    need = L.dsa_decode_workspace_size(4, 40000, 64, 128, 2048, 32, 4, 128)
    assert need > 0
    assert f(*args, need - 1, None, None) == WORKSPACE
    assert b"workspace" in L.dsa_last_error()
    bad = list(args)
    bad[0] = None
    assert f(*bad, need, None, None) == INVALID
    bad = list(args)
    bad[7] = 0
    assert f(*bad, need, None, None) == INVALID
    bad = list(args)
    bad[11] = 16  # Hq
    assert f(*bad, need, None, None) == UNSUPPORTED
    bad = list(args)
    bad[18] = FAKE + 16  # workspace not 256-byte aligned
    assert f(*bad, need, None, None) == INVALID


def test_indexer_kl_rejects_bad_arguments_and_small_workspaces(L):
    f = L.dsa_indexer_kl_forward
    sc, sI = ctypes.c_float(0.088), ctypes.c_float(1.0 / 2048)
    need = L.dsa_indexer_kl_workspace_size(300, 32)
    # lse per (row, head) + lse per row + one partial per (row, 64-key tile), 256-byte aligned
    assert need >= 300 * 32 * 4 + 300 * 4 + 300 * 5 * 4
    ws = 0x100000  # 256-byte aligned
    args = [FAKE] * 5 + [300, 64, 128, 32, 4, 128, sc, sI, FAKE, FAKE, ws]
    assert f(*args, need - 1, None, None) == WORKSPACE
    bad = list(args)
    bad[15] = ws + 16  # workspace not 256-byte aligned
    assert f(*bad, need, None, None) == WORKSPACE
    bad = list(args)
    bad[3] = None  # Q
    assert f(*bad, need, None, None) == INVALID
    bad = list(args)
    bad[5] = 1 << 16  # L * L >= 2^31
    assert f(*bad, need, None, None) == INVALID
    bad = list(args)
    bad[9] = 3  # Hkv does not divide Hq
    assert f(*bad, need, None, None) == INVALID
    bad = list(args)
    bad[10] = 96  # d
    assert f(*bad, need, None, None) == UNSUPPORTED
    bad = list(args)
    bad[12] = ctypes.c_float(0.0)  # scale_I
    assert f(*bad, need, None, None) == INVALID
    bad = list(args)
    bad[6], bad[7] = 16, 128  # an indexer shape the scorer does not have
    assert f(*bad, need, None, None) == UNSUPPORTED

    g = L.dsa_indexer_kl_backward
    nb = L.dsa_indexer_kl_backward_workspace_size(300, 64, 128)
    assert nb >= 8 * 300 * 128 * 4  # eight head groups of dk partials
    assert L.dsa_indexer_kl_backward_workspace_size(300, 11, 128) == 256  # one group: no partials
    bargs = [FAKE] * 4 + [300, 64, 128, FAKE, FAKE, FAKE, ws]
    assert g(*bargs, nb - 1, None, None) == WORKSPACE
    bad = list(bargs)
    bad[5] = 0  # H_I
    assert g(*bad, nb, None, None) == INVALID
    bad = list(bargs)
    bad[6] = 96  # d_I
    assert g(*bad, nb, None, None) == UNSUPPORTED
    bad = list(bargs)
    bad[3] = None  # G
    assert g(*bad, nb, None, None) == INVALID


def test_dedup_workspace_size_and_argument_checks(L):
    """The dedup attention's workspace: per slot (a block of 128 / G queries,
    at most 4096 slots per wave) one int32 count (the counts 256-byte
    aligned), `cap` int32 keys and cap / 64 x (128 / G) 64-bit masks, cap =
    min((128 / G) k, L) rounded up to 64.  Shapes outside the kernel's
    support get their own status before the workspace is looked at."""
    size = L.dsa_sparse_attn_prefill_dedup_workspace_size

    def expect(Lq, G, k):
        qb = 128 // G
        nslot = min(-(-Lq // qb), 4096)
        cap = -(-min(qb * k, Lq) // 64) * 64
        return -(-nslot * 4 // 256) * 256 + nslot * cap * 4 + nslot * (cap // 64) * qb * 8

    assert size(3001, 32, 4, 128, 256) == expect(3001, 8, 256)
    assert size(262144, 32, 4, 128, 2048) == expect(262144, 8, 2048)
    assert size(1999, 8, 2, 64, 256) == expect(1999, 4, 256)
    assert size(1000, 8, 4, 128, 64) == 0        # G = 2: no 128-row tile
    assert size(1000, 32, 4, 96, 64) == 0        # d = 96
    f = L.dsa_sparse_attn_prefill_dedup
    sc = ctypes.c_float(0.088)
    need = size(3001, 32, 4, 128, 256)
    args = [FAKE] * 4 + [3001, 32, 4, 128, 256, sc, FAKE, FAKE]
    assert f(*args, need - 1, None, None) == WORKSPACE
    bad = list(args)
    bad[11] = None                               # workspace
    assert f(*bad, need, None, None) == INVALID
    bad = list(args)
    bad[5], bad[6] = 8, 4                        # G = 2
    assert f(*bad, need, None, None) == UNSUPPORTED
    bad = list(args)
    bad[7] = 96                                  # d
    assert f(*bad, need, None, None) == UNSUPPORTED
    bad = list(args)
    bad[4] = 262145                              # beyond the bitmap
    assert f(*bad, need, None, None) == UNSUPPORTED
    bad = list(args)
    bad[4], bad[5], bad[6], bad[8] = 131072, 16, 4, 2048   # G = 4: 32 x 2048 keys per block
    assert f(*bad, 1 << 40, None, None) == UNSUPPORTED
    bad = list(args)
    bad[9] = ctypes.c_float(0.0)                 # scale
    assert f(*bad, need, None, None) == INVALID
    bad = list(args)
    bad[3] = None                                # idx
    assert f(*bad, need, None, None) == INVALID


def test_check_device_error_rejects_bad_arguments(L):
    code = ctypes.c_int(0)
    assert L.dsa_check_device_error(None, None, None) == INVALID
    assert b"code is NULL" in L.dsa_last_error()
    assert L.dsa_check_device_error(FAKE + 2, ctypes.byref(code), None) == INVALID
    assert b"4-byte aligned" in L.dsa_last_error()


def test_every_launching_call_rejects_a_misaligned_error_word(L):
    """Each call takes its own device error word (4-byte aligned, or NULL for
    the per-device word); a misaligned one is refused before any launch."""
    sc = ctypes.c_float(0.125)
    bad_err = FAKE + 2
    calls = {
        "dsa_index_topk": [FAKE, FAKE, FAKE, 64, 4, 64, 8, FAKE, bad_err, None],
        "dsa_index_topk_varlen": [FAKE, FAKE, FAKE, FAKE, 1, 64, 4, 64, 8, FAKE, bad_err, None],
        "dsa_index_scores": [FAKE, FAKE, FAKE, 64, 4, 64, FAKE, bad_err, None],
        "dsa_sparse_attn_prefill": [FAKE] * 4 + [64, 8, 2, 64, 16, sc, FAKE, None, bad_err, None],
        "dsa_sparse_attn_backward": [FAKE] * 7 + [64, 8, 2, 64, 16, sc, FAKE, FAKE, FAKE, bad_err,
                                                  None],
        "dsa_sparse_attn_prefill_dedup": [FAKE] * 4 + [64, 8, 2, 64, 16, sc, FAKE, FAKE,
                                                       1 << 30, bad_err, None],
        "dsa_prefill_from_host": [FAKE] * 15 + [64, 4, 64, 8, 2, 64, 16, sc, 128, bad_err, None,
                                                 None, None],
        "dsa_sparse_attn_decode": [FAKE] * 7 + [4, 40000, 64, 128, 32, 4, 128, 2048,
                                                ctypes.c_float(0.088), FAKE, None, FAKE, 1 << 30,
                                                bad_err, None],
        "dsa_decode_from_host": [FAKE] * 12 + [4, 40000, 64, 128, 32, 4, 128, 2048,
                                               ctypes.c_float(0.088), FAKE, FAKE, FAKE, 1 << 30,
                                               bad_err, None],
        "dsa_sparse_attn_decode_noalloc": [FAKE] * 7 + [4, 40000, 64, 128, 32, 4, 128, 2048,
                                                        ctypes.c_float(0.088), FAKE, None,
                                                        bad_err, None],
        "dsa_indexer_kl_forward": [FAKE] * 5 + [300, 64, 128, 32, 4, 128, sc, sc, FAKE, FAKE,
                                                0x100000, 1 << 30, bad_err, None],
        "dsa_indexer_kl_backward": [FAKE] * 4 + [300, 64, 128, FAKE, FAKE, FAKE, 0x100000,
                                                 1 << 30, bad_err, None],
    }
    for name, args in calls.items():
        assert getattr(L, name)(*args) == INVALID, name
        assert b"err is not 4-byte aligned" in L.dsa_last_error(), name


def test_noalloc_checks_arguments_before_the_scratch_size(L):
    """Bad or unsupported shapes get their own status, as from the decode with
    a workspace; only a valid request too large for the built-in array gets
    DSA_ERR_WORKSPACE."""
    f = L.dsa_sparse_attn_decode_noalloc
    sc = ctypes.c_float(0.088)
    # B = 8192 (> 4096): invalid, although its scratch would also exceed 64 MiB
    args = [FAKE] * 7 + [8192, 1 << 30, 64, 128, 32, 4, 128, 2048, sc, FAKE, None, None, None]
    assert f(*args) == INVALID
    # Hq = 16 with a large batch: unsupported, not a workspace error
    args = [FAKE] * 7 + [4000, 1 << 30, 64, 128, 16, 4, 128, 2048, sc, FAKE, None, None, None]
    assert f(*args) == UNSUPPORTED
    # a valid shape whose scratch exceeds the array
    args = [FAKE] * 7 + [4000, 1 << 30, 64, 128, 32, 4, 128, 2048, sc, FAKE, None, None, None]
    assert f(*args) == WORKSPACE
    assert b"64" in L.dsa_last_error() or b"array" in L.dsa_last_error()


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(dsa, "_lib", None)
    monkeypatch.setattr(dsa, "LIB_PATH", "/nonexistent/libdsa_b200.so")
    with pytest.raises(RuntimeError, match="missing"):
        dsa.lib()


def test_binding_rejects_host_and_malformed_tensors(L):
    import torch
    q = torch.zeros((64, 4, 64), dtype=torch.uint8)
    k = torch.zeros((64, 64), dtype=torch.uint8)
    w = torch.zeros((64, 4), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.index_topk(q, k, w, 8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.index_scores(q, k, w)
    Q = torch.zeros((64, 8, 64), dtype=torch.bfloat16)
    K = torch.zeros((64, 2, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.indexer_kl_forward(q, k, w, Q, K, 0.125, 1.0,
                               kl=torch.zeros(64), G=torch.zeros((64, 64)),
                               workspace=torch.zeros(1 << 20, dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.indexer_kl_backward(q, k, w, torch.zeros((64, 64)),
                                dq_I=torch.zeros((64, 4, 64)), dk_I=torch.zeros((64, 64)),
                                dw=torch.zeros((64, 4)),
                                workspace=torch.zeros(256, dtype=torch.uint8))


def test_binding_checks_layout_before_the_call():
    import torch
    # a tensor that claims to live on the GPU, to reach the layout checks on a host
    class FakeCuda(torch.Tensor):
        @property
        def is_cuda(self):
            return True
    t = torch.zeros((8, 8), dtype=torch.float32).as_subclass(FakeCuda)
    with pytest.raises(ValueError, match="contiguous"):
        dsa._dev(t.t(), "x")
    with pytest.raises(ValueError, match="4-byte elements"):
        dsa._dev(torch.zeros(8, dtype=torch.float64).as_subclass(FakeCuda), "w", 4)
    assert dsa._dev(t, "x", 4) == t.data_ptr()


def test_binding_host_input_prefill_errors_are_value_errors():
    """prefill_from_host refuses a device tensor where a host one belongs, and
    a call without its copy streams, with ValueError (before the library)."""
    import torch

    class FakeCuda(torch.Tensor):
        @property
        def is_cuda(self):
            return True

    L_, H, dI, Hq, Hkv, d = 64, 4, 64, 8, 2, 64
    host = dict(q_I=torch.zeros((L_, H, dI), dtype=torch.uint8),
                k_I=torch.zeros((L_, dI), dtype=torch.uint8),
                w=torch.zeros((L_, H)), Q=torch.zeros((L_, Hq, d), dtype=torch.bfloat16),
                K=torch.zeros((L_, Hkv, d), dtype=torch.bfloat16),
                V=torch.zeros((L_, Hkv, d), dtype=torch.bfloat16),
                O=torch.zeros((L_, Hq, d), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="h2d_stream"):
        dsa.prefill_from_host(host, {}, 8, 0.125)
    bad = dict(host, Q=host["Q"].as_subclass(FakeCuda))
    with pytest.raises(ValueError, match="contiguous host tensor"):
        dsa.prefill_from_host(bad, {}, 8, 0.125, h2d_stream=1, d2h_stream=2)


def test_binding_error_word_must_be_int32():
    import torch
    with pytest.raises(ValueError, match="int32"):
        dsa._err(torch.zeros(1, dtype=torch.int64))
    assert dsa._err(None) is None
