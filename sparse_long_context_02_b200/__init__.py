"""B200-native DeepSeek-Sparse-Attention hot path (indexer -> top-k -> sparse
GQA attention, prefill and decode).

This module is the Python binding of ``libdsa_b200.so`` (C ABI in
``include/dsa.h``): it checks and marshals arguments and calls the library;
every step of the computation runs in the library's CUDA kernels.  PyTorch
only provides device memory and streams.  There is no fallback: if the
library is missing, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa_b200.so")

DSA_OK = 0
DEVERR_NONE, DEVERR_TIMEOUT, DEVERR_INDEX = 0, 1, 2

_lib = None


class DSAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with "
                "`python -m sparse_long_context_02_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, f32, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                                 ctypes.c_size_t)
        L.dsa_version.restype = i32
        L.dsa_version.argtypes = []
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_status_string.argtypes = [i32]
        L.dsa_last_error.restype = ctypes.c_char_p
        L.dsa_last_error.argtypes = []
        L.dsa_index_topk.restype = i32
        L.dsa_index_topk.argtypes = [vp, vp, vp, i64, i32, i32, i32, vp, vp, vp]
        L.dsa_index_scores.restype = i32
        L.dsa_index_scores.argtypes = [vp, vp, vp, i64, i32, i32, vp, vp, vp]
        L.dsa_sparse_attn_prefill_dedup.restype = i32
        L.dsa_sparse_attn_prefill_dedup.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32,
                                                    ctypes.c_float, vp, vp, sz, vp, vp]
        L.dsa_sparse_attn_prefill_dedup_workspace_size.restype = sz
        L.dsa_sparse_attn_prefill_dedup_workspace_size.argtypes = [i64, i32, i32, i32, i32]
        L.dsa_prefill_from_host.restype = i32
        L.dsa_prefill_from_host.argtypes = [vp] * 15 + [i64, i32, i32, i32, i32, i32, i32,
                                                          ctypes.c_float, i64, vp, vp, vp, vp]
        L.dsa_index_topk_varlen.restype = i32
        L.dsa_index_topk_varlen.argtypes = [vp, vp, vp, vp, i32, i64, i32, i32, i32, vp, vp, vp]
        L.dsa_sparse_attn_prefill.restype = i32
        L.dsa_sparse_attn_prefill.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32, f32, vp,
                                              vp, vp, vp]
        L.dsa_sparse_attn_backward.restype = i32
        L.dsa_sparse_attn_backward.argtypes = [vp] * 7 + [i64, i32, i32, i32, i32, f32, vp, vp,
                                                          vp, vp, vp]
        L.dsa_decode_workspace_size.restype = sz
        L.dsa_decode_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, i32, i32]
        L.dsa_sparse_attn_decode.restype = i32
        L.dsa_sparse_attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                             i32, i32, i32, f32, vp, vp, vp, sz, vp, vp]
        L.dsa_decode_from_host.restype = i32
        L.dsa_decode_from_host.argtypes = [vp] * 11 + [vp, i32, i64, i32, i32, i32, i32, i32, i32,
                                                       f32, vp, vp, vp, sz, vp, vp]
        L.dsa_sparse_attn_decode_noalloc.restype = i32
        L.dsa_sparse_attn_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32,
                                                     i32, i32, i32, i32, i32, f32, vp, vp, vp,
                                                     vp]
        L.dsa_indexer_kl_workspace_size.restype = sz
        L.dsa_indexer_kl_workspace_size.argtypes = [i64, i32]
        L.dsa_indexer_kl_forward.restype = i32
        L.dsa_indexer_kl_forward.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, f32,
                                             f32, vp, vp, vp, sz, vp, vp]
        L.dsa_indexer_kl_backward.restype = i32
        L.dsa_indexer_kl_backward_workspace_size.restype = sz
        L.dsa_indexer_kl_backward_workspace_size.argtypes = [i64, i32, i32]
        L.dsa_indexer_kl_backward.argtypes = [vp, vp, vp, vp, i64, i32, i32, vp, vp, vp, vp, sz,
                                              vp, vp]
        L.dsa_index_topk_rows.restype = i32
        L.dsa_index_topk_rows.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, vp, vp, vp]
        L.dsa_sparse_attn_rows.restype = i32
        L.dsa_sparse_attn_rows.argtypes = [vp, vp, vp, vp, i64, i64, i32, i32, i32, i32, f32, vp,
                                           vp, vp, vp]
        L.dsa_decode_select_shard.restype = i32
        L.dsa_decode_select_shard.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, vp, vp,
                                              vp, sz, vp, vp]
        L.dsa_decode_merge_shards.restype = i32
        L.dsa_decode_merge_shards.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp]
        L.dsa_decode_attn_shard_workspace_size.restype = sz
        L.dsa_decode_attn_shard_workspace_size.argtypes = [i32, i64, i32, i32, i32]
        L.dsa_decode_attn_shard.restype = i32
        L.dsa_decode_attn_shard.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                            f32, vp, vp, vp, sz, vp, vp]
        L.dsa_decode_combine_shards.restype = i32
        L.dsa_decode_combine_shards.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp]
        L.dsa_check_device_error.restype = i32
        L.dsa_check_device_error.argtypes = [vp, ctypes.POINTER(i32), vp]
        _lib = L
    return _lib


def _check(status: int, name: str) -> None:
    if status != DSA_OK:
        L = lib()
        raise DSAError(status, f"{name}: {L.dsa_status_string(status).decode()}: "
                               f"{L.dsa_last_error().decode()}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, name: str, nbytes_per_elem: Optional[int] = None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.type == "cuda" and t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, but the library launches on the current "
                         f"device cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if nbytes_per_elem is not None and t.element_size() != nbytes_per_elem:
        raise ValueError(f"{name} must have {nbytes_per_elem}-byte elements, got {t.dtype}")
    return t.data_ptr()


def _err(err: Optional[torch.Tensor]) -> Optional[int]:
    """The caller's device error word (a one-element int32 CUDA tensor), or
    None for the library's per-device word."""
    if err is None:
        return None
    if err.dtype != torch.int32 or err.numel() < 1:
        raise ValueError("err must be an int32 CUDA tensor of at least one element")
    return _dev(err, "err", 4)


def error_word(device=None) -> torch.Tensor:
    """A fresh (zeroed) device error word for the calls of one stream."""
    return torch.zeros(1, dtype=torch.int32, device=device if device is not None else "cuda")


def version() -> int:
    return lib().dsa_version()


def index_topk(q_I: torch.Tensor, k_I: torch.Tensor, w: torch.Tensor, k: int,
               idx: Optional[torch.Tensor] = None, stream=None, err=None) -> torch.Tensor:
    """Indexer + top-k.  q_I [L][H_I][d_I] and k_I [L][d_I] e4m3 (uint8 or
    float8_e4m3fn), w [L][H_I] float32 -> idx [L][k] int32 (ascending, -1 pad)."""
    L, H, d = q_I.shape
    if idx is None:
        idx = torch.empty((L, k), dtype=torch.int32, device=q_I.device)
    _check(lib().dsa_index_topk(_dev(q_I, "q_I", 1), _dev(k_I, "k_I", 1), _dev(w, "w", 4), L, H, d,
                                k, _dev(idx, "idx", 4), _err(err), _stream(stream)),
           "dsa_index_topk")
    return idx


def index_topk_varlen(q_I: torch.Tensor, k_I: torch.Tensor, w: torch.Tensor,
                      cu_seqlens: torch.Tensor, k: int, idx: Optional[torch.Tensor] = None,
                      stream=None, err=None) -> torch.Tensor:
    """Indexer + top-k over a packed batch: cu_seqlens [nseq + 1] int32 on the
    device (0 ... L); row t of a sequence sees only that sequence's keys up to
    t.  idx holds packed key positions (ascending, -1 pad)."""
    L, H, d = q_I.shape
    if idx is None:
        idx = torch.empty((L, k), dtype=torch.int32, device=q_I.device)
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
        raise ValueError("dsa_index_topk_varlen: cu_seqlens must be an int32 device tensor")
    nseq = cu_seqlens.numel() - 1
    _check(lib().dsa_index_topk_varlen(_dev(q_I, "q_I", 1), _dev(k_I, "k_I", 1), _dev(w, "w", 4),
                                       _dev(cu_seqlens, "cu_seqlens", 4), nseq, L, H, d, k,
                                       _dev(idx, "idx", 4), _err(err), _stream(stream)),
           "dsa_index_topk_varlen")
    return idx


def index_scores(q_I: torch.Tensor, k_I: torch.Tensor, w: torch.Tensor,
                 scores: Optional[torch.Tensor] = None, stream=None, err=None) -> torch.Tensor:
    """Dense causal indexer scores [L][L] float32 (-inf above the diagonal)."""
    L, H, d = q_I.shape
    if scores is None:
        scores = torch.empty((L, L), dtype=torch.float32, device=q_I.device)
    _check(lib().dsa_index_scores(_dev(q_I, "q_I", 1), _dev(k_I, "k_I", 1), _dev(w, "w", 4), L, H,
                                  d, _dev(scores, "scores", 4), _err(err), _stream(stream)),
           "dsa_index_scores")
    return scores


def sparse_attn_prefill(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, idx: torch.Tensor,
                        scale: float, O: Optional[torch.Tensor] = None,
                        stream=None, err=None, lse: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Sparse GQA attention.  Q [L][Hq][d], K/V [L][Hkv][d] bf16, idx [L][k]
    int32 -> O [L][Hq][d] bf16.  With `lse` (a [L][Hq] float32 tensor), also
    each row's log-sum-exp, the input of sparse_attn_backward."""
    L, Hq, d = Q.shape
    Hkv = K.shape[1]
    k = idx.shape[1]
    if O is None:
        O = torch.empty_like(Q)
    _check(lib().dsa_sparse_attn_prefill(_dev(Q, "Q", 2), _dev(K, "K", 2), _dev(V, "V", 2),
                                         _dev(idx, "idx", 4), L, Hq, Hkv, d, k, float(scale),
                                         _dev(O, "O", 2),
                                         _dev(lse, "lse", 4) if lse is not None else None,
                                         _err(err), _stream(stream)),
           "dsa_sparse_attn_prefill")
    return O


def sparse_attn_backward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, idx: torch.Tensor,
                         O: torch.Tensor, lse: torch.Tensor, dO: torch.Tensor, scale: float,
                         dQ: Optional[torch.Tensor] = None, dK: Optional[torch.Tensor] = None,
                         dV: Optional[torch.Tensor] = None, stream=None, err=None):
    """Gradients through the sparse attention.  Q, K, V, idx as
    sparse_attn_prefill; O and lse the forward's outputs; dO [L][Hq][d] bf16.
    Returns (dQ [L][Hq][d], dK [L][Hkv][d], dV [L][Hkv][d]), float32."""
    L, Hq, d = Q.shape
    Hkv = K.shape[1]
    k = idx.shape[1]
    if dQ is None:
        dQ = torch.empty((L, Hq, d), dtype=torch.float32, device=Q.device)
    if dK is None:
        dK = torch.empty((L, Hkv, d), dtype=torch.float32, device=Q.device)
    if dV is None:
        dV = torch.empty((L, Hkv, d), dtype=torch.float32, device=Q.device)
    _check(lib().dsa_sparse_attn_backward(
        _dev(Q, "Q", 2), _dev(K, "K", 2), _dev(V, "V", 2), _dev(idx, "idx", 4), _dev(O, "O", 2),
        _dev(lse, "lse", 4), _dev(dO, "dO", 2), L, Hq, Hkv, d, k, float(scale),
        _dev(dQ, "dQ", 4), _dev(dK, "dK", 4), _dev(dV, "dV", 4), _err(err), _stream(stream)),
        "dsa_sparse_attn_backward")
    return dQ, dK, dV


def _host(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host tensor")
    return t.data_ptr()


def prefill_from_host(host: dict, dev: dict, k: int, scale: float, chunk_rows: int = 8192,
                      stream=None, h2d_stream=None, d2h_stream=None, err=None) -> None:
    """Whole prefill from host inputs with copies and kernels overlapped in
    row chunks.  host: q_I, k_I, w, Q, K, V (inputs) and O (output), pinned
    CPU tensors; dev: device buffers of the same names plus idx [L][k].
    Asynchronous on `stream` (host["O"] is filled when it completes)."""
    L, H, d_I = host["q_I"].shape
    Hq, d = host["Q"].shape[1], host["Q"].shape[2]
    Hkv = host["K"].shape[1]
    if h2d_stream is None or d2h_stream is None:
        raise ValueError("dsa_prefill_from_host: pass h2d_stream and d2h_stream")
    names = ("q_I", "k_I", "w", "Q", "K", "V")
    args = [_host(host[n], n) for n in names] + [_host(host["O"], "O")]
    args += [_dev(dev[n], n) for n in names] + [_dev(dev["idx"], "idx", 4), _dev(dev["O"], "O")]
    _check(lib().dsa_prefill_from_host(*args, L, H, d_I, Hq, Hkv, d, k, float(scale), chunk_rows,
                                       _err(err), _stream(stream), _stream(h2d_stream),
                                       _stream(d2h_stream)),
           "dsa_prefill_from_host")


def dedup_workspace_size(L: int, Hq: int, Hkv: int, d: int, k: int) -> int:
    """Bytes of workspace sparse_attn_prefill_dedup needs (0: shape unsupported)."""
    return lib().dsa_sparse_attn_prefill_dedup_workspace_size(L, Hq, Hkv, d, k)


def sparse_attn_prefill_dedup(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                              idx: torch.Tensor, scale: float, O: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None, stream=None,
                              err=None) -> torch.Tensor:
    """sparse_attn_prefill for blocks of 128 / (Hq / Hkv) adjacent queries
    that gather the union of their index rows once (pays when adjacent rows
    overlap).  `workspace`: a uint8 device tensor of at least
    dedup_workspace_size(...) bytes, allocated here when None."""
    L, Hq, d = Q.shape
    Hkv = K.shape[1]
    k = idx.shape[1]
    if O is None:
        O = torch.empty_like(Q)
    need = dedup_workspace_size(L, Hq, Hkv, d, k)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=Q.device)
    _check(lib().dsa_sparse_attn_prefill_dedup(_dev(Q, "Q", 2), _dev(K, "K", 2), _dev(V, "V", 2),
                                               _dev(idx, "idx", 4), L, Hq, Hkv, d, k,
                                               float(scale), _dev(O, "O", 2),
                                               _dev(workspace, "workspace", 1),
                                               workspace.numel() * workspace.element_size(),
                                               _err(err), _stream(stream)),
           "dsa_sparse_attn_prefill_dedup")
    return O


def decode_workspace_size(B: int, total_n: int, H_I: int, d_I: int, k: int, Hq: int, Hkv: int,
                          d: int) -> int:
    return lib().dsa_decode_workspace_size(B, total_n, H_I, d_I, k, Hq, Hkv, d)


def sparse_attn_decode(q_I, w, Q, kI_cache, K_cache, V_cache, cache_off, k: int, scale: float,
                       O=None, idx_out=None, workspace=None, stream=None, err=None):
    """One new token per sequence.  Returns (O [B][Hq][d] bf16, idx_out or None)."""
    B, H, dI = q_I.shape
    _, Hq, d = Q.shape
    total_n = kI_cache.shape[0]
    Hkv = K_cache.shape[1]
    if O is None:
        O = torch.empty_like(Q)
    need = decode_workspace_size(B, total_n, H, dI, k, Hq, Hkv, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    _check(lib().dsa_sparse_attn_decode(
        _dev(q_I, "q_I", 1), _dev(w, "w", 4), _dev(Q, "Q", 2), _dev(kI_cache, "kI_cache", 1),
        _dev(K_cache, "K_cache", 2), _dev(V_cache, "V_cache", 2), _dev(cache_off, "cache_off", 8),
        B, total_n, H, dI, Hq, Hkv, d, k, float(scale), _dev(O, "O", 2),
        _dev(idx_out, "idx_out", 4) if idx_out is not None else None,
        _dev(workspace, "workspace", 1), workspace.numel(), _err(err), _stream(stream)),
        "dsa_sparse_attn_decode")
    return O, idx_out


def decode_from_host(host: dict, dev: dict, cache_off, k: int, scale: float, stream=None,
                     err=None) -> None:
    """One decode step with the queries in (pinned) host memory and the caches
    on the device: host q_I, w, Q (inputs) and O (output, optionally idx);
    dev q_I, w, Q, kI_cache, K_cache, V_cache, O, workspace (optionally idx).
    Asynchronous on `stream` (host["O"] is filled when it completes)."""
    B, H, dI = host["q_I"].shape
    Hq, d = host["Q"].shape[1], host["Q"].shape[2]
    total_n, Hkv = dev["kI_cache"].shape[0], dev["K_cache"].shape[1]
    ih = _host(host["idx"], "idx") if host.get("idx") is not None else None
    idx = dev.get("idx")
    ws = dev["workspace"]
    _check(lib().dsa_decode_from_host(
        _host(host["q_I"], "q_I"), _host(host["w"], "w"), _host(host["Q"], "Q"),
        _host(host["O"], "O"), ih, _dev(dev["q_I"], "q_I", 1), _dev(dev["w"], "w", 4),
        _dev(dev["Q"], "Q", 2), _dev(dev["kI_cache"], "kI_cache", 1),
        _dev(dev["K_cache"], "K_cache", 2), _dev(dev["V_cache"], "V_cache", 2),
        _dev(cache_off, "cache_off", 8), B, total_n, H, dI, Hq, Hkv, d, k, float(scale),
        _dev(dev["O"], "O", 2), _dev(idx, "idx", 4) if idx is not None else None,
        _dev(ws, "workspace", 1), ws.numel(), _err(err), _stream(stream)),
        "dsa_decode_from_host")


def sparse_attn_decode_noalloc(q_I, w, Q, kI_cache, K_cache, V_cache, cache_off, k: int,
                               scale: float, O=None, idx_out=None, stream=None, err=None):
    """sparse_attn_decode without a workspace argument, for callers that
    cannot allocate device memory at call time: the scratch is a fixed
    64 MiB array inside the library (see include/dsa.h).  Calls that overlap
    on the GPU share that array and must be serialized by the caller."""
    B, H, dI = q_I.shape
    _, Hq, d = Q.shape
    total_n = kI_cache.shape[0]
    Hkv = K_cache.shape[1]
    if O is None:
        O = torch.empty_like(Q)
    _check(lib().dsa_sparse_attn_decode_noalloc(
        _dev(q_I, "q_I", 1), _dev(w, "w", 4), _dev(Q, "Q", 2), _dev(kI_cache, "kI_cache", 1),
        _dev(K_cache, "K_cache", 2), _dev(V_cache, "V_cache", 2), _dev(cache_off, "cache_off", 8),
        B, total_n, H, dI, Hq, Hkv, d, k, float(scale), _dev(O, "O", 2),
        _dev(idx_out, "idx_out", 4) if idx_out is not None else None, _err(err),
        _stream(stream)), "dsa_sparse_attn_decode_noalloc")
    return O, idx_out


def device_error(stream=None, err=None) -> int:
    """Synchronizes the stream; returns and clears a device error word: the
    caller's `err` tensor, or the library's per-device word when None."""
    code = ctypes.c_int(0)
    _check(lib().dsa_check_device_error(_err(err), ctypes.byref(code), _stream(stream)),
           "dsa_check_device_error")
    return code.value


def indexer_kl_workspace_size(L: int, Hq: int) -> int:
    return lib().dsa_indexer_kl_workspace_size(L, Hq)


def indexer_kl_forward(q_I: torch.Tensor, k_I: torch.Tensor, w: torch.Tensor, Q: torch.Tensor,
                       K: torch.Tensor, scale: float, scale_I: float = 1.0,
                       kl: Optional[torch.Tensor] = None, G: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None, err=None):
    """Indexer warm-up loss.  Returns (kl [L] float32, G [L][L] float32 =
    d(sum kl)/dI, zero above the diagonal).  q_I/k_I e4m3, w float32, Q/K
    bf16 (layouts as dsa_indexer_kl_forward)."""
    L, H_I, d_I = q_I.shape
    _, Hq, d = Q.shape
    Hkv = K.shape[1]
    dev = q_I.device
    if kl is None:
        kl = torch.empty(L, dtype=torch.float32, device=dev)
    if G is None:
        G = torch.empty((L, L), dtype=torch.float32, device=dev)
    need = indexer_kl_workspace_size(L, Hq)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check(lib().dsa_indexer_kl_forward(
        _dev(q_I, "q_I", 1), _dev(k_I, "k_I", 1), _dev(w, "w", 4), _dev(Q, "Q", 2),
        _dev(K, "K", 2), L, H_I, d_I, Hq, Hkv, d, float(scale), float(scale_I), _dev(kl, "kl", 4),
        _dev(G, "G", 4), _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _err(err), _stream(stream)), "dsa_indexer_kl_forward")
    return kl, G


def indexer_kl_backward(q_I: torch.Tensor, k_I: torch.Tensor, w: torch.Tensor, G: torch.Tensor,
                        dq_I: Optional[torch.Tensor] = None, dk_I: Optional[torch.Tensor] = None,
                        dw: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None, err=None):
    """Gradients of sum_t kl[t] with respect to q_I, k_I and w, from G.
    Returns (dq_I [L][H_I][d_I], dk_I [L][d_I], dw [L][H_I]), float32."""
    L, H_I, d_I = q_I.shape
    dev = q_I.device
    if workspace is None:
        workspace = torch.empty(lib().dsa_indexer_kl_backward_workspace_size(L, H_I, d_I),
                                dtype=torch.uint8, device=dev)
    if dq_I is None:
        dq_I = torch.empty((L, H_I, d_I), dtype=torch.float32, device=dev)
    if dk_I is None:
        dk_I = torch.empty((L, d_I), dtype=torch.float32, device=dev)
    if dw is None:
        dw = torch.empty((L, H_I), dtype=torch.float32, device=dev)
    _check(lib().dsa_indexer_kl_backward(
        _dev(q_I, "q_I", 1), _dev(k_I, "k_I", 1), _dev(w, "w", 4), _dev(G, "G", 4), L, H_I, d_I,
        _dev(dq_I, "dq_I", 4), _dev(dk_I, "dk_I", 4), _dev(dw, "dw", 4),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _err(err), _stream(stream)), "dsa_indexer_kl_backward")
    return dq_I, dk_I, dw


# ------------------------------------------------------------------ sharded calls

def index_topk_rows(q_I: torch.Tensor, k_I: torch.Tensor, w: torch.Tensor, row0: int, k: int,
                    idx: Optional[torch.Tensor] = None, stream=None, err=None) -> torch.Tensor:
    """Indexer + top-k for the query rows [row0, row0 + len(q_I)) of a longer
    sequence: q_I [R][H_I][d_I] and w [R][H_I] hold those rows, k_I holds
    (at least) keys 0 .. row0 + R - 1.  Returns idx [R][k]."""
    R, H, d = q_I.shape
    row1 = row0 + R
    if k_I.shape[0] < row1:
        raise ValueError("index_topk_rows: k_I must hold every key up to the last row")
    if idx is None:
        idx = torch.empty((R, k), dtype=torch.int32, device=q_I.device)
    _check(lib().dsa_index_topk_rows(_dev(q_I, "q_I", 1), _dev(k_I, "k_I", 1), _dev(w, "w", 4),
                                     row0, row1, H, d, k, _dev(idx, "idx", 4), _err(err),
                                     _stream(stream)), "dsa_index_topk_rows")
    return idx


def sparse_attn_rows(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, idx: torch.Tensor,
                     scale: float, O: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, stream=None, err=None) -> torch.Tensor:
    """Sparse attention for R query rows (Q [R][Hq][d], idx [R][k]) over the
    keys of K / V [n][Hkv][d].  Returns O [R][Hq][d]."""
    R, Hq, d = Q.shape
    n, Hkv = K.shape[0], K.shape[1]
    k = idx.shape[1]
    if O is None:
        O = torch.empty_like(Q)
    _check(lib().dsa_sparse_attn_rows(_dev(Q, "Q", 2), _dev(K, "K", 2), _dev(V, "V", 2),
                                      _dev(idx, "idx", 4), R, n, Hq, Hkv, d, k, float(scale),
                                      _dev(O, "O", 2),
                                      _dev(lse, "lse", 4) if lse is not None else None,
                                      _err(err), _stream(stream)), "dsa_sparse_attn_rows")
    return O


def decode_select_shard(q_I, w, kI_cache, cache_off, k: int, key_base=None, ord_out=None,
                        key_out=None, workspace=None, stream=None, err=None):
    """This rank's exact top-k per sequence over its cache rows: returns
    (ord_out [B][k] uint32 as int32 bits, key_out [B][k] int32 global keys)."""
    B, H, dI = q_I.shape
    total_n = kI_cache.shape[0]
    dev = q_I.device
    if ord_out is None:
        ord_out = torch.empty((B, k), dtype=torch.int32, device=dev)
    if key_out is None:
        key_out = torch.empty((B, k), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(decode_workspace_size(B, total_n, H, dI, k, 32, 4, 128),
                                dtype=torch.uint8, device=dev)
    _check(lib().dsa_decode_select_shard(
        _dev(q_I, "q_I", 1), _dev(w, "w", 4), _dev(kI_cache, "kI_cache", 1),
        _dev(cache_off, "cache_off", 8),
        _dev(key_base, "key_base", 8) if key_base is not None else None, B, total_n, H, dI, k,
        _dev(ord_out, "ord_out", 4), _dev(key_out, "key_out", 4), _dev(workspace, "workspace", 1),
        workspace.numel(), _err(err), _stream(stream)), "dsa_decode_select_shard")
    return ord_out, key_out


def decode_merge_shards(ord_in, key_in, idx=None, stream=None, err=None):
    """Global index rows from the P ranks' gathered lists [P][B][k]."""
    P, B, k = key_in.shape
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=key_in.device)
    _check(lib().dsa_decode_merge_shards(_dev(ord_in, "ord_in", 4), _dev(key_in, "key_in", 4), P,
                                         B, k, _dev(idx, "idx", 4), _err(err), _stream(stream)),
           "dsa_decode_merge_shards")
    return idx


def decode_attn_shard(Q, K_cache, V_cache, cache_off, key_base, idx, scale: float, part_o=None,
                      part_ml=None, workspace=None, stream=None, err=None):
    """This rank's attention partials (part_o [B][Hq][d], part_ml [B][Hq][2])."""
    B, Hq, d = Q.shape
    total_n, Hkv = K_cache.shape[0], K_cache.shape[1]
    k = idx.shape[1]
    dev = Q.device
    if part_o is None:
        part_o = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    if part_ml is None:
        part_ml = torch.empty((B, Hq, 2), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(lib().dsa_decode_attn_shard_workspace_size(B, total_n, k, Hq, d),
                                dtype=torch.uint8, device=dev)
    _check(lib().dsa_decode_attn_shard(
        _dev(Q, "Q", 2), _dev(K_cache, "K_cache", 2), _dev(V_cache, "V_cache", 2),
        _dev(cache_off, "cache_off", 8), _dev(key_base, "key_base", 8), _dev(idx, "idx", 4), B,
        total_n, Hq, Hkv, d, k, float(scale), _dev(part_o, "part_o", 4),
        _dev(part_ml, "part_ml", 4), _dev(workspace, "workspace", 1), workspace.numel(),
        _err(err), _stream(stream)), "dsa_decode_attn_shard")
    return part_o, part_ml


def decode_combine_shards(part_o, part_ml, O=None, stream=None, err=None):
    """Output rows O [B][Hq][d] bf16 from the gathered partials [P][B][Hq][*]."""
    P, B, Hq, d = part_o.shape
    if O is None:
        O = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=part_o.device)
    _check(lib().dsa_decode_combine_shards(_dev(part_o, "part_o", 4), _dev(part_ml, "part_ml", 4),
                                           P, B, Hq, d, _dev(O, "O", 2), _err(err),
                                           _stream(stream)), "dsa_decode_combine_shards")
    return O
