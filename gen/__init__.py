"""Seeded synthetic inputs for the DSA hot path.

Test and benchmark infrastructure, shared by the CPU oracle and the CUDA path
(the one module the two have in common).  It draws random values and stores
them in the formats the path consumes; it holds none of the method's
arithmetic.

The five workloads follow the problem statement of the Keye-VL-2.0 pages
(technical-report summary, section 1: top-2048 keys per query, 128K and 256K
contexts; section 8: decode over a long cache).  Indexer values are integers
drawn uniformly from [-8, 8] and stored as FP8 e4m3 (exact); the per-head
weights are integers in {0..3} stored as fp32; attention Q/K/V are N(0, 1)
rounded to bf16.  The video workload clusters indexer keys and K/V around a
per-frame centroid (240 frames of 16 text + 1076 vision tokens, then 64
trailing text tokens).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Dict, Optional

import numpy as np

from .build import build as _build, LIB_PATH

# Tensor ids: one independent stream per tensor.
T_QI, T_KI, T_W, T_Q, T_K, T_V, T_LENS, T_IDX_CENT, T_K_CENT, T_V_CENT = range(1, 11)

SEED_BASE = 20260000

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _build()
        L = ctypes.CDLL(LIB_PATH)
        u64, u32, i32, i64, dbl, vp = (ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int,
                                       ctypes.c_int64, ctypes.c_double, ctypes.c_void_p)
        L.dsagen_int_e4m3.argtypes = [u64, u32, u64, u64, i32, i32, vp, i32]
        L.dsagen_int_f32.argtypes = [u64, u32, u64, u64, i32, i32, vp, i32]
        L.dsagen_int_i64.argtypes = [u64, u32, u64, u64, i32, i32, vp, i32]
        L.dsagen_normal_bf16.argtypes = [u64, u32, u64, u64, dbl, vp, i32]
        L.dsagen_encode_e4m3.argtypes = [vp, u64, vp]
        L.dsagen_encode_bf16.argtypes = [vp, u64, vp]
        L.dsagen_video_int_e4m3.argtypes = [u64, u32, u32, u64, u64, u64, u64, i64, i64, i64,
                                            i32, i32, i32, i32, i32, i32, i32, i32, vp, i32]
        L.dsagen_video_normal_bf16.argtypes = [u64, u32, u32, u64, u64, u64, i64, i64, i64,
                                               dbl, vp, i32]
        for f in (L.dsagen_int_e4m3, L.dsagen_int_f32, L.dsagen_int_i64, L.dsagen_normal_bf16,
                  L.dsagen_encode_e4m3, L.dsagen_encode_bf16, L.dsagen_video_int_e4m3,
                  L.dsagen_video_normal_bf16):
            f.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ------------------------------------------------------------------ raw draws

def int_e4m3(seed, tensor, start, count, lo=-8, hi=8, nthreads=0, out=None) -> np.ndarray:
    out = np.empty(count, np.uint8) if out is None else out
    lib().dsagen_int_e4m3(seed, tensor, start, count, lo, hi, _ptr(out), nthreads)
    return out


def int_f32(seed, tensor, start, count, lo=0, hi=3, nthreads=0, out=None) -> np.ndarray:
    out = np.empty(count, np.float32) if out is None else out
    lib().dsagen_int_f32(seed, tensor, start, count, lo, hi, _ptr(out), nthreads)
    return out


def int_i64(seed, tensor, start, count, lo, hi, nthreads=0) -> np.ndarray:
    out = np.empty(count, np.int64)
    lib().dsagen_int_i64(seed, tensor, start, count, lo, hi, _ptr(out), nthreads)
    return out


def normal_bf16(seed, tensor, start, count, sigma=1.0, nthreads=0, out=None) -> np.ndarray:
    """bf16 bit patterns (uint16) of sigma * N(0, 1)."""
    out = np.empty(count, np.uint16) if out is None else out
    lib().dsagen_normal_bf16(seed, tensor, start, count, sigma, _ptr(out), nthreads)
    return out


def encode_e4m3(values) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(values, np.float64))
    out = np.empty(v.shape, np.uint8)
    lib().dsagen_encode_e4m3(_ptr(v), v.size, _ptr(out))
    return out


def encode_bf16(values) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(values, np.float64))
    out = np.empty(v.shape, np.uint16)
    lib().dsagen_encode_bf16(_ptr(v), v.size, _ptr(out))
    return out


# ---------------------------------------------------------------- workloads

@dataclasses.dataclass(frozen=True)
class Config:
    id: int
    name: str
    kind: str                 # "prefill" or "decode"
    k: int
    H_I: int
    d_I: int
    Hq: int
    Hkv: int
    d: int
    L: int = 0                # prefill sequence length
    B: int = 0                # decode batch
    n_lo: int = 0             # decode cached lengths ~ U{n_lo..n_hi}
    n_hi: int = 0
    video: bool = False
    frames: int = 240
    frame_text: int = 16
    frame_vision: int = 1076
    seed: Optional[int] = None

    @property
    def seed_(self) -> int:
        return SEED_BASE + self.id if self.seed is None else self.seed

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[int, Config] = {
    1: Config(1, "tiny prefill L=2048 k=256", "prefill", k=256, H_I=4, d_I=64,
              Hq=8, Hkv=2, d=64, L=2048),
    2: Config(2, "prefill L=32768 k=2048", "prefill", k=2048, H_I=64, d_I=128,
              Hq=32, Hkv=4, d=128, L=32768),
    3: Config(3, "prefill L=131072 k=2048", "prefill", k=2048, H_I=64, d_I=128,
              Hq=32, Hkv=4, d=128, L=131072),
    4: Config(4, "decode B=64 n~U[32768,262144] k=2048", "decode", k=2048, H_I=64, d_I=128,
              Hq=32, Hkv=4, d=128, B=64, n_lo=32768, n_hi=262144),
    5: Config(5, "video prefill L=262144 k=2048", "prefill", k=2048, H_I=64, d_I=128,
              Hq=32, Hkv=4, d=128, L=262144, video=True),
}

# The workloads by name.
TINY_PREFILL = CONFIGS[1]    # tiny prefill L=2048 k=256 (small heads)
PREFILL_32K = CONFIGS[2]     # prefill L=32768 k=2048
PREFILL_128K = CONFIGS[3]    # prefill L=131072 k=2048
DECODE_B64 = CONFIGS[4]      # decode B=64, n ~ U[32768, 262144], k=2048
VIDEO_256K = CONFIGS[5]      # video prefill L=262144 k=2048


def custom(**kw) -> Config:
    """A small prefill (or decode) workload with the i.i.d. recipe; id 0."""
    base = dict(id=0, name="custom", kind="prefill", k=16, H_I=4, d_I=64, Hq=8, Hkv=2, d=64,
                L=64)
    base.update(kw)
    return Config(**base)


# -- prefill tensors, generated for a token range [t0, t1) ------------------

def prefill_qI(cfg: Config, t0=0, t1=None, nthreads=0) -> np.ndarray:
    t1 = cfg.L if t1 is None else t1
    row = cfg.H_I * cfg.d_I
    n = (t1 - t0) * row
    if cfg.video:
        out = np.empty(n, np.uint8)
        lib().dsagen_video_int_e4m3(cfg.seed_, T_QI, T_IDX_CENT, t0 * row, n, row, cfg.d_I,
                                    cfg.frame_text + cfg.frame_vision, cfg.frame_text,
                                    cfg.frames, -6, 6, -2, 2, -8, 8, -8, 8, _ptr(out), nthreads)
    else:
        out = int_e4m3(cfg.seed_, T_QI, t0 * row, n, -8, 8, nthreads)
    return out.reshape(t1 - t0, cfg.H_I, cfg.d_I)


def prefill_kI(cfg: Config, t0=0, t1=None, nthreads=0) -> np.ndarray:
    t1 = cfg.L if t1 is None else t1
    row = cfg.d_I
    n = (t1 - t0) * row
    if cfg.video:
        out = np.empty(n, np.uint8)
        lib().dsagen_video_int_e4m3(cfg.seed_, T_KI, T_IDX_CENT, t0 * row, n, row, cfg.d_I,
                                    cfg.frame_text + cfg.frame_vision, cfg.frame_text,
                                    cfg.frames, -6, 6, -2, 2, -8, 8, -8, 8, _ptr(out), nthreads)
    else:
        out = int_e4m3(cfg.seed_, T_KI, t0 * row, n, -8, 8, nthreads)
    return out.reshape(t1 - t0, cfg.d_I)


def prefill_w(cfg: Config, t0=0, t1=None, nthreads=0) -> np.ndarray:
    t1 = cfg.L if t1 is None else t1
    return int_f32(cfg.seed_, T_W, t0 * cfg.H_I, (t1 - t0) * cfg.H_I, 0, 3,
                   nthreads).reshape(t1 - t0, cfg.H_I)


def prefill_Q(cfg: Config, t0=0, t1=None, nthreads=0) -> np.ndarray:
    t1 = cfg.L if t1 is None else t1
    row = cfg.Hq * cfg.d
    return normal_bf16(cfg.seed_, T_Q, t0 * row, (t1 - t0) * row, 1.0,
                       nthreads).reshape(t1 - t0, cfg.Hq, cfg.d)


def _prefill_kv(cfg: Config, tensor: int, cent: int, t0, t1, nthreads) -> np.ndarray:
    t1 = cfg.L if t1 is None else t1
    row = cfg.Hkv * cfg.d
    n = (t1 - t0) * row
    if cfg.video:
        out = np.empty(n, np.uint16)
        lib().dsagen_video_normal_bf16(cfg.seed_, tensor, cent, t0 * row, n, row,
                                       cfg.frame_text + cfg.frame_vision, cfg.frame_text,
                                       cfg.frames, 0.5, _ptr(out), nthreads)
    else:
        out = normal_bf16(cfg.seed_, tensor, t0 * row, n, 1.0, nthreads)
    return out.reshape(t1 - t0, cfg.Hkv, cfg.d)


def prefill_K(cfg: Config, t0=0, t1=None, nthreads=0) -> np.ndarray:
    return _prefill_kv(cfg, T_K, T_K_CENT, t0, t1, nthreads)


def prefill_V(cfg: Config, t0=0, t1=None, nthreads=0) -> np.ndarray:
    return _prefill_kv(cfg, T_V, T_V_CENT, t0, t1, nthreads)


def prefill_inputs(cfg: Config, nthreads=0) -> Dict[str, np.ndarray]:
    assert cfg.kind == "prefill"
    return dict(q_I=prefill_qI(cfg, nthreads=nthreads), k_I=prefill_kI(cfg, nthreads=nthreads),
                w=prefill_w(cfg, nthreads=nthreads), Q=prefill_Q(cfg, nthreads=nthreads),
                K=prefill_K(cfg, nthreads=nthreads), V=prefill_V(cfg, nthreads=nthreads))


# -- decode tensors -----------------------------------------------------------

def decode_lengths(cfg: Config) -> np.ndarray:
    return int_i64(cfg.seed_, T_LENS, 0, cfg.B, cfg.n_lo, cfg.n_hi, 1)


def decode_offsets(cfg: Config) -> np.ndarray:
    """[B + 1] prefix sums of the cached lengths (rows of the packed caches)."""
    n = decode_lengths(cfg)
    return np.concatenate([[0], np.cumsum(n)]).astype(np.int64)


def decode_queries(cfg: Config, nthreads=0) -> Dict[str, np.ndarray]:
    B = cfg.B
    return dict(
        q_I=int_e4m3(cfg.seed_, T_QI, 0, B * cfg.H_I * cfg.d_I, -8, 8,
                     nthreads).reshape(B, cfg.H_I, cfg.d_I),
        w=int_f32(cfg.seed_, T_W, 0, B * cfg.H_I, 0, 3, nthreads).reshape(B, cfg.H_I),
        Q=normal_bf16(cfg.seed_, T_Q, 0, B * cfg.Hq * cfg.d, 1.0,
                      nthreads).reshape(B, cfg.Hq, cfg.d))


def decode_kI_rows(cfg: Config, r0: int, r1: int, nthreads=0) -> np.ndarray:
    return int_e4m3(cfg.seed_, T_KI, r0 * cfg.d_I, (r1 - r0) * cfg.d_I, -8, 8,
                    nthreads).reshape(r1 - r0, cfg.d_I)


def decode_K_rows(cfg: Config, r0: int, r1: int, nthreads=0) -> np.ndarray:
    row = cfg.Hkv * cfg.d
    return normal_bf16(cfg.seed_, T_K, r0 * row, (r1 - r0) * row, 1.0,
                       nthreads).reshape(r1 - r0, cfg.Hkv, cfg.d)


def decode_V_rows(cfg: Config, r0: int, r1: int, nthreads=0) -> np.ndarray:
    row = cfg.Hkv * cfg.d
    return normal_bf16(cfg.seed_, T_V, r0 * row, (r1 - r0) * row, 1.0,
                       nthreads).reshape(r1 - r0, cfg.Hkv, cfg.d)


def decode_inputs(cfg: Config, nthreads=0) -> Dict[str, np.ndarray]:
    """All decode tensors at once (small decode workloads; the full-size
    cache is better produced in row ranges with decode_*_rows)."""
    assert cfg.kind == "decode"
    off = decode_offsets(cfg)
    N = int(off[-1])
    d = decode_queries(cfg, nthreads)
    d.update(cache_off=off, kI_cache=decode_kI_rows(cfg, 0, N, nthreads),
             K_cache=decode_K_rows(cfg, 0, N, nthreads),
             V_cache=decode_V_rows(cfg, 0, N, nthreads))
    return d
