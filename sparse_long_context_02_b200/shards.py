"""Partition plans for running one workload on P GPUs (one process per GPU).

Host logic only: which query rows and which cache rows each rank owns.  The
kernels run through the C ABI; the exchanges between ranks are the caller's
collectives (NCCL all-gathers over NVLink in bench.py).

Prefill (the query tokens of one long sequence): every query needs every
earlier key, and the indexer's and the attention's cost of row t grow with
t (the indexer linearly; the attention up to k), so contiguous row ranges
would leave the last rank with most of the work.  The rows are cut into 2P
equal blocks and rank r takes blocks r and 2P - 1 - r ("zig-zag"), which
gives every rank about the same number of causal pairs.  Each rank holds
its own rows of q_I, w and Q, and all keys (k_I, K, V) up to its last row,
gathered from the ranks that own them.

Decode (cache shards): each sequence's cache is cut into P contiguous parts,
rank r holding part r (a part may be empty for a short sequence).
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np

ROW_ALIGN = 128  # blocks start on a key tile (and on the indexer's 4-row query block)


def zigzag_blocks(L: int, P: int) -> List[Tuple[int, int]]:
    """The 2P blocks [b0, b1) of rows 0 .. L-1, block starts aligned to
    ROW_ALIGN (the last block takes the remainder; blocks may be empty for
    very short L)."""
    nb = 2 * P
    step = -(-L // nb)
    step = -(-step // ROW_ALIGN) * ROW_ALIGN
    return [(min(L, i * step), min(L, (i + 1) * step)) for i in range(nb)]


def zigzag_rows(L: int, P: int, rank: int) -> List[Tuple[int, int]]:
    """The non-empty row ranges of `rank`: blocks rank and 2P - 1 - rank."""
    blocks = zigzag_blocks(L, P)
    own = [blocks[rank], blocks[2 * P - 1 - rank]]
    return [(a, b) for a, b in own if b > a]


def block_owner(L: int, P: int) -> List[int]:
    """owner[i] = the rank that holds block i."""
    return [i if i < P else 2 * P - 1 - i for i in range(2 * P)]


def causal_pairs(rows: List[Tuple[int, int]], k: int = 0) -> float:
    """Indexer work of the rows: sum over t of (t + 1) pairs (with k > 0,
    the attention's sum of min(k, t + 1) instead)."""
    tot = 0.0
    for a, b in rows:
        t = np.arange(a, b, dtype=np.float64)
        tot += float((np.minimum(t + 1, k) if k else t + 1).sum())
    return tot


def cache_parts(lens: np.ndarray, P: int) -> List[dict]:
    """Per rank: lens_r [B] (rows of each sequence held), off_r [B + 1]
    (prefix sums: the rank's packed cache), base_r [B] (global position of
    the rank's first row of each sequence), and src [B] (where that first
    row sits in the sequence-major packed cache of the whole batch)."""
    lens = np.asarray(lens, np.int64)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    out = []
    for r in range(P):
        lo = (lens * r) // P
        hi = (lens * (r + 1)) // P
        lr = hi - lo
        out.append(dict(lens=lr, off=np.concatenate([[0], np.cumsum(lr)]).astype(np.int64),
                        base=lo.astype(np.int64), src=(off[:-1] + lo).astype(np.int64)))
    return out
