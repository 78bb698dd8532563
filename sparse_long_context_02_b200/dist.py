"""One workload on P GPUs, one process per GPU (torch.distributed).

The per-rank steps are the library's C-ABI calls; the exchanges between
ranks are torch.distributed collectives (NCCL over NVLink on GPUs; the same
code runs over gloo on CPU tensors in the tests).  No collective touches a
kernel's operands while it runs, and nothing here reads another GPU's
memory directly.

Prefill (query shards, zig-zag blocks: see shards.py): each rank holds its
two row blocks of every input; one exchange step all-gathers the blocks of
k_I, K and V, so every rank holds every key, and the rank then selects and
attends for its own rows.  Output rows (idx, O) stay on their rank.

Decode:
* batch shards - each rank decodes its own sequences (no exchange);
  sequences are dealt longest first to the least-loaded rank;
* cache shards - each rank holds part of every sequence's cache; two small
  exchanges (the k kept (score, key) pairs per sequence, then the attention
  partials) give every rank the one-GPU result (see include/dsa.h).
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import torch
import torch.distributed as tdist

from . import shards


def gather_zigzag(mine: Sequence[torch.Tensor], out: torch.Tensor, L: int, P: int,
                  group=None) -> None:
    """All-gather the zig-zag blocks of one row-major tensor: `mine` holds
    this rank's blocks (block r, then block 2P - 1 - r, each a full block of
    rows, the last one padded), `out` [>= 2P * blk rows] receives every block
    at its rows.  Two collectives: the first half of the blocks arrives in
    rank order, i.e. in place; the second half arrives reversed and is moved
    to its rows."""
    blocks = shards.zigzag_blocks(L, P)
    blk = blocks[0][1] - blocks[0][0]
    first = out[: P * blk]
    tdist.all_gather_into_tensor(first, mine[0].contiguous(), group=group)
    tmp = torch.empty((P * blk,) + tuple(out.shape[1:]), dtype=out.dtype, device=out.device)
    tdist.all_gather_into_tensor(tmp, mine[1].contiguous(), group=group)
    for r in range(P):  # rank r sent block 2P - 1 - r
        b = 2 * P - 1 - r
        n = min(blk, max(0, out.shape[0] - b * blk))
        if n:
            out[b * blk: b * blk + n].copy_(tmp[r * blk: r * blk + n])


def own_blocks(t: torch.Tensor, L: int, P: int, rank: int) -> List[torch.Tensor]:
    """This rank's two blocks of a full tensor, each padded to the block size
    (the source of gather_zigzag when a rank has the whole tensor)."""
    blocks = shards.zigzag_blocks(L, P)
    blk = blocks[0][1] - blocks[0][0]
    res = []
    for b in (rank, 2 * P - 1 - rank):
        a, z = blocks[b]
        x = torch.zeros((blk,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        if z > a:
            x[: z - a].copy_(t[a:z])
        res.append(x)
    return res


def prefill_rows_step(dsa, rows: List[tuple], mine: Dict[str, torch.Tensor],
                      keys: Dict[str, torch.Tensor], k: int, scale: float, stream=None,
                      err=None) -> None:
    """Selection and attention of this rank's row blocks.  `mine[name][j]`
    is block j's q_I, w, Q, idx, O (rows of that block only); `keys` holds
    k_I, K, V for every row (after gather_zigzag)."""
    for j, (a, b) in enumerate(rows):
        n = b - a
        dsa.index_topk_rows(mine["q_I"][j][:n], keys["k_I"][:b], mine["w"][j][:n], a, k,
                            idx=mine["idx"][j][:n], stream=stream, err=err)
        dsa.sparse_attn_rows(mine["Q"][j][:n], keys["K"][:b], keys["V"][:b], mine["idx"][j][:n],
                             scale, O=mine["O"][j][:n], stream=stream, err=err)


def deal_sequences(lens: Sequence[int], P: int) -> List[List[int]]:
    """Batch shards: sequences, longest first, each to the rank with the
    fewest cache rows so far (ties to the lower rank); each rank's list is
    in ascending sequence order."""
    load = [0] * P
    own: List[List[int]] = [[] for _ in range(P)]
    for b in sorted(range(len(lens)), key=lambda i: (-int(lens[i]), i)):
        r = min(range(P), key=lambda j: (load[j], j))
        own[r].append(b)
        load[r] += int(lens[b])
    return [sorted(x) for x in own]


def decode_cache_step(dsa, q_I, w, Q, kI, K, V, off_r, base_r, k: int, scale: float, P: int,
                      group=None, stream=None, err=None, work=None):
    """Cache-sharded decode of the whole batch on this rank's part of every
    sequence's cache: local top-k pairs, all-gather, merge; local attention
    partials, all-gather, merge.  Returns (idx [B][k], O [B][Hq][d])."""
    B = q_I.shape[0]
    work = {} if work is None else work
    ords, keys = dsa.decode_select_shard(q_I, w, kI, off_r, k, key_base=base_r,
                                         ord_out=work.get("ord"), key_out=work.get("key"),
                                         workspace=work.get("ws"), stream=stream, err=err)
    def buf(name, like):
        t = work.get(name)
        if t is None:
            t = torch.empty((P,) + tuple(like.shape), dtype=like.dtype, device=like.device)
            work[name] = t
        return t

    all_o, all_k = buf("all_ord", ords), buf("all_key", keys)
    tdist.all_gather_into_tensor(all_o, ords, group=group)
    tdist.all_gather_into_tensor(all_k, keys, group=group)
    idx = dsa.decode_merge_shards(all_o, all_k, idx=work.get("idx"), stream=stream, err=err)
    po, pml = dsa.decode_attn_shard(Q, K, V, off_r, base_r, idx, scale, part_o=work.get("po"),
                                    part_ml=work.get("pml"), workspace=work.get("ws_a"),
                                    stream=stream, err=err)
    all_po, all_pml = buf("all_po", po), buf("all_pml", pml)
    tdist.all_gather_into_tensor(all_po, po, group=group)
    tdist.all_gather_into_tensor(all_pml, pml, group=group)
    O = dsa.decode_combine_shards(all_po, all_pml, O=work.get("O"), stream=stream, err=err)
    return idx, O
