"""Writes the oracle's index rows of a full-size prefill workload as SHA-256
digests, one per block of consecutive query rows.

Every query keeps the min(k, t+1) best keys (Kwai Keye-VL-2.0 technical-report
summary, section 1: each query keeps its 2048 most relevant positions), so
the selected set of every row at the full workload sizes has exactly one
correct value.  The oracle needs hours for the 128K and 256K workloads, far
too long for a test run, so this script runs it once and stores, per block
of ``block_rows`` rows, the SHA-256 of the rows as the oracle writes them
(int32 little-endian, ascending, -1 padded, k entries per row).  The GPU
tests hash the library's rows the same way and compare block by block.

Only ``gen`` (seeded inputs) and ``oracle`` are used here: no value comes
from the CUDA path.  The file is keyed by the workload, its seed and the
SHA-256 of the oracle's and the generator's C sources; the tests refuse a
file whose keys do not match the sources they run with.

The run is resumable: finished blocks are kept in the output file and a
rerun computes only the missing ones.

    python tests/golden/make_index_digests.py prefill_32k prefill_128k video_256k
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import gen  # noqa: E402
import oracle  # noqa: E402

WORKLOADS = {"prefill_32k": gen.PREFILL_32K, "prefill_128k": gen.PREFILL_128K,
             "video_256k": gen.VIDEO_256K}
BLOCK_ROWS = 1024


def source_sha256(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def keys(cfg) -> dict:
    """What a digest file must match to be used."""
    return {"workload": cfg.name, "L": cfg.L, "k": cfg.k, "H_I": cfg.H_I, "d_I": cfg.d_I,
            "video": cfg.video, "seed": cfg.seed_, "block_rows": BLOCK_ROWS,
            "oracle_sha256": source_sha256(os.path.join(ROOT, "oracle", "dsa_oracle.c")),
            "gen_sha256": source_sha256(os.path.join(ROOT, "gen", "dsa_gen.c"))}


def digest_path(name: str) -> str:
    return os.path.join(HERE, f"index_digests_{name}.json")


def block_digest(rows_i32: np.ndarray) -> str:
    a = np.ascontiguousarray(rows_i32, dtype="<i4")
    return hashlib.sha256(a.tobytes()).hexdigest()


def load(name: str):
    """The stored digests of workload ``name`` ({block: hex}) and their keys,
    or (None, None) when there is no file."""
    p = digest_path(name)
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        d = json.load(f)
    return {int(b): h for b, h in d["digests"].items()}, d["keys"]


def _save(name: str, k: dict, digests: dict) -> None:
    p = digest_path(name)
    tmp = p + ".tmp"
    with open(tmp, "w") as f:
        json.dump({"keys": k, "nblocks": -(-k["L"] // BLOCK_ROWS),
                   "digests": {str(b): digests[b] for b in sorted(digests)}}, f, indent=0)
        f.write("\n")
    os.replace(tmp, p)


def run(name: str, nthreads: int = 0) -> None:
    cfg = WORKLOADS[name]
    k = keys(cfg)
    digests, stored = load(name)
    if digests is None or stored != k:
        digests = {}
    nblocks = -(-cfg.L // BLOCK_ROWS)
    todo = [b for b in range(nblocks) if b not in digests]
    if not todo:
        print(f"{name}: all {nblocks} blocks present", flush=True)
        return
    q_I, k_I, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    for b in todo:
        t0 = time.time()
        rows = np.arange(b * BLOCK_ROWS, min(cfg.L, (b + 1) * BLOCK_ROWS), dtype=np.int64)
        idx = oracle.index_topk(q_I, k_I, w, cfg.k, rows=rows, nthreads=nthreads)
        digests[b] = block_digest(idx)
        _save(name, k, digests)
        print(f"{name}: block {b + 1}/{nblocks} in {time.time() - t0:.1f} s", flush=True)


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("workloads", nargs="+", choices=sorted(WORKLOADS))
    ap.add_argument("--threads", type=int, default=0, help="oracle threads (0: all cores)")
    a = ap.parse_args()
    for name in a.workloads:
        run(name, a.threads)


if __name__ == "__main__":
    main()
