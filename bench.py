#!/usr/bin/env python
"""Benchmark of the DSA hot path on B200 (one process per GPU).

One step = one pass of the whole hot path over one batch of synthetic input:
  prefill of a 131072-token sequence (indexer + top-2048 + sparse GQA
  attention: dsa_index_topk, dsa_sparse_attn_prefill), then
  one decode step of 64 sequences with cached lengths ~ U[32768, 262144]
  (dsa_sparse_attn_decode).
`value` is prefill query-tokens/s over the device time of the prefill part of
the step; the decode part is reported as decode tokens/s.  Inputs are resident
in HBM when the timed region starts; L2 is flushed (256 MiB write) between
timed steps, outside the per-step events.  With torchrun every rank runs its
own independent workload (weak scaling, no collective on the data path).

`--impl reference` times the CPU oracle (the reference arm of this build) on a
bounded sample of the same workload and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen  # noqa: E402

METRIC = ("prefill query-tokens/s & decode tokens/s at 128K ctx, k=2048; "
          "% FP8/HBM roofline")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefill-config", type=int, default=gen.PREFILL_128K.id,
                    help="workload id of the prefill part (0: no prefill part)")
    ap.add_argument("--prefill-L", type=int, default=0,
                    help="run the prefill workload at this sequence length instead of its own "
                         "(a smaller case of the same recipe, for profiling)")
    ap.add_argument("--decode-config", type=int, default=gen.DECODE_B64.id,
                    help="workload id of the decode part (0: no decode part)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="use only the first B sequences of the decode workload (profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunk", type=int, default=8192,
                    help="rows per chunk of the host-input prefill in the e2e measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--attn", default="auto", choices=["auto", "rows", "dedup"],
                    help="prefill attention kernel: one CTA per query row, the adjacent-query "
                         "dedup kernel, or auto (dedup on the video workload)")
    ap.add_argument("--union-stats", type=int, default=0, metavar="G",
                    help="instead of timing: run the prefill indexer once and report how many "
                         "distinct keys the index rows of G consecutive queries select together "
                         "(the traffic an adjacent-query dedup would read)")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the per-workload lines of the tiny, 32K and 256K-video prefills "
                         "(timed after the headline step, on one GPU)")
    ap.add_argument("--replicas", action="store_true",
                    help="with several GPUs: every rank solves its own copy of the workload "
                         "(weak scaling) instead of sharing one workload")
    ap.add_argument("--decode-shard", default="batch", choices=["batch", "cache"],
                    help="with several GPUs: split the decode batch by sequence (no exchange) "
                         "or every sequence's cache (two all-gathers per step)")
    ap.add_argument("--attn-bwd", action="store_true",
                    help="instead of the inference step: time the sparse attention's training "
                         "pass (forward with lse, then dsa_sparse_attn_backward) on the prefill "
                         "workload's index rows")
    ap.add_argument("--kl", type=int, default=0, metavar="L",
                    help="instead of the inference step: time the indexer warm-up KL loss "
                         "(forward: loss and dL/dI; backward: dq_I, dk_I, dw) at sequence "
                         "length L with the prefill workload's head shapes")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return dict(hbm=float(m["hbm_gbs"]), bf16=float(m["bf16_tflops"]),
                    bf16_sus=float(m["bf16_tflops_sustained"]), src="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------------ work model

def prefill_flops(cfg) -> float:
    """Indexer: 2 * H_I * d_I FLOP per causal (t, s) pair."""
    return 2.0 * cfg.H_I * cfg.d_I * cfg.L * (cfg.L + 1) / 2.0


def prefill_attn_bytes(cfg) -> float:
    """Gather: 2 * Hkv * d * 2 bytes per selected row, plus Q, O and the index row."""
    L, k = cfg.L, cfg.k
    sel = k * L - k * (k - 1) / 2.0 if L >= k else L * (L + 1) / 2.0  # sum_t min(k, t+1)
    row = 2 * cfg.Hkv * cfg.d * 2
    per_tok = 2 * cfg.Hq * cfg.d * 2 + 4 * k
    return sel * row + L * per_tok


def decode_bytes(cfg, lens) -> float:
    """k_I scan (d_I bytes per cached key) + gathered K/V rows + queries/outputs."""
    sel = float(np.minimum(lens, cfg.k).sum())
    return (float(lens.sum()) * cfg.d_I + sel * 2 * cfg.Hkv * cfg.d * 2
            + cfg.B * (cfg.H_I * cfg.d_I + cfg.H_I * 4 + 2 * 2 * cfg.Hq * cfg.d))


# ------------------------------------------------------------------ DRAM traffic

# DRAM bytes of one launch per unit of work, from the committed measurement
# record of single-kernel ncu captures (profiles/dram_traffic.json); valid
# only for the kernel sources the counters were taken on.
def traffic_record() -> dict:
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


def csrc_sha256(sources) -> str:
    import hashlib
    root = os.path.join(ROOT, "sparse_long_context_02_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(sources):
        h.update(name.encode())
        with open(os.path.join(root, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def dram_traffic(kernel: str, pcfg):
    """(bytes per launch or None, why) for the bench's prefill workload."""
    t = traffic_record().get(kernel)
    if t is None or pcfg is None:
        return None, "no capture"
    if not t.get("scales_with_units"):
        return None, f"measured at {t['workload']}; does not scale with L"
    if t["src_sha256"] != csrc_sha256(t["sources"]):
        return None, "kernel sources changed since the capture"
    per = (t["dram_read_bytes"] + t["dram_write_bytes"]) / t["units"]
    return per * pcfg.L, f"{t['summary']}, scaled by L from {t['workload']}"


def l2_read_peak(torch) -> float:
    """GB/s of reads that hit L2: 16-byte ld.global.cg loads over a buffer
    small enough to stay in L2 (24 or 48 MiB), 100 passes, best of the
    sizes and of 5 runs (libdsa_probe.so, a measurement utility built beside
    the library).  The bound of a kernel whose gathered rows hit L2."""
    import ctypes
    from sparse_long_context_02_b200 import build as dsa_build
    L = ctypes.CDLL(dsa_build.build_probe())
    L.dsa_probe_l2_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_void_p, ctypes.c_void_p]
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    sink = torch.zeros(4, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream()
    best = 0.0
    for mib in (24, 48):
        buf = torch.ones((mib << 20) // 4, dtype=torch.float32, device="cuda")
        for rep in range(6):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            if L.dsa_probe_l2_read(buf.data_ptr(), buf.numel() * 4, 100, 4 * sms,
                                   sink.data_ptr(), st.cuda_stream) != 0:
                raise RuntimeError("L2 probe launch failed")
            e1.record(st)
            torch.cuda.synchronize()
            if rep:  # the first run warms the buffer into L2
                best = max(best, 100 * buf.numel() * 4 / (e0.elapsed_time(e1) / 1e3) / 1e9)
    return best


_FP8_PROBE = None


def fp8_mma_peak(torch) -> float:
    """TFLOP/s of the tensor cores on the indexer's own product shape
    (tcgen05.mma kind::f8f6f4, e4m3 -> f32, M = 128, N = 256, K = 128 per
    tile) with resident operands and nothing else to do: one CTA per SM,
    20 000 tiles each (libdsa_probe.so, a measurement utility built beside
    the library).  Best of 5 runs after a warm-up: a burst figure."""
    global _FP8_PROBE
    if _FP8_PROBE is not None:
        return _FP8_PROBE
    import ctypes
    from sparse_long_context_02_b200 import build as dsa_build
    L = ctypes.CDLL(dsa_build.build_probe())
    L.dsa_probe_fp8_mma.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p]
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    sink = torch.zeros(4, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream()
    iters, best = 20000, 0.0
    for rep in range(6):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        if L.dsa_probe_fp8_mma(iters, sink.data_ptr(), err.data_ptr(), st.cuda_stream) != 0:
            raise RuntimeError("FP8 probe launch failed")
        e1.record(st)
        torch.cuda.synchronize()
        if rep:
            flop = 2.0 * 128 * 256 * 128 * iters * sms
            best = max(best, flop / (e0.elapsed_time(e1) / 1e3) / 1e12)
    if int(err.item()) != 0:
        raise RuntimeError("FP8 probe: a bounded wait gave up")
    _FP8_PROBE = best
    return best


def fp8_alt_peaks(torch, achieved: float) -> dict:
    """The indexer's rate against the FP8 rate measured here and against the
    nominal dense FP8 figure (4.5 PFLOP/s), beside the main fraction."""
    pk = fp8_mma_peak(torch)
    return {"fp8_probe": dict(peak=pk, frac=achieved / pk, unit="TFLOP/s",
                              source="measured here: tcgen05 kind::f8f6f4 M128 N256 with "
                                     "resident operands (libdsa_probe.so), burst"),
            "nominal": dict(peak=4500.0, frac=achieved / 4500.0, unit="TFLOP/s")}


# ------------------------------------------------------------------ ranks

def rank_workloads(pcfg, dcfg, rank: int, world: int):
    """Weak scaling: every rank solves its own problem of the same shape (the
    seeds differ by rank, so no two ranks hold the same data)."""
    if world <= 1:
        return pcfg, dcfg
    return (pcfg and pcfg.with_(seed=pcfg.seed_ + 1000 * rank),
            dcfg and dcfg.with_(seed=dcfg.seed_ + 1000 * rank))


def max_over_ranks(values, world: int, device=None):
    """Elementwise max of per-rank timings (the slowest rank sets the pace)."""
    arr = np.asarray(values, dtype=np.float64)
    if world <= 1:
        return arr
    import torch
    import torch.distributed as tdist
    t = torch.tensor(arr, device=device if device is not None else "cpu")
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return t.cpu().numpy()


def job_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the max time."""
    return world * units_per_rank / seconds


# ------------------------------------------------------------------ clocks

class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"])
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in open(self.path):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return dict(sm_mhz=statistics.median(sm) if sm else None,
                    sm_max_mhz=max(smax) if smax else None, reasons=sorted(reasons),
                    samples=len(sm))


# ------------------------------------------------------------------ our arm

def upload(torch, a: np.ndarray, dtype=None, pin=False):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    if pin:
        t = t.pin_memory()
    return t.cuda(non_blocking=False), t


def build_prefill(torch, cfg, keep_host: bool):
    import sparse_long_context_02_b200 as dsa  # noqa: F401
    host = gen.prefill_inputs(cfg)
    dev, pinned = {}, {}
    for name, dt in (("q_I", None), ("k_I", None), ("w", None), ("Q", torch.bfloat16),
                     ("K", torch.bfloat16), ("V", torch.bfloat16)):
        dev[name], h = upload(torch, host[name], dt, pin=keep_host)
        if keep_host:
            pinned[name] = h
    dev["idx"] = torch.empty((cfg.L, cfg.k), dtype=torch.int32, device="cuda")
    dev["O"] = torch.empty((cfg.L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
    return dev, pinned, host


def build_decode(torch, cfg, keep_host: bool):
    import sparse_long_context_02_b200 as dsa
    off = gen.decode_offsets(cfg)
    N = int(off[-1])
    q = gen.decode_queries(cfg)
    dev, pinned = {}, {}
    for name, dt in (("q_I", None), ("w", None), ("Q", torch.bfloat16)):
        dev[name], h = upload(torch, q[name], dt, pin=keep_host)
        if keep_host:
            pinned[name] = h
    dev["cache_off"], h = upload(torch, off, None, pin=keep_host)
    if keep_host:
        pinned["cache_off"] = h
    # caches: generated in row blocks straight into device memory
    dev["kI_cache"] = torch.empty((N, cfg.d_I), dtype=torch.uint8, device="cuda")
    dev["K_cache"] = torch.empty((N, cfg.Hkv, cfg.d), dtype=torch.bfloat16, device="cuda")
    dev["V_cache"] = torch.empty((N, cfg.Hkv, cfg.d), dtype=torch.bfloat16, device="cuda")
    step = 1 << 19
    for r0 in range(0, N, step):
        r1 = min(N, r0 + step)
        dev["kI_cache"][r0:r1].copy_(torch.from_numpy(gen.decode_kI_rows(cfg, r0, r1)))
        dev["K_cache"][r0:r1].copy_(torch.from_numpy(
            gen.decode_K_rows(cfg, r0, r1).view(np.int16)).view(torch.bfloat16))
        dev["V_cache"][r0:r1].copy_(torch.from_numpy(
            gen.decode_V_rows(cfg, r0, r1).view(np.int16)).view(torch.bfloat16))
    dev["O"] = torch.empty((cfg.B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
    dev["idx"] = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device="cuda")
    need = dsa.decode_workspace_size(cfg.B, N, cfg.H_I, cfg.d_I, cfg.k, cfg.Hq, cfg.Hkv, cfg.d)
    dev["ws"] = torch.empty(need, dtype=torch.uint8, device="cuda")
    return dev, pinned, off


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as tdist
    import sparse_long_context_02_b200 as dsa

    torch.cuda.set_device(local_rank)
    pcfg = gen.CONFIGS[args.prefill_config] if args.prefill_config else None
    if pcfg is not None and args.prefill_L:
        pcfg = pcfg.with_(L=args.prefill_L, name=f"{pcfg.name} at L={args.prefill_L}")
    dcfg = gen.CONFIGS[args.decode_config] if args.decode_config else None
    if dcfg is not None and args.decode_batch:
        dcfg = dcfg.with_(B=args.decode_batch)
    pcfg, dcfg = rank_workloads(pcfg, dcfg, rank, world)
    keep_host = not args.no_e2e
    P, Ph, p_host = build_prefill(torch, pcfg, keep_host) if pcfg else ({}, {}, None)
    D, Dh, off = build_decode(torch, dcfg, keep_host) if dcfg else ({}, {}, np.zeros(1))
    lens = np.diff(off)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def prefill():
        if pcfg is None:
            return
        dsa.index_topk(P["q_I"], P["k_I"], P["w"], pcfg.k, idx=P["idx"], stream=stream)

    use_dedup = pcfg is not None and (args.attn == "dedup" or (args.attn == "auto" and pcfg.video))
    dd_ws = None
    if use_dedup:
        dd_ws = torch.empty(dsa.dedup_workspace_size(pcfg.L, pcfg.Hq, pcfg.Hkv, pcfg.d, pcfg.k),
                            dtype=torch.uint8, device="cuda")

    def attn():
        if pcfg is None:
            return
        if use_dedup:
            dsa.sparse_attn_prefill_dedup(P["Q"], P["K"], P["V"], P["idx"], pcfg.scale, O=P["O"],
                                          workspace=dd_ws, stream=stream)
        else:
            dsa.sparse_attn_prefill(P["Q"], P["K"], P["V"], P["idx"], pcfg.scale, O=P["O"],
                                    stream=stream)

    def decode():
        if dcfg is None:
            return
        dsa.sparse_attn_decode(D["q_I"], D["w"], D["Q"], D["kI_cache"], D["K_cache"],
                               D["V_cache"], D["cache_off"], dcfg.k, dcfg.scale, O=D["O"],
                               idx_out=D["idx"], workspace=D["ws"], stream=stream)

    # prefill: the indexer, then the attention (the dedup attention: a plan and a
    # tensor-core kernel per wave of 4096 blocks of 128 / G queries);
    # decode: index, merge, attention, combine
    n_attn = 1
    if use_dedup:
        qb = 128 // (pcfg.Hq // pcfg.Hkv)
        n_attn = 2 * (-(-(-(-pcfg.L // qb)) // 4096))
    launches_per_step = ((1 + n_attn) if pcfg else 0) + (4 if dcfg else 0)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        prefill()
        if ev is not None:
            ev[1].record(stream)
        attn()
        if ev is not None:
            ev[2].record(stream)
        decode()
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if dsa.device_error() != 0:
        raise RuntimeError("device error during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = Clocks(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                    else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    if world > 1:
        tdist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    if world > 1:
        tdist.barrier()
    clk = clocks.stop()
    t_idx = [e[0].elapsed_time(e[1]) for e in evs]
    t_att = [e[1].elapsed_time(e[2]) for e in evs]
    t_dec = [e[2].elapsed_time(e[3]) for e in evs]
    err = dsa.device_error()
    if err != 0:
        raise RuntimeError(f"device error {err} in the timed region")

    # ms over the K steps, max over ranks
    tot = max_over_ranks([sum(t_idx) + sum(t_att), sum(t_dec)], world, device="cuda")
    K = args.steps
    prefill_ms = tot[0] / K
    decode_ms = tot[1] / K
    value = job_throughput(pcfg.L, world, prefill_ms / 1e3) if pcfg else 0.0
    decode_tps = job_throughput(dcfg.B, world, decode_ms / 1e3) if dcfg else 0.0

    # ---- roofline of each kernel, reported for the dominant one
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_sus"]
    ms_idx, ms_att, ms_dec = (statistics.mean(t_idx), statistics.mean(t_att),
                              statistics.mean(t_dec))
    kernels = {}
    if pcfg:
        kernels["dsa_index_topk"] = dict(
            bound="tensor", ms=ms_idx, work=prefill_flops(pcfg),
            achieved=prefill_flops(pcfg) / (ms_idx / 1e3) / 1e12, peak=fp8_peak, unit="TFLOP/s")
        kernels["dsa_index_topk"].update(
            fp8_alt_peaks(torch, kernels["dsa_index_topk"]["achieved"]))
        # the gathered rows mostly hit L2 (94 % at L = 65536): its bound is
        # L2 read bandwidth, measured here
        l2pk = l2_read_peak(torch)
        a_by, a_fl = (dedup_attn_cost(torch, pcfg, P["idx"]) if use_dedup
                      else (prefill_attn_bytes(pcfg), None))
        aname = "dsa_sparse_attn_prefill_dedup" if use_dedup else "dsa_sparse_attn_prefill"
        kernels[aname] = dict(
            bound="l2", ms=ms_att, work=a_by, achieved=a_by / (ms_att / 1e3) / 1e9, peak=l2pk,
            peak_source="measured here: L2-resident 16-byte reads (libdsa_probe.so)",
            unit="GB/s", hbm_peak=pk["hbm"])
        if a_fl is not None:
            kernels[aname]["tensor"] = dict(achieved=a_fl / (ms_att / 1e3) / 1e12,
                                            peak=pk["bf16_sus"], unit="TFLOP/s",
                                            frac=a_fl / (ms_att / 1e3) / 1e12 / pk["bf16_sus"])
    if dcfg:
        kernels["dsa_sparse_attn_decode"] = dict(
            bound="hbm", ms=ms_dec, work=decode_bytes(dcfg, lens),
            achieved=decode_bytes(dcfg, lens) / (ms_dec / 1e3) / 1e9, peak=pk["hbm"],
            unit="GB/s")
        kernels["dsa_sparse_attn_decode"]["spec"] = dict(  # the HBM3e data-sheet figure
            peak=8000.0, frac=kernels["dsa_sparse_attn_decode"]["achieved"] / 8000.0, unit="GB/s")
    for v in kernels.values():
        v["frac"] = v["achieved"] / v["peak"]
    dom = max(kernels, key=lambda n: kernels[n]["ms"])
    dk = kernels[dom]
    traffic, traffic_src = dram_traffic(dom, pcfg)
    roofline = dict(bound=dk["bound"], achieved=dk["achieved"], peak=dk["peak"], unit=dk["unit"],
                    frac=dk["frac"], traffic=traffic, traffic_source=traffic_src, kernel=dom,
                    peak_source=f"{pk['src']} ({'2 x sustained bf16' if dk['bound'] == 'tensor' else 'hbm copy'})")

    # ---- end to end through the public API with host buffers
    e2e = None
    if keep_host:
        O_host = torch.empty(P["O"].shape if pcfg else (1,), dtype=torch.bfloat16).pin_memory()
        Od_host = torch.empty(D["O"].shape if dcfg else (1,), dtype=torch.bfloat16).pin_memory()
        h2d_p = sum(v.numel() * v.element_size() for v in Ph.values())
        h2d_d = sum(Dh[n].numel() * Dh[n].element_size() for n in ("q_I", "w", "Q")) if dcfg else 0
        d2h_p = O_host.numel() * 2 if pcfg else 0
        d2h_d = Od_host.numel() * 2 if dcfg else 0
        ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        if world > 1:
            tdist.barrier()
        torch.cuda.synchronize()
        h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
        for i in range(K):
            flush.zero_()
            ev2[i][0].record(stream)
            if pcfg:
                # the library's host-input prefill: row chunks whose copies
                # overlap the kernels of the chunks before them
                dsa.prefill_from_host(dict(Ph, O=O_host), P, pcfg.k, pcfg.scale,
                                      chunk_rows=args.e2e_chunk, stream=stream,
                                      h2d_stream=h2d_s, d2h_stream=d2h_s)
            ev2[i][1].record(stream)
            if dcfg:
                # the library's host-input decode: queries in, outputs out,
                # the caches resident on the device
                dsa.decode_from_host(dict(q_I=Dh["q_I"], w=Dh["w"], Q=Dh["Q"], O=Od_host),
                                     dict(q_I=D["q_I"], w=D["w"], Q=D["Q"],
                                          kI_cache=D["kI_cache"], K_cache=D["K_cache"],
                                          V_cache=D["V_cache"], O=D["O"], idx=D["idx"],
                                          workspace=D["ws"]),
                                     D["cache_off"], dcfg.k, dcfg.scale, stream=stream)
            ev2[i][2].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            tdist.barrier()
        e_p = sum(e[0].elapsed_time(e[1]) for e in ev2)
        e_d = sum(e[1].elapsed_time(e[2]) for e in ev2)
        et = max_over_ranks([e_p, e_d], world, device="cuda")
        e2e = dict(value=job_throughput(pcfg.L, world, et[0] / K / 1e3) if pcfg else 0.0,
                   unit="query-tokens/s",
                   h2d_bytes_per_step=int(h2d_p + h2d_d), d2h_bytes_per_step=int(d2h_p + d2h_d),
                   decode_value=job_throughput(dcfg.B, world, et[1] / K / 1e3) if dcfg else 0.0,
                   decode_unit="tokens/s", ms_per_step=float((et[0] + et[1]) / K))
        # result read back: a sanity check that the copy carried real output
        if not torch.isfinite(O_host.float()).all():
            raise RuntimeError("non-finite output")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and pcfg:
        cpu = cpu_baseline(pcfg, p_host, args.cpu_seconds, dcfg)

    others = None
    if world == 1 and not args.no_other_configs and pcfg is not None:
        del P, Ph, p_host
        torch.cuda.empty_cache()
        others = other_configs(torch, dsa, pk, args, stream, flush)

    return dict(value=value, prefill_ms=prefill_ms, decode_ms=decode_ms, decode_tps=decode_tps,
                clocks=clk, kernels=kernels, roofline=roofline, e2e=e2e, cpu=cpu,
                launches=launches_per_step * K, pcfg=pcfg, dcfg=dcfg, others=others)


def dedup_stats(torch, idx, qb: int):
    """(distinct keys, distinct keys rounded up to the 64-key chunk) summed
    over the blocks of qb consecutive index rows (counted on the device)."""
    L, k = idx.shape
    nb = (L + qb - 1) // qb
    pad = nb * qb - L
    distinct = chunked = 0
    for b0 in range(0, nb, 2048):
        b1 = min(nb, b0 + 2048)
        x = idx[b0 * qb:min(L, b1 * qb)]
        if b1 == nb and pad:
            x = torch.cat([x, torch.full((pad, k), -1, dtype=x.dtype, device=x.device)])
        x, _ = torch.sort(x.reshape(b1 - b0, qb * k), dim=1)
        new = torch.ones_like(x, dtype=torch.bool)
        new[:, 1:] = x[:, 1:] != x[:, :-1]
        per = ((x >= 0) & new).sum(dim=1)
        distinct += int(per.sum().item())
        chunked += int(((per + 63) // 64 * 64).sum().item())
    return distinct, chunked


def dedup_attn_cost(torch, cfg, idx):
    """Algorithmic cost of the adjacent-query dedup attention (blocks of
    128 / G queries): bytes = the K and V rows of every distinct key of a
    block, once per block, plus Q, O and the index rows; FLOPs = the two
    products of the 128-row tiles over each block's chunked key list, for
    every KV group."""
    qb = 128 // (cfg.Hq // cfg.Hkv)
    distinct, chunked = dedup_stats(torch, idx, qb)
    L, k = idx.shape
    by = distinct * 2 * cfg.Hkv * cfg.d * 2 + L * (2 * cfg.Hq * cfg.d * 2 + 4 * k)
    fl = 2.0 * 2 * 128 * cfg.d * chunked * cfg.Hkv
    return by, fl


def other_configs(torch, dsa, pk, args, stream, flush):
    """The other prefill workloads (tiny, 32K, 256K video), each timed as its
    own steps (indexer + top-k, then attention; the dedup attention on the
    video workload), with the same rooflines; min(steps, 5) timed steps."""
    out = {}
    fp8_peak = 2.0 * pk["bf16_sus"]
    l2pk = l2_read_peak(torch)
    for cfg in (gen.TINY_PREFILL, gen.PREFILL_32K, gen.VIDEO_256K):
        h = gen.prefill_inputs(cfg)
        t = {n: torch.from_numpy(h[n]).cuda() for n in ("q_I", "k_I", "w")}
        bf = {n: torch.from_numpy(h[n].view(np.int16)).view(torch.bfloat16).cuda()
              for n in ("Q", "K", "V")}
        del h
        idx = torch.empty((cfg.L, cfg.k), dtype=torch.int32, device="cuda")
        O = torch.empty_like(bf["Q"])
        attn = dsa.sparse_attn_prefill_dedup if cfg.video else dsa.sparse_attn_prefill
        kw = {}
        if cfg.video:
            kw["workspace"] = torch.empty(dsa.dedup_workspace_size(cfg.L, cfg.Hq, cfg.Hkv, cfg.d,
                                                                   cfg.k),
                                          dtype=torch.uint8, device="cuda")

        def step(ev=None):
            if ev:
                ev[0].record(stream)
            dsa.index_topk(t["q_I"], t["k_I"], t["w"], cfg.k, idx=idx, stream=stream)
            if ev:
                ev[1].record(stream)
            attn(bf["Q"], bf["K"], bf["V"], idx, cfg.scale, O=O, stream=stream, **kw)
            if ev:
                ev[2].record(stream)

        for _ in range(max(1, args.warmup)):
            flush.zero_()
            step()
        n = max(1, min(args.steps, 5))
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
        for i in range(n):
            flush.zero_()
            step(evs[i])
        torch.cuda.synchronize()
        if dsa.device_error() != 0:
            raise RuntimeError(f"device error in the {cfg.name} workload")
        mi = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
        ma = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        fl, by = prefill_flops(cfg), prefill_attn_bytes(cfg)
        afl = None
        if cfg.video:  # the dedup kernel gathers each distinct key of a block once
            by, afl = dedup_attn_cost(torch, cfg, idx)
        out[cfg.name] = dict(
            steps=n, ms_per_step=mi + ma, value=cfg.L / ((mi + ma) / 1e3),
            unit="query-tokens/s",
            kernels={"dsa_index_topk": dict(bound="tensor", ms=mi, achieved=fl / (mi / 1e3) / 1e12,
                                            peak=fp8_peak, unit="TFLOP/s",
                                            frac=fl / (mi / 1e3) / 1e12 / fp8_peak,
                                            **fp8_alt_peaks(torch, fl / (mi / 1e3) / 1e12)),
                     attn.__name__: dict(bound="l2", ms=ma, achieved=by / (ma / 1e3) / 1e9,
                                         peak=l2pk, unit="GB/s",
                                         frac=by / (ma / 1e3) / 1e9 / l2pk)})
        if afl is not None:  # the dedup kernel's tensor work, against the bf16 peak
            out[cfg.name]["kernels"][attn.__name__]["tensor"] = dict(
                achieved=afl / (ma / 1e3) / 1e12, peak=pk["bf16_sus"], unit="TFLOP/s",
                frac=afl / (ma / 1e3) / 1e12 / pk["bf16_sus"])
        del t, bf, idx, O, kw
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ one workload on N GPUs

def run_sharded(args, rank, world, local_rank):
    """One workload shared by the N ranks (strong scaling).  Prefill: the
    query rows in zig-zag blocks, one NCCL exchange step (all-gather of the
    blocks of k_I, K and V) and then each rank's selection and attention for
    its rows.  Decode: batch shards (each rank its own sequences), or cache
    shards (each rank part of every sequence, two all-gathers).  The step
    time is the max over ranks of each rank's device time."""
    import torch
    import torch.distributed as tdist
    import sparse_long_context_02_b200 as dsa
    from sparse_long_context_02_b200 import dist, shards

    torch.cuda.set_device(local_rank)
    pcfg = gen.CONFIGS[args.prefill_config] if args.prefill_config else None
    if pcfg is not None and args.prefill_L:
        pcfg = pcfg.with_(L=args.prefill_L, name=f"{pcfg.name} at L={args.prefill_L}")
    dcfg = gen.CONFIGS[args.decode_config] if args.decode_config else None
    if dcfg is not None and args.decode_batch:
        dcfg = dcfg.with_(B=args.decode_batch)
    stream = torch.cuda.current_stream()
    dev = torch.device("cuda", local_rank)
    bf = torch.bfloat16

    e2e_on = not args.no_e2e
    h2d = []  # (pinned host, device) pairs of the rank's inputs, for the e2e leg

    def t_(a, dt=None, inp=True):
        x = torch.from_numpy(np.ascontiguousarray(a))
        x = x.view(dt) if dt is not None else x
        if e2e_on and inp:
            x = x.pin_memory()
            d_ = x.to(dev)
            h2d.append((x, d_))
            return d_
        return x.to(dev)

    # ---- prefill: this rank's rows and key blocks
    Pf = {}
    if pcfg:
        L = pcfg.L
        blocks = shards.zigzag_blocks(L, world)
        blk = blocks[0][1] - blocks[0][0]
        rows = shards.zigzag_rows(L, world, rank)
        mine = {n: [] for n in ("q_I", "w", "Q", "idx", "O")}
        own = {n: [] for n in ("k_I", "K", "V")}
        for b in (rank, 2 * world - 1 - rank):
            a, z = blocks[b]
            n = z - a
            pad = lambda x: np.concatenate([x, np.zeros((blk - n,) + x.shape[1:], x.dtype)])  # noqa: E731
            mine["q_I"].append(t_(pad(gen.prefill_qI(pcfg, a, z))))
            mine["w"].append(t_(pad(gen.prefill_w(pcfg, a, z))))
            mine["Q"].append(t_(pad(gen.prefill_Q(pcfg, a, z)).view(np.int16), bf))
            mine["idx"].append(torch.empty((blk, pcfg.k), dtype=torch.int32, device=dev))
            mine["O"].append(torch.empty((blk, pcfg.Hq, pcfg.d), dtype=bf, device=dev))
            own["k_I"].append(t_(pad(gen.prefill_kI(pcfg, a, z))))
            own["K"].append(t_(pad(gen.prefill_K(pcfg, a, z)).view(np.int16), bf))
            own["V"].append(t_(pad(gen.prefill_V(pcfg, a, z)).view(np.int16), bf))
        keys = dict(k_I=torch.empty((2 * world * blk, pcfg.d_I), dtype=torch.uint8, device=dev),
                    K=torch.empty((2 * world * blk, pcfg.Hkv, pcfg.d), dtype=bf, device=dev),
                    V=torch.empty((2 * world * blk, pcfg.Hkv, pcfg.d), dtype=bf, device=dev))
        Pf = dict(rows=rows, mine=mine, own=own, keys=keys)

    # ---- decode: batch shards or cache shards
    Df = {}
    if dcfg:
        off = gen.decode_offsets(dcfg)
        lens = np.diff(off)
        q = gen.decode_queries(dcfg)

        def cache_rows(segs):
            """Packed cache of (global start, length) pieces, in order."""
            n = int(sum(m for _, m in segs))
            kI = torch.empty((n, dcfg.d_I), dtype=torch.uint8, device=dev)
            K = torch.empty((n, dcfg.Hkv, dcfg.d), dtype=bf, device=dev)
            V = torch.empty_like(K)
            at = 0
            for s0, m in segs:
                for c0 in range(0, m, 1 << 19):
                    c1 = min(m, c0 + (1 << 19))
                    r0, r1 = s0 + c0, s0 + c1
                    kI[at + c0:at + c1].copy_(torch.from_numpy(gen.decode_kI_rows(dcfg, r0, r1)))
                    K[at + c0:at + c1].copy_(torch.from_numpy(
                        gen.decode_K_rows(dcfg, r0, r1).view(np.int16)).view(bf))
                    V[at + c0:at + c1].copy_(torch.from_numpy(
                        gen.decode_V_rows(dcfg, r0, r1).view(np.int16)).view(bf))
                at += m
            return kI, K, V

        if args.decode_shard == "batch":
            seqs = dist.deal_sequences(lens, world)[rank]
            kI, K, V = cache_rows([(int(off[b]), int(lens[b])) for b in seqs])
            off_r = np.concatenate([[0], np.cumsum(lens[seqs])]).astype(np.int64)
            if not seqs:
                off_r = np.zeros(1, np.int64)
            Df = dict(mode="batch", seqs=seqs, q_I=t_(q["q_I"][seqs]), w=t_(q["w"][seqs]),
                      Q=t_(q["Q"][seqs].view(np.int16), bf), kI=kI, K=K, V=V, off=t_(off_r),
                      O=torch.empty((len(seqs), dcfg.Hq, dcfg.d), dtype=bf, device=dev),
                      idx=torch.empty((len(seqs), dcfg.k), dtype=torch.int32, device=dev))
            Df["ws"] = torch.empty(dsa.decode_workspace_size(
                len(seqs), int(off_r[-1]), dcfg.H_I, dcfg.d_I, dcfg.k, dcfg.Hq, dcfg.Hkv, dcfg.d),
                dtype=torch.uint8, device=dev)
        else:
            part = shards.cache_parts(lens, world)[rank]
            kI, K, V = cache_rows([(int(off[b]) + int(part["base"][b]), int(part["lens"][b]))
                                   for b in range(dcfg.B)])
            Df = dict(mode="cache", q_I=t_(q["q_I"]), w=t_(q["w"]), Q=t_(q["Q"].view(np.int16), bf),
                      kI=kI, K=K, V=V, off=t_(part["off"]), base=t_(part["base"]), work={})

    def prefill():
        if not Pf:
            return
        for name in ("k_I", "K", "V"):
            dist.gather_zigzag(Pf["own"][name], Pf["keys"][name], pcfg.L, world)
        dist.prefill_rows_step(dsa, Pf["rows"], Pf["mine"], Pf["keys"], pcfg.k, pcfg.scale,
                               stream=stream)

    def decode():
        if not Df:
            return
        if Df["mode"] == "batch":
            if Df["seqs"]:
                dsa.sparse_attn_decode(Df["q_I"], Df["w"], Df["Q"], Df["kI"], Df["K"], Df["V"],
                                       Df["off"], dcfg.k, dcfg.scale, O=Df["O"],
                                       idx_out=Df["idx"], workspace=Df["ws"], stream=stream)
        else:
            dist.decode_cache_step(dsa, Df["q_I"], Df["w"], Df["Q"], Df["kI"], Df["K"], Df["V"],
                                   Df["off"], Df["base"], dcfg.k, dcfg.scale, world,
                                   stream=stream, work=Df["work"])

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        prefill()
        decode()
    torch.cuda.synchronize()
    if dsa.device_error() != 0:
        raise RuntimeError("device error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = Clocks(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ
                    else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    tdist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        prefill()
        evs[i][1].record(stream)
        decode()
        evs[i][2].record(stream)
    torch.cuda.synchronize()
    tdist.barrier()
    clk = clocks.stop()
    if dsa.device_error() != 0:
        raise RuntimeError("device error in the timed region")
    t_p = sum(e[0].elapsed_time(e[1]) for e in evs)
    t_d = sum(e[1].elapsed_time(e[2]) for e in evs)
    tot = max_over_ranks([t_p, t_d], world, device=dev)
    K_ = args.steps
    prefill_ms, decode_ms = tot[0] / K_, tot[1] / K_

    # ---- end to end: every step copies the rank's inputs from pinned host
    # memory and its output rows back
    e2e = None
    if e2e_on:
        outs = (Pf["mine"]["O"] if Pf else []) + ([Df["O"]] if Df.get("mode") == "batch" else [])
        d2h = [(torch.empty(o.shape, dtype=o.dtype).pin_memory(), o) for o in outs]
        ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_)]
        tdist.barrier()
        torch.cuda.synchronize()
        for i in range(K_):
            flush.zero_()
            ev2[i][0].record(stream)
            for h, d_ in h2d:
                d_.copy_(h, non_blocking=True)
            prefill()
            decode()
            for h, d_ in d2h:
                h.copy_(d_, non_blocking=True)
            ev2[i][1].record(stream)
        torch.cuda.synchronize()
        tdist.barrier()
        et = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in ev2)], world, device=dev)[0]
        bi = sum(h.numel() * h.element_size() for h, _ in h2d)
        bo = sum(h.numel() * h.element_size() for h, _ in d2h)
        e2e = dict(value=(pcfg.L / (et / K_ / 1e3)) if pcfg else 0.0, unit="query-tokens/s",
                   h2d_bytes_per_step=int(bi), d2h_bytes_per_step=int(bo),
                   ms_per_step=float(et / K_), note="rank 0's bytes; every rank copies its own")
    launches = (4 if pcfg else 0) + (4 if (dcfg and args.decode_shard == "batch") else
                                     (6 if dcfg else 0))
    par = []
    if pcfg:
        par.append(f"prefill: {2 * world} zig-zag row blocks, NCCL all-gather of k_I/K/V")
    if dcfg:
        par.append("decode: batch shards" if args.decode_shard == "batch" else
                   "decode: cache shards, NCCL all-gather of top-k pairs and partials")
    return dict(value=(pcfg.L / (prefill_ms / 1e3)) if pcfg else 0.0, prefill_ms=prefill_ms,
                decode_ms=decode_ms, decode_tps=(dcfg.B / (decode_ms / 1e3)) if dcfg else 0.0,
                clocks=clk, launches=launches * K_, pcfg=pcfg, dcfg=dcfg, parallelism="; ".join(par),
                e2e=e2e)


# ------------------------------------------------------------------ oracle timing

def sample_rows(L, n, seed=0):
    """n query rows stratified over [0, L): the sample's mean causal length
    matches the whole sequence's."""
    rng = np.random.default_rng(seed)
    return np.array(sorted(int((i + rng.random()) * L / n) for i in range(n)), np.int64)


def oracle_prefill_rows(pcfg, host, rows, nthreads=0):
    import oracle
    idx = oracle.index_topk(host["q_I"], host["k_I"], host["w"], pcfg.k, rows=rows,
                            nthreads=nthreads)
    oracle.sparse_attn(host["Q"], host["K"], host["V"], idx, pcfg.scale, rows=rows,
                       nthreads=nthreads, idx_by_row=True)


def cpu_baseline(pcfg, host, seconds, dcfg=None):
    """The oracle on this host's cores: prefill rows per second on a
    stratified sample of the workload's rows (the sample's mean causal length
    matches the sequence's, so the rate extrapolates to the whole prefill by
    the row count), and decode tokens per second on the decode workload's two
    shortest sequences (extrapolated to the batch by cached rows)."""
    cores = os.cpu_count() or 1
    # calibrate on a small stratified sample, then size the timed sample
    probe = sample_rows(pcfg.L, max(cores, 8), seed=1)
    t0 = time.perf_counter()
    oracle_prefill_rows(pcfg, host, probe)
    dt = time.perf_counter() - t0
    n = int(max(cores, min(16 * cores, len(probe) * seconds / max(dt, 1e-3))))
    rows = sample_rows(pcfg.L, n, seed=2)
    t0 = time.perf_counter()
    oracle_prefill_rows(pcfg, host, rows)
    dt = time.perf_counter() - t0
    out = dict(value=n / dt, unit="query-tokens/s", cores=cores, kind="oracle",
               extrapolated=True, rows=n,
               sample=f"{n} query rows stratified over t in [0, {pcfg.L}) of the "
                      f"{pcfg.name} workload (indexer + top-k + attention per row), "
                      f"{dt:.1f} s; rate extrapolated to all {pcfg.L} rows")
    if dcfg is not None:
        import oracle
        off = gen.decode_offsets(dcfg)
        lens = np.diff(off)
        seqs = [int(b) for b in np.argsort(lens)[:2]]
        q = gen.decode_queries(dcfg)
        sub = np.concatenate([[0], np.cumsum(lens[seqs])]).astype(np.int64)
        kI = np.concatenate([gen.decode_kI_rows(dcfg, off[b], off[b + 1]) for b in seqs])
        K = np.concatenate([gen.decode_K_rows(dcfg, off[b], off[b + 1]) for b in seqs])
        V = np.concatenate([gen.decode_V_rows(dcfg, off[b], off[b + 1]) for b in seqs])
        t0 = time.perf_counter()
        oracle.decode(q["q_I"][seqs], q["w"][seqs], q["Q"][seqs], kI, K, V, sub, dcfg.k,
                      dcfg.scale)
        dd = time.perf_counter() - t0
        rows_per_s = float(sub[-1]) / dd
        out["decode"] = dict(value=rows_per_s / float(lens.sum()) * dcfg.B, unit="tokens/s",
                             extrapolated=True,
                             sample=f"sequences {seqs} ({int(sub[-1])} cached rows), {dd:.1f} s; "
                                    f"rate per cached row extrapolated to the batch's "
                                    f"{int(lens.sum())} rows")
    return out


def workload_config(pcfg, dcfg, world=1):
    names = [c.name for c in (pcfg, dcfg) if c is not None]
    c = dict(workload=" + ".join(names), parallelism=f"independent problem per rank x{world}",
             l2="flushed between timed steps (256 MiB write, outside the events)")
    if pcfg is not None:
        c.update(prefill_L=pcfg.L, k=pcfg.k, H_I=pcfg.H_I, d_I=pcfg.d_I, Hq=pcfg.Hq,
                 Hkv=pcfg.Hkv, d=pcfg.d)
    if dcfg is not None:
        c.update(decode_B=dcfg.B, decode_n=f"U[{dcfg.n_lo},{dcfg.n_hi}]", k=dcfg.k)
    return c


def run_reference(args):
    pcfg = gen.CONFIGS[args.prefill_config or gen.PREFILL_128K.id]
    host = gen.prefill_inputs(pcfg)
    cores = os.cpu_count() or 1
    probe = sample_rows(pcfg.L, max(cores, 8), seed=1)
    t0 = time.perf_counter()
    oracle_prefill_rows(pcfg, host, probe)
    dt = time.perf_counter() - t0
    n = int(max(cores, min(16 * cores, len(probe) * 8.0 / max(dt, 1e-3))))
    for w in range(args.warmup):
        oracle_prefill_rows(pcfg, host, sample_rows(pcfg.L, max(1, n // 4), seed=100 + w))
    times = []
    for i in range(args.steps):
        rows = sample_rows(pcfg.L, n, seed=10 + i)
        t0 = time.perf_counter()
        oracle_prefill_rows(pcfg, host, rows)
        times.append(time.perf_counter() - t0)
    value = n * args.steps / sum(times)
    sample = (f"{n} query rows per step, stratified over t in [0, {pcfg.L}) of the {pcfg.name} "
              f"workload (indexer + top-k + attention per row); the oracle's throughput on the "
              f"prefill part, in the unit of `value`")
    return dict(impl="reference", metric=METRIC, value=value, unit="query-tokens/s",
                n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                ms_per_step=1e3 * sum(times) / args.steps, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                config=workload_config(pcfg, gen.CONFIGS[args.decode_config]
                                       if args.decode_config else None),
                cpu_baseline=dict(value=value, unit="query-tokens/s", cores=cores, kind="oracle",
                                  sample=sample),
                e2e=dict(value=value, unit="query-tokens/s", h2d_bytes_per_step=0,
                         d2h_bytes_per_step=0))


def union_stats(args) -> dict:
    """Distinct keys selected by blocks of G consecutive query rows, over the
    rows whose index sets are full (t + 1 >= k): the rows an adjacent-query
    dedup would gather once per block instead of once per row."""
    import torch
    import sparse_long_context_02_b200 as dsa
    G = args.union_stats
    cfg = gen.CONFIGS[args.prefill_config]
    host = gen.prefill_inputs(cfg)
    idx = dsa.index_topk(torch.from_numpy(host["q_I"]).cuda(), torch.from_numpy(host["k_I"]).cuda(),
                         torch.from_numpy(host["w"]).cuda(), cfg.k)
    t0 = (cfg.k + G - 1) // G * G  # first block of full rows
    nb = (cfg.L - t0) // G
    fr = []
    for b0 in range(0, nb, 1024):  # blocks in batches (sorting needs memory)
        b1 = min(nb, b0 + 1024)
        x = idx[t0 + b0 * G:t0 + b1 * G].reshape(b1 - b0, G * cfg.k)
        x, _ = torch.sort(x, dim=1)
        distinct = 1 + (x[:, 1:] != x[:, :-1]).sum(dim=1)
        fr.append(distinct.float() / (G * cfg.k))
    fr = torch.cat(fr).cpu().numpy()
    return dict(metric="distinct selected keys per block of %d queries / (%d k)" % (G, G),
                workload=cfg.name, blocks=int(nb), mean=float(fr.mean()),
                p10=float(np.percentile(fr, 10)), p50=float(np.percentile(fr, 50)),
                p90=float(np.percentile(fr, 90)), k=cfg.k, data="synthetic")


def kl_flops(L, H_I, d_I, Hq, d):
    """Algorithmic tensor work of the warm-up loss per causal (t, s) pair:
    forward = indexer scores (FP8, 2 H_I d_I) + two passes over the attention
    scores (bf16, 2 x 2 Hq d); backward = the indexer scores again in each of
    its two kernels (FP8, 2 x 2 H_I d_I) + the dS products with k_I and q_I
    (bf16, 2 x 2 H_I d_I)."""
    pairs = L * (L + 1) / 2.0
    return dict(fwd_fp8=pairs * 2 * H_I * d_I, fwd_bf16=pairs * 2 * 2 * Hq * d,
                bwd_fp8=pairs * 2 * 2 * H_I * d_I, bwd_bf16=pairs * 2 * 2 * H_I * d_I)


def kl_bench(args) -> dict:
    """Times dsa_indexer_kl_forward and dsa_indexer_kl_backward with CUDA events
    (L2 flushed before each step), reports tokens/s of forward + backward and
    the tensor roofline of each call: the time its FP8 and bf16 work would
    take at the measured peaks, divided by the measured time."""
    import torch
    import sparse_long_context_02_b200 as dsa
    L = args.kl
    base = gen.PREFILL_128K
    cfg = gen.custom(L=L, H_I=base.H_I, d_I=base.d_I, k=8, Hq=base.Hq, Hkv=base.Hkv, d=base.d,
                     seed=51)
    host = gen.prefill_inputs(cfg)
    q, kI, w = (torch.from_numpy(host[n]).cuda() for n in ("q_I", "k_I", "w"))
    Q, K = (torch.from_numpy(host[n].view(np.int16)).view(torch.bfloat16).cuda() for n in ("Q", "K"))
    scale_I = 1.0 / 2048
    kl = torch.empty(L, dtype=torch.float32, device="cuda")
    G = torch.empty((L, L), dtype=torch.float32, device="cuda")
    ws = torch.empty(dsa.indexer_kl_workspace_size(L, cfg.Hq), dtype=torch.uint8, device="cuda")
    dq = torch.empty((L, cfg.H_I, cfg.d_I), dtype=torch.float32, device="cuda")
    dk = torch.empty((L, cfg.d_I), dtype=torch.float32, device="cuda")
    dw = torch.empty((L, cfg.H_I), dtype=torch.float32, device="cuda")
    wsb = torch.empty(dsa.lib().dsa_indexer_kl_backward_workspace_size(L, cfg.H_I, cfg.d_I),
                      dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def step(ev=None):
        if ev:
            ev[0].record()
        dsa.indexer_kl_forward(q, kI, w, Q, K, cfg.scale, scale_I, kl=kl, G=G, workspace=ws)
        if ev:
            ev[1].record()
        dsa.indexer_kl_backward(q, kI, w, G, dq_I=dq, dk_I=dk, dw=dw, workspace=wsb)
        if ev:
            ev[2].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = Clocks(torch.cuda.current_device())
    clocks.start()
    tf, tb = [], []
    for _ in range(args.steps):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        step(ev)
        torch.cuda.synchronize()
        tf.append(ev[0].elapsed_time(ev[1]))
        tb.append(ev[1].elapsed_time(ev[2]))
    ck = clocks.stop()
    if dsa.device_error() != dsa.DEVERR_NONE:
        raise RuntimeError("device error during the KL loss")
    pk = peaks()
    fp8_peak = 2 * pk["bf16_sus"]  # TFLOP/s
    bf16_peak = pk["bf16_sus"]
    fl = kl_flops(L, cfg.H_I, cfg.d_I, cfg.Hq, cfg.d)
    ms_f, ms_b = float(np.mean(tf)), float(np.mean(tb))

    def roof(ms, f8, b16):
        ideal_ms = (f8 / (fp8_peak * 1e12) + b16 / (bf16_peak * 1e12)) * 1e3
        return dict(bound="tensor", ms=ms, flops=f8 + b16,
                    achieved=(f8 + b16) / (ms * 1e-3) / 1e12, unit="TFLOP/s",
                    ideal_ms=ideal_ms, frac=ideal_ms / ms)

    return dict(metric="indexer warm-up KL loss, forward + backward tokens/s",
                value=L / ((ms_f + ms_b) * 1e-3), unit="tokens/s", higher_is_better=True,
                steps=args.steps, warmup=args.warmup, dtype="fp8-e4m3/bf16", data="synthetic",
                config=dict(workload="indexer KL loss L=%d" % L, L=L, H_I=cfg.H_I, d_I=cfg.d_I,
                            Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, scale_I=scale_I,
                            l2="flushed before each step (256 MiB write, outside the events)"),
                forward=roof(ms_f, fl["fwd_fp8"], fl["fwd_bf16"]),
                backward=roof(ms_b, fl["bwd_fp8"], fl["bwd_bf16"]),
                peaks=dict(fp8_tflops=fp8_peak, bf16_tflops=bf16_peak,
                           source=pk["src"] + " (bf16 sustained; fp8 = 2 x bf16)"),
                clocks=ck, mean_kl=float(kl.mean().item()))


def attn_bwd_bytes(cfg) -> float:
    """Backward traffic the method itself implies: per selected row the K and
    V rows gathered (2 * Hkv * d * 2 B) and the fp32 reductions into dK and
    dV (2 * Hkv * d * 4 B); per token Q, O and dO (3 * Hq * d * 2 B), lse
    (Hq * 4 B), the index row (4 k B) and dQ (Hq * d * 4 B)."""
    L, k = cfg.L, cfg.k
    sel = k * L - k * (k - 1) / 2.0 if L >= k else L * (L + 1) / 2.0
    row = 2 * cfg.Hkv * cfg.d * (2 + 4)
    per_tok = 3 * cfg.Hq * cfg.d * 2 + cfg.Hq * 4 + 4 * k + cfg.Hq * cfg.d * 4
    return sel * row + L * per_tok


def attn_bwd_bench(args) -> dict:
    """Times the forward (with lse) and dsa_sparse_attn_backward on the prefill
    workload's own index rows (from dsa_index_topk) with a seeded dO; L2
    flushed before each timed call."""
    import torch
    import sparse_long_context_02_b200 as dsa
    cfg = gen.CONFIGS[args.prefill_config]
    host = gen.prefill_inputs(cfg)
    t = {n: torch.from_numpy(host[n]).cuda() for n in ("q_I", "k_I", "w")}
    bf = {n: torch.from_numpy(host[n].view(np.int16)).view(torch.bfloat16).cuda()
          for n in ("Q", "K", "V")}
    idx = dsa.index_topk(t["q_I"], t["k_I"], t["w"], cfg.k)
    dO = torch.from_numpy(gen.normal_bf16(cfg.seed_ + 777, 99, 0, bf["Q"].numel()).view(
        np.int16)).view(torch.bfloat16).reshape(bf["Q"].shape).cuda()
    O = torch.empty_like(bf["Q"])
    lse = torch.empty((cfg.L, cfg.Hq), dtype=torch.float32, device="cuda")
    dQ = torch.empty((cfg.L, cfg.Hq, cfg.d), dtype=torch.float32, device="cuda")
    dK = torch.empty((cfg.L, cfg.Hkv, cfg.d), dtype=torch.float32, device="cuda")
    dV = torch.empty_like(dK)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def fwd():
        dsa.sparse_attn_prefill(bf["Q"], bf["K"], bf["V"], idx, cfg.scale, O=O, lse=lse)

    def bwd():
        dsa.sparse_attn_backward(bf["Q"], bf["K"], bf["V"], idx, O, lse, dO, cfg.scale,
                                 dQ=dQ, dK=dK, dV=dV)

    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    clocks = Clocks(torch.cuda.current_device())
    clocks.start()
    tf, tb = [], []
    for _ in range(args.steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        flush.zero_()
        ev[0].record()
        fwd()
        ev[1].record()
        flush.zero_()
        ev[2].record()
        bwd()
        ev[3].record()
        torch.cuda.synchronize()
        tf.append(ev[0].elapsed_time(ev[1]))
        tb.append(ev[2].elapsed_time(ev[3]))
    ck = clocks.stop()
    if dsa.device_error() != dsa.DEVERR_NONE:
        raise RuntimeError("device error in the attention backward")
    pk = peaks()
    ms_b = float(np.mean(tb))
    work = attn_bwd_bytes(cfg)
    return dict(metric="sparse attention backward query-tokens/s", value=cfg.L / (ms_b * 1e-3),
                unit="query-tokens/s", higher_is_better=True, steps=args.steps,
                warmup=args.warmup, dtype="bf16/fp32", data="synthetic",
                config=dict(workload=cfg.name + " (attention backward)", L=cfg.L, k=cfg.k,
                            Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d,
                            l2="flushed before each timed call (256 MiB write)"),
                forward_ms=float(np.mean(tf)), backward_ms=ms_b,
                roofline=dict(bound="hbm", achieved=work / (ms_b * 1e-3) / 1e9, peak=pk["hbm"],
                              unit="GB/s", frac=work / (ms_b * 1e-3) / 1e9 / pk["hbm"],
                              traffic=None, kernel="dsa_sparse_attn_backward",
                              work_bytes=work, peak_source=pk["src"] + " (hbm copy)"),
                clocks=ck, gpu_launches=3 * args.steps)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.union_stats:
        if rank == 0:
            print(json.dumps(union_stats(args)), flush=True)
        return
    if args.kl:
        if rank == 0:
            print(json.dumps(kl_bench(args)), flush=True)
        return
    if args.attn_bwd:
        if rank == 0:
            print(json.dumps(attn_bwd_bench(args)), flush=True)
        return

    import datetime
    import torch
    import torch.distributed as tdist
    if world > 1:
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                 device_id=torch.device("cuda", local_rank))
    try:
        if world > 1 and not args.replicas:
            r = run_sharded(args, rank, world, local_rank)
        else:
            r = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            tdist.destroy_process_group()
    if rank != 0:
        return
    if "parallelism" in r:
        pcfg, dcfg = r["pcfg"], r["dcfg"]
        cfg = workload_config(pcfg, dcfg, world)
        cfg["parallelism"] = r["parallelism"]
        print(json.dumps(dict(
            metric=METRIC, value=r["value"], unit="query-tokens/s", n_gpus=world,
            steps=args.steps, warmup=args.warmup, ms_per_step=r["prefill_ms"] + r["decode_ms"],
            higher_is_better=True, scaling="strong", vs_baseline=None, dtype="fp8-e4m3/bf16",
            data="synthetic", config=cfg,
            decode=dict(value=r["decode_tps"], unit="tokens/s", ms_per_step=r["decode_ms"]),
            prefill_ms=r["prefill_ms"], clocks=r["clocks"], gpu_launches=r["launches"],
            **({"e2e": r["e2e"]} if r["e2e"] else {}))), flush=True)
        return
    pcfg, dcfg = r["pcfg"], r["dcfg"]
    out = dict(
        metric=METRIC, value=r["value"], unit="query-tokens/s", n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=r["prefill_ms"] + r["decode_ms"],
        higher_is_better=True, scaling="weak", vs_baseline=None, dtype="fp8-e4m3/bf16",
        data="synthetic",
        config=workload_config(pcfg, dcfg, world),
        decode=dict(value=r["decode_tps"], unit="tokens/s", ms_per_step=r["decode_ms"]),
        prefill_ms=r["prefill_ms"],
        kernels=r["kernels"], roofline=r["roofline"], clocks=r["clocks"],
        gpu_launches=r["launches"],
    )
    if r["e2e"] is not None:
        out["e2e"] = r["e2e"]
    if r["cpu"] is not None:
        out["cpu_baseline"] = r["cpu"]
    if r.get("others"):
        out["configs"] = r["others"]
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
