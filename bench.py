"""Benchmark: prefix-sliding decode tokens/s and KV GB/s at W=4096 on B200.

One step = one pass of the hot path over one batch: append the new token of
each of B=8 sequences to its ring (ring write, eviction, position bookkeeping)
and run the decode attention for those 8 sequences (visible-range derivation,
split-K streaming of the prefix and window rows, split merge).  Workload:
16 query / 8 kv heads, head_dim 128, P=128, W=4096, bf16 with fp32
accumulation, every sequence past t=65536 so the window is full
(4224 visible rows, 138.4 MB of K/V read per step).  Steps rotate over 4
disjoint batches of 8 sequences (553 MB of resident K/V, more than 4x L2), so
every step streams from HBM.  The timed steps are replayed from one CUDA graph.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun each rank runs its own sequences (weak scaling, no collective on
the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefix-sliding decode tokens/s and KV GB/s (% of B200 HBM peak) at W=4096"
UNIT = "tokens/s"

B, HQ, HKV, D, P, W = 8, 16, 8, 128, 128, 4096
ROT = 4                     # disjoint batches rotated through
T_START = 65536             # decode positions start here (window full)
SEED = 0


def workload_config():
    n_vis = P + W
    return {"workload": f"decode B={B} Hq={HQ} Hkv={HKV} d={D} P={P} W={W} bf16, t>={T_START} "
                        f"(window full, {n_vis} visible rows)",
            "global_batch": B, "Hq": HQ, "Hkv": HKV, "head_dim": D, "P": P, "W": W,
            "t_start": T_START, "visible_rows": n_vis,
            "l2": f"inputs larger than L2: {ROT} disjoint batches of {B} sequences rotated "
                  f"({ROT * kv_bytes_per_step() / 1e6:.0f} MB resident K/V)"}


def rank_seed(rank: int) -> int:
    """Each rank decodes its own sequences: the inputs of rank r use seed SEED + 1000 r."""
    return SEED + 1000 * rank


def max_over_ranks(value: float, dist, device) -> float:
    """Largest value over all ranks (the job lasts as long as its slowest rank)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, steps: int, ms_total: float) -> float:
    """Whole-job decode throughput: B tokens per step on every rank."""
    return world * B * steps / (ms_total / 1e3)


def kv_bytes_per_seq():
    return HKV * (P + W) * D * 2 * 2          # K and V rows, bf16


def kv_bytes_per_step():
    return B * kv_bytes_per_seq()


def prefill_flops(Wp: int) -> float:
    """Visible (query, key) pairs of the chunk-prefill step, 4 d flops per pair per
    query head (Q K^T and P V): every query of a block at t0 = 100000 sees its
    P + W keys (the window is full)."""
    return 4.0 * D * HQ * PF_N * (PF_P + Wp) * PF_SEQS


def prompt_flops() -> float:
    """Visible pairs of the prompt-prefill step: prompt query t sees t + 1 keys."""
    return 4.0 * D * HQ * (PR_P * (PR_P + 1) / 2) * PF_SEQS


def decode_traffic():
    """DRAM bytes per decode launch from the committed ncu record, or None when
    the decode kernel's sources have changed since that capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for src in rec["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec["sources_sha256"]:
        return None
    return rec["dram_bytes_read_per_launch"] + rec["dram_bytes_write_per_launch"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j["hbm_gbs"], "measured"
    return 6650.0, "fallback"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ------------------------------------------------------------ clocks --------
class ClockSampler:
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
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for nm, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        busy = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------ our arm -------
class Workload:
    """Sequences, their synthetic histories and per-step inputs on one GPU."""

    def __init__(self, rank: int, steps_needed: int, prefix: int = P):
        import torch

        import synth
        from prefix_sliding_window_ring_b200 import PS_BF16, Cache

        self.torch = torch
        self.S = B * ROT
        self.seed = rank_seed(rank)
        self.kscale = synth.chan_scale(self.seed, HKV, D)
        self.P = prefix
        self.cache = Cache(W, max(prefix, 1), HKV, D, PS_BF16, self.S)
        self.scale = 1.0 / math.sqrt(D)

        def dev(a):
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

        self.dev = dev
        for s in range(self.S):
            kp = synth.rows(self.seed, synth.TID_K, s, HKV, 0, prefix, D, "bf16", self.kscale)
            vp = synth.rows(self.seed, synth.TID_V, s, HKV, 0, prefix, D, "bf16")
            self.cache.seq_reset(s, (s * 613) % W)
            self.cache.prefill_prefix(s, dev(kp), dev(vp), prefix)
            t0 = T_START + s  # staggered positions
            kw = synth.rows(self.seed, synth.TID_K, s, HKV, t0 - W, W, D, "bf16", self.kscale)
            vw = synth.rows(self.seed, synth.TID_V, s, HKV, t0 - W, W, D, "bf16")
            self.cache.import_window(s, t0, dev(kw), dev(vw), W, (s * 613) % W)
        torch.cuda.synchronize()
        self.next_pos = [T_START + s for s in range(self.S)]
        # per-step inputs: each batch group appends one token per sequence per visit
        visits = (steps_needed + ROT - 1) // ROT + 1
        self.kin, self.vin, self.qin = {}, {}, {}
        for s in range(self.S):
            p0 = self.next_pos[s]
            self.kin[s] = synth.rows(self.seed, synth.TID_K, s, HKV, p0, visits, D, "bf16", self.kscale)
            self.vin[s] = synth.rows(self.seed, synth.TID_V, s, HKV, p0, visits, D, "bf16")
            self.qin[s] = synth.rows(self.seed, synth.TID_Q, s, HQ, p0, visits, D, "bf16")
        # device pools [ROT][visits][B][H][D]
        self.visits = visits
        self.k_pool = [dev(np.stack([self.kin[r * B + b] for b in range(B)], axis=1)) for r in range(ROT)]
        self.v_pool = [dev(np.stack([self.vin[r * B + b] for b in range(B)], axis=1)) for r in range(ROT)]
        self.q_pool = [dev(np.stack([self.qin[r * B + b] for b in range(B)], axis=1)) for r in range(ROT)]
        self.out = [torch.empty((B, HQ, D), dtype=torch.bfloat16, device="cuda") for _ in range(ROT)]
        self.ws = self.cache.decode_workspace(B, HQ)
        self.visit = [0] * ROT

    def ids(self, r):
        return list(range(r * B, (r + 1) * B))

    def step(self, i, stream=None, host=None):
        """One hot-path step on batch group i % ROT: append each sequence's token
        and attend at it (ps_decode_step: ring append, visible ranges, split-K
        decode and split merge in one streaming launch plus the merge launch)."""
        r = i % ROT
        v = self.visit[r]
        ids = self.ids(r)
        ts = [self.next_pos[s] for s in ids]
        if host is None:
            k, vv, q = self.k_pool[r][v], self.v_pool[r][v], self.q_pool[r][v]
        else:
            k, vv, q = host(r, v)
        self.cache.decode_step(q, k, vv, ids, ts, HQ, self.scale, self.out[r], self.ws, stream)
        for s in ids:
            self.next_pos[s] += 1
        self.visit[r] += 1
        return self.out[r]

    def decode_only(self, i, stream=None):
        r = i % ROT
        ids = self.ids(r)
        ts = [self.next_pos[s] - 1 for s in ids]
        self.cache.attend_decode(self.q_pool[r][0], ids, ts, HQ, self.scale, self.out[r], self.ws,
                                 stream)


def _check_device(wl):
    code = wl.cache.device_error()
    if code:
        raise RuntimeError(f"device error word {code:#x} set by a kernel")


def upload_graph(torch, g, stream):
    """Upload an instantiated CUDA graph to the device before its timed replay.

    The first launch of a graph otherwise uploads it inside the launch, which
    costs several microseconds per node and would be counted as kernel time."""
    import ctypes
    rt = ctypes.CDLL("libcudart.so.12")  # the runtime torch has loaded
    rt.cudaGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    rt.cudaGraphUpload.restype = ctypes.c_int
    rc = rt.cudaGraphUpload(ctypes.c_void_p(int(g.raw_cuda_graph_exec())),
                            ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"cudaGraphUpload failed with error {rc}")
    torch.cuda.synchronize()


def graph_kernel_nodes(g) -> int:
    """Kernel nodes in a captured CUDA graph (captured with keep_graph=True):
    the launches of the library's kernels in the replayed steps."""
    import ctypes
    rt = ctypes.CDLL("libcudart.so.12")  # the runtime torch has loaded
    graph = ctypes.c_void_p(int(g.raw_cuda_graph()))
    n = ctypes.c_size_t(0)
    rt.cudaGraphGetNodes.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    if rt.cudaGraphGetNodes(graph, None, ctypes.byref(n)) != 0:
        raise RuntimeError("cudaGraphGetNodes failed")
    nodes = (ctypes.c_void_p * max(n.value, 1))()
    if rt.cudaGraphGetNodes(graph, nodes, ctypes.byref(n)) != 0:
        raise RuntimeError("cudaGraphGetNodes failed")
    rt.cudaGraphNodeGetType.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    kernels = 0
    for i in range(n.value):
        t = ctypes.c_int(-1)
        if rt.cudaGraphNodeGetType(ctypes.c_void_p(nodes[i]), ctypes.byref(t)) != 0:
            raise RuntimeError("cudaGraphNodeGetType failed")
        kernels += t.value == 0  # cudaGraphNodeTypeKernel
    return int(kernels)


def time_graph(torch, fn, n):
    """Capture n calls of fn(i) into one CUDA graph, upload it, replay it once,
    return ms per call."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(n):
            fn(i, s)
    torch.cuda.synchronize()
    upload_graph(torch, g, s)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del g
    return ms / n


def run_ours(args, rank, world, local_rank):
    import torch
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as td
        import datetime
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                              device_id=torch.device("cuda", local_rank))
        dist = td

    K, Wm = args.steps, args.warmup
    total_steps = Wm + K + K + K + 6
    wl = Workload(rank, total_steps)
    # warm-up (eager), also loads every kernel
    for i in range(Wm):
        wl.step(i)
    torch.cuda.synchronize()
    _check_device(wl)

    # ---- timed region: K steps replayed from one CUDA graph ----
    clocks = ClockSampler(local_rank) if rank == 0 else None
    if clocks:
        clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph(keep_graph=True)
    base = Wm
    with torch.cuda.graph(g, stream=s):
        for i in range(K):
            wl.step(base + i, s)
    torch.cuda.synchronize()
    launches = graph_kernel_nodes(g)  # the library's kernels in the K timed steps
    g.instantiate()
    upload_graph(torch, g, s)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    ms_total = e0.elapsed_time(e1)
    del g
    ms_total = max_over_ranks(ms_total, dist, "cuda")
    clk = clocks.stop() if clocks else None
    _check_device(wl)
    ms_step = ms_total / K
    value = job_tokens_per_s(world, K, ms_total)

    # ---- dominant kernel (decode) timed on its own stream, rotating batches ----
    ms_dec = time_graph(torch, lambda i, st: wl.decode_only(i, st), max(K, 4 * ROT))
    bytes_launch = kv_bytes_per_step()
    achieved = bytes_launch / (ms_dec / 1e3) / 1e9
    peak, peak_kind = load_peaks()

    # ---- prefix overhead: the same decode with no pinned prefix (plain sliding window) ----
    overhead = None
    if rank == 0 and not args.no_prefill:
        wl0 = Workload(rank, 4, prefix=0)
        for i in range(4):
            wl0.decode_only(i)
        torch.cuda.synchronize()
        ms0 = time_graph(torch, lambda i, st: wl0.decode_only(i, st), max(K, 4 * ROT))
        _check_device(wl0)
        bytes0 = B * HKV * W * D * 2 * 2
        overhead = {"note": "decode kernel, same W and batch; P=0 is plain sliding-window attention",
                    "P128": {"us_per_launch": round(ms_dec * 1e3, 2), "visible_rows": P + W,
                             "GBps": round(achieved, 1)},
                    "P0": {"us_per_launch": round(ms0 * 1e3, 2), "visible_rows": W,
                           "GBps": round(bytes0 / (ms0 / 1e3) / 1e9, 1)},
                    "time_ratio": round(ms_dec / ms0, 4)}
        wl0.cache.close()
        del wl0
        torch.cuda.empty_cache()

    # ---- end to end through the public API with host buffers ----
    # Each step's inputs sit in one pinned host record [q | k | v] and cross
    # to the device in one copy; the call gets views of the device copy, and
    # its output is read back into pinned host memory, all on one stream.
    # The K steps -- upload, ps_decode_step, read-back, each step -- are
    # captured into one CUDA graph and replayed, as a serving loop would run
    # them; the same steps issued eagerly from Python are reported beside it
    # (there the host's issue path, not the device, sets the pace).
    nq, nk = B * HQ * D, B * HKV * D
    hin = [torch.cat([wl.q_pool[r].reshape(wl.visits, -1), wl.k_pool[r].reshape(wl.visits, -1),
                      wl.v_pool[r].reshape(wl.visits, -1)], dim=1).cpu().pin_memory()
           for r in range(ROT)]
    hout = torch.empty((B, HQ, D), dtype=torch.bfloat16).pin_memory()
    din = torch.empty(nq + 2 * nk, dtype=torch.bfloat16, device="cuda")
    dq = din[:nq].view(B, HQ, D)
    dk = din[nq:nq + nk].view(B, HKV, D)
    dv = din[nq + nk:].view(B, HKV, D)

    def e2e_step(i, stream=None):
        r = i % ROT
        v = wl.visit[r]
        din.copy_(hin[r][v], non_blocking=True)
        out = wl.step(i, stream, host=lambda r_, v_: (dk, dv, dq))
        hout.copy_(out, non_blocking=True)

    base = Wm + K
    for i in range(2):
        e2e_step(base + i)
    torch.cuda.synchronize()
    base += 2
    # Graph of the K steps with the copies on a second stream: the upload of
    # step i+1 (into the other of two input buffers) overlaps the decode of
    # step i, and the read-back of step i overlaps the decode of step i+1.
    # Every step still uploads its own inputs and reads back its own output.
    din2 = [din, torch.empty_like(din)]
    dviews = [(d[:nq].view(B, HQ, D), d[nq:nq + nk].view(B, HKV, D), d[nq + nk:].view(B, HKV, D))
              for d in din2]
    hout2 = [hout, torch.empty_like(hout).pin_memory()]
    s2 = torch.cuda.Stream()
    s_in = torch.cuda.Stream()   # uploads
    s_out = torch.cuda.Stream()  # read-backs (the other copy direction, concurrently)
    for x_ in (s2, s_in, s_out):
        x_.wait_stream(torch.cuda.current_stream())
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=s2):
        s_in.wait_stream(s2)
        s_out.wait_stream(s2)
        ev_in = [torch.cuda.Event() for _ in range(K)]
        ev_dec = [torch.cuda.Event() for _ in range(K)]
        ev_out = [torch.cuda.Event() for _ in range(K)]
        for i in range(K):
            b = i % 2
            r = (base + i) % ROT
            v = wl.visit[r]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_dec[i - 2])  # input buffer b is free again
                din2[b].copy_(hin[r][v], non_blocking=True)
                ev_in[i].record(s_in)
            s2.wait_event(ev_in[i])
            if i >= 2:
                s2.wait_event(ev_out[i - 2])  # output buffer b has been read back
            qv, kv_, vv = dviews[b]
            out = wl.step(base + i, s2, host=lambda r_, v_: (kv_, vv, qv))
            ev_dec[i].record(s2)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_dec[i])
                hout2[b].copy_(out, non_blocking=True)
                ev_out[i].record(s_out)
        s2.wait_stream(s_in)
        s2.wait_stream(s_out)
    torch.cuda.synchronize()
    upload_graph(torch, g2, s2)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(s2):
        e0.record(s2)
        g2.replay()
        e1.record(s2)
    torch.cuda.synchronize()
    del g2
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), dist, "cuda")
    _check_device(wl)
    e2e_value = job_tokens_per_s(world, K, ms_e2e)
    base += K
    # the same steps issued eagerly, one Python call after another
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record()
    for i in range(K):
        e2e_step(base + i)
    e1.record()
    torch.cuda.synchronize()
    ms_eager = max_over_ranks(e0.elapsed_time(e1), dist, "cuda")
    _check_device(wl)
    e2e_eager = job_tokens_per_s(world, K, ms_eager)
    h2d = (B * HKV * D * 2) * 2 + B * HQ * D * 2
    d2h = B * HQ * D * 2

    prefill = None
    if rank == 0 and not args.no_prefill:
        prefill = prefill_measure(max(3, min(args.steps, 10)))
    ragged = shared = paged = t_sweep = gqa = None
    if rank == 0 and not args.no_prefill:
        ragged = ragged_measure(max(3, min(args.steps, 10)))
        gqa = gqa_measure(max(args.steps, 16))
        shared = shared_prefix_measure(max(3, min(args.steps, 10)))
        paged = paged_measure(max(3, min(args.steps, 10)))
        try:  # an extra section: a failure here is reported, not fatal to the line
            t_sweep = t_sweep_measure(max(args.steps, 16))
        except Exception as e:  # noqa: BLE001
            t_sweep = {"error": f"{type(e).__name__}: {e}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl.seed, wl.kscale, budget_s=args.cpu_seconds)

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**workload_config(), "parallelism": f"replicas x{world} (sequences sharded, no collective)"},
        "kv_gbs": round(kv_bytes_per_step() / (ms_step / 1e3) / 1e9, 1),
        "kv_frac_of_peak": round(kv_bytes_per_step() / (ms_step / 1e3) / 1e9 / peak, 4),
        "roofline": {"bound": "hbm", "kernel": "ps::k_decode_mma<128,2> (tensor-core decode; "
                               "the merge in-kernel in cluster mode, else k_decode_merge)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                     "bytes_per_launch": bytes_launch, "ms_per_launch": round(ms_dec, 5),
                     "traffic": decode_traffic()},
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "copies": "one upload of a pinned [q | k | v] record and one read-back of the "
                          "output per step, on the decode stream",
                "issue": "the K steps (upload, ps_decode_step, read-back) captured into one "
                         "CUDA graph and replayed; uploads and read-backs on two more streams, "
                         "double-buffered, overlapping the neighbouring steps' kernels",
                "eager": {"value": round(e2e_eager, 1), "unit": UNIT,
                          "issue": "the same steps issued one by one from Python"}},
        "gpu_launches": launches,  # kernel nodes of the timed graph (the K steps)
        "clocks": clk,
        "cpu_baseline": cpu,
        "prefill": prefill,
        "prefix_overhead": overhead,
        "ragged": ragged,
        "shared_prefix": shared,
        "paged": paged,
        "t_sweep": t_sweep,
        "gqa": gqa,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ prefill -------
PF_P, PF_N, PF_T0, PF_SEQS = 256, 2048, 100000, 4


def load_bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)["bf16_tflops"], "measured (burst)"
    return 1590.0, "fallback"


def prefill_measure(steps: int):
    """Chunked prefill/extend on the tensor-core kernel: 4 sequences, each a
    2048-query block at t0=100000 (window full), P=256, W in {4096, 16384}.
    One step = one ps_attend_chunk_batch call over the 4 blocks (packed).
    Throughput counts only visible (query, key) pairs:
    4 * d * Hq * sum over queries of (P + W) flops."""
    import torch

    import synth
    from prefix_sliding_window_ring_b200 import PS_BF16, Cache
    peak, peak_src = load_bf16_peak()

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    res = {"workload": f"{PF_SEQS} sequences x {PF_N}-query blocks at t0={PF_T0}, "
                       f"Hq={HQ} Hkv={HKV} d={D} P={PF_P}, bf16",
           "kernel": "ps::k_chunk_tc (tcgen05)", "peak": peak, "peak_source": peak_src,
           "unit": "TFLOP/s"}
    ids = list(range(PF_SEQS))
    for Wp in (4096, 16384):
        c = Cache(Wp, PF_P, HKV, D, PS_BF16, PF_SEQS)
        qs, kbs, vbs = [], [], []
        for s in range(PF_SEQS):
            c.seq_reset(s, 0)
            c.prefill_prefix(s, dev(synth.rows(SEED, synth.TID_K, s, HKV, 0, PF_P, D, "bf16")),
                             dev(synth.rows(SEED, synth.TID_V, s, HKV, 0, PF_P, D, "bf16")), PF_P)
            c.import_window(s, PF_T0,
                            dev(synth.rows(SEED, synth.TID_K, s, HKV, PF_T0 - Wp, Wp, D, "bf16")),
                            dev(synth.rows(SEED, synth.TID_V, s, HKV, PF_T0 - Wp, Wp, D, "bf16")),
                            Wp, (977 * s) % Wp)
            qs.append(dev(synth.rows(SEED, synth.TID_Q, s, HQ, PF_T0, PF_N, D, "bf16")))
            kbs.append(dev(synth.rows(SEED, synth.TID_K, s, HKV, PF_T0, PF_N, D, "bf16")))
            vbs.append(dev(synth.rows(SEED, synth.TID_V, s, HKV, PF_T0, PF_N, D, "bf16")))
        # the blocks packed end to end, as the batched call takes them
        q, kb, vb = torch.cat(qs), torch.cat(kbs), torch.cat(vbs)
        o = torch.empty_like(q)
        del qs, kbs, vbs
        scale = 1.0 / math.sqrt(D)

        def step(i, st=None):
            # one launch over the four sequences' query tiles
            c.attend_chunk_batch(ids, [PF_T0] * PF_SEQS, [PF_N] * PF_SEQS, q, kb, vb, HQ, scale,
                                 o, 0, st)

        for i in range(3):
            step(i)
        torch.cuda.synchronize()
        if c.device_error():
            raise RuntimeError("device error word set by the chunk kernel")
        ms = min(time_graph(torch, step, steps) for _ in range(2))
        flops = prefill_flops(Wp)
        tf = flops / (ms / 1e3) / 1e12
        res[f"W{Wp}"] = {"ms_per_step": round(ms, 4), "gflop_per_step": round(flops / 1e9, 1),
                         "achieved": round(tf, 1), "frac": round(tf / peak, 4)}
        c.close()
        del q, kb, vb, o
        torch.cuda.empty_cache()
    res["prompt"] = prompt_measure(steps, peak)
    return res


PR_P = 4096  # prompt length of the prompt-prefill measurement


def paged_prefill_measure(steps: int):
    """The chunk workload (4 sequences x 2048-query blocks at t0=100000,
    W=4096, P=256, Hq=16, Hkv=8, d=128, bf16) on an unpaged cache and on paged
    caches with 256-, 64- and 16-row pages (each window imported whole).
    One step = one ps_attend_chunk_batch call."""
    import torch

    import synth
    from prefix_sliding_window_ring_b200 import PS_BF16, Cache
    peak, _ = load_bf16_peak()

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    Wp = 4096
    ids = list(range(PF_SEQS))
    kw_ = dev(np.stack([synth.rows(SEED, synth.TID_K, s, HKV, PF_T0 - Wp, Wp, D, "bf16")
                        for s in range(PF_SEQS)]))
    vw_ = dev(np.stack([synth.rows(SEED, synth.TID_V, s, HKV, PF_T0 - Wp, Wp, D, "bf16")
                        for s in range(PF_SEQS)]))
    q = torch.cat([dev(synth.rows(SEED, synth.TID_Q, s, HQ, PF_T0, PF_N, D, "bf16"))
                   for s in range(PF_SEQS)])
    kb = torch.cat([dev(synth.rows(SEED, synth.TID_K, s, HKV, PF_T0, PF_N, D, "bf16"))
                    for s in range(PF_SEQS)])
    vb = torch.cat([dev(synth.rows(SEED, synth.TID_V, s, HKV, PF_T0, PF_N, D, "bf16"))
                    for s in range(PF_SEQS)])
    o = torch.empty_like(q)
    scale = 1.0 / math.sqrt(D)
    res = {"workload": f"{PF_SEQS} sequences x {PF_N}-query blocks at t0={PF_T0}, W={Wp}, "
                       f"P={PF_P}, Hq={HQ} Hkv={HKV} d={D}, bf16",
           "unit": "ms per call"}
    for page in (0, 256, 64, 16):
        c = Cache(Wp, PF_P, HKV, D, PS_BF16, PF_SEQS, page_rows=page,
                  num_pages=PF_SEQS * Wp // page if page else 0)
        for s in range(PF_SEQS):
            c.seq_reset(s, (977 * s) % Wp)
            c.prefill_prefix(s, dev(synth.rows(SEED, synth.TID_K, s, HKV, 0, PF_P, D, "bf16")),
                             dev(synth.rows(SEED, synth.TID_V, s, HKV, 0, PF_P, D, "bf16")), PF_P)
            c.import_window(s, PF_T0, kw_[s].contiguous(), vw_[s].contiguous(), Wp, (977 * s) % Wp)

        def step(i, st=None):
            c.attend_chunk_batch(ids, [PF_T0] * PF_SEQS, [PF_N] * PF_SEQS, q, kb, vb, HQ, scale,
                                 o, 0, st)

        for i in range(3):
            step(i)
        torch.cuda.synchronize()
        if c.device_error():
            raise RuntimeError("device error word set by a chunk call")
        ms = min(time_graph(torch, step, steps) for _ in range(2))
        tf = prefill_flops(Wp) / (ms / 1e3) / 1e12
        res[f"page_rows_{page}" if page else "unpaged"] = {
            "ms": round(ms, 4), "achieved_tflops": round(tf, 1), "frac": round(tf / peak, 4)}
        c.close()
    return res


def chunk_small_measure(steps: int):
    """Small chunk blocks: the split decode path against the chunk kernel.
    The chunk workload's shape (Hq=16, Hkv=8, d=128, P=256, W=4096, t0=100000,
    window full) with blocks of n queries for B = 1 and 4 sequences, each
    block size timed with the small-block bound at 0 (chunk kernel) and above
    n (split decode).  16 sequences' caches (285 MB, larger than L2) are
    rotated, a batch per step.  One step = one ps_attend_chunk_batch call."""
    import torch

    import synth
    from prefix_sliding_window_ring_b200 import PS_BF16, Cache

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    Wp, nseq = 4096, 16
    c = Cache(Wp, PF_P, HKV, D, PS_BF16, nseq)
    for s in range(nseq):
        c.seq_reset(s, 0)
        c.prefill_prefix(s, dev(synth.rows(SEED, synth.TID_K, s, HKV, 0, PF_P, D, "bf16")),
                         dev(synth.rows(SEED, synth.TID_V, s, HKV, 0, PF_P, D, "bf16")), PF_P)
        c.import_window(s, PF_T0,
                        dev(synth.rows(SEED, synth.TID_K, s, HKV, PF_T0 - Wp, Wp, D, "bf16")),
                        dev(synth.rows(SEED, synth.TID_V, s, HKV, PF_T0 - Wp, Wp, D, "bf16")),
                        Wp, (977 * s) % Wp)
    scale = 1.0 / math.sqrt(D)
    nmax = 64
    q = dev(synth.rows(SEED, synth.TID_Q, 0, HQ, PF_T0, 4 * nmax, D, "bf16"))
    kb = dev(synth.rows(SEED, synth.TID_K, 0, HKV, PF_T0, 4 * nmax, D, "bf16"))
    vb = dev(synth.rows(SEED, synth.TID_V, 0, HKV, PF_T0, 4 * nmax, D, "bf16"))
    o = torch.empty_like(q)
    res = {"workload": f"blocks of n queries at t0={PF_T0}, Hq={HQ} Hkv={HKV} d={D} P={PF_P} "
                       f"W={Wp}, bf16; 16 caches rotated (larger than L2)",
           "unit": "us per call", "rows": []}
    for B in (1, 4):
        for n in (1, 2, 3, 4, 8, 12, 16, 24, 32, 48, 64):
            row = {"B": B, "n": n}
            for name, bound in (("chunk_kernel", 0), ("split_decode", 1 << 20)):
                c.set_chunk_small_max(bound)

                def step(i, st=None):
                    ids = [((i % (nseq // B)) * B + b) for b in range(B)]
                    c.attend_chunk_batch(ids, [PF_T0] * B, [n] * B, q[:B * n], kb[:B * n],
                                         vb[:B * n], HQ, scale, o[:B * n], 0, st)

                for i in range(3):
                    step(i)
                torch.cuda.synchronize()
                if c.device_error():
                    raise RuntimeError("device error word set by a chunk call")
                ms = min(time_graph(torch, step, steps) for _ in range(2))
                row[name] = round(ms * 1e3, 2)
            res["rows"].append(row)
    c.set_chunk_small_max(0)
    for B in (1, 4):
        rows = [r for r in res["rows"] if r["B"] == B]
        faster = [r["n"] for r in rows if r["split_decode"] < r["chunk_kernel"]]
        res[f"split_faster_up_to_B{B}"] = max(faster) if faster else 0
    c.close()
    return res


def prompt_measure(steps: int, peak: float):
    """Prompt prefill (queries inside the pinned prefix, causal over it) on the
    tensor-core kernel: 4 sequences with a 4096-token prompt each, one
    ps_attend_prompt_batch call over the 4 prompts (packed).  Visible pairs only:
    4 * d * Hq * sum over t < P of (t + 1) flops per sequence."""
    import torch

    import synth
    from prefix_sliding_window_ring_b200 import PS_BF16, Cache

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    c = Cache(W, PR_P, HKV, D, PS_BF16, PF_SEQS)
    qs = []
    for s in range(PF_SEQS):
        c.prefill_prefix(s, dev(synth.rows(SEED, synth.TID_K, s, HKV, 0, PR_P, D, "bf16")),
                         dev(synth.rows(SEED, synth.TID_V, s, HKV, 0, PR_P, D, "bf16")), PR_P)
        qs.append(dev(synth.rows(SEED, synth.TID_Q, s, HQ, 0, PR_P, D, "bf16")))
    q = torch.cat(qs)  # the prompts packed end to end
    o = torch.empty_like(q)
    del qs
    scale = 1.0 / math.sqrt(D)
    ids = list(range(PF_SEQS))

    def step(i, st=None):
        c.attend_prompt_batch(ids, [0] * PF_SEQS, [PR_P] * PF_SEQS, q, HQ, scale, o, st)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    if c.device_error():
        raise RuntimeError("device error word set by the prompt kernel")
    ms = min(time_graph(torch, step, steps) for _ in range(2))
    flops = prompt_flops()
    tf = flops / (ms / 1e3) / 1e12
    c.close()
    del q, o
    torch.cuda.empty_cache()
    return {"workload": f"{PF_SEQS} sequences x {PR_P}-token prompt (causal over the pinned prefix), "
                        f"Hq={HQ} Hkv={HKV} d={D}, bf16",
            "ms_per_step": round(ms, 4), "gflop_per_step": round(flops / 1e9, 1),
            "achieved": round(tf, 1), "frac": round(tf / peak, 4)}


def ragged_measure(steps: int):
    """The ragged serving batch: 64 sequences with their own prefix lengths
    P_s ~ U[64, 512], positions t_s ~ U[P_s, 131072] and ring head offsets, one
    ps_decode_step per step (about 1.13 GB of visible K/V: larger than L2)."""
    import torch

    import synth
    from prefix_sliding_window_ring_b200 import PS_BF16, Cache
    from synth import workloads

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    draws = workloads.ragged_draws(0)
    S = len(draws)
    Pm = workloads.RAGGED_P_RANGE[1]
    c = Cache(W, Pm, HKV, D, PS_BF16, S)
    for s, r in enumerate(draws):
        c.seq_reset(s, 0)
        c.prefill_prefix(s, dev(synth.rows(SEED, synth.TID_K, s, HKV, 0, r.P, D, "bf16")),
                         dev(synth.rows(SEED, synth.TID_V, s, HKV, 0, r.P, D, "bf16")), r.P)
        n = min(W, r.t - r.P)
        if n > 0:
            c.import_window(s, r.t,
                            dev(synth.rows(SEED, synth.TID_K, s, HKV, r.t - n, n, D, "bf16")),
                            dev(synth.rows(SEED, synth.TID_V, s, HKV, r.t - n, n, D, "bf16")),
                            n, r.h0)
    total = 3 + 2 * steps
    q = dev(np.stack([synth.rows(SEED, synth.TID_Q, s, HQ, r.t, total, D, "bf16")
                      for s, r in enumerate(draws)], axis=1))
    kn = dev(np.stack([synth.rows(SEED, synth.TID_K, s, HKV, r.t, total, D, "bf16")
                       for s, r in enumerate(draws)], axis=1))
    vn = dev(np.stack([synth.rows(SEED, synth.TID_V, s, HKV, r.t, total, D, "bf16")
                       for s, r in enumerate(draws)], axis=1))
    out = torch.empty((S, HQ, D), dtype=torch.bfloat16, device="cuda")
    ws = c.decode_workspace(S, HQ)
    ids = list(range(S))
    pos = [r.t for r in draws]
    scale = 1.0 / math.sqrt(D)
    rows = []

    def step(i, st=None):
        c.decode_step(q[i], kn[i], vn[i], ids, pos, HQ, scale, out, ws, st)
        rows.append(sum(r.P + min(W, p + 1 - r.P) for r, p in zip(draws, pos)))
        for s in range(S):
            pos[s] += 1

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    if c.device_error():
        raise RuntimeError("device error word set by the ragged decode")
    n0 = len(rows)
    ms = time_graph(torch, lambda i, st: step(3 + i, st), steps)
    kv = HKV * D * 2 * 2 * (sum(rows[n0:]) / steps)
    if c.device_error():
        raise RuntimeError("device error word set by the ragged decode")
    c.close()
    del q, kn, vn
    torch.cuda.empty_cache()
    return {"workload": f"{S} sequences, P_s~U[64,512], t_s~U[P_s,131072], W={W}, "
                        f"Hq={HQ} Hkv={HKV} d={D}, bf16 (ps_decode_step)",
            "ms_per_step": round(ms, 5), "tokens_per_s": round(S / (ms / 1e3), 1),
            "kv_bytes_per_step": int(kv), "kv_gbs": round(kv / (ms / 1e3) / 1e9, 1),
            "frac": round(kv / (ms / 1e3) / 1e9 / load_peaks()[0], 4)}


SP_P = 4096  # system-prompt length of the shared-prefix measurement


def shared_prefix_measure(steps: int):
    """Prompt reuse (ps_share_prefix): B=8 sequences with the same 4096-token
    pinned prefix, W=4096, t >= 65536, decoded by ps_decode_step -- once with
    the prefix held once and shared, once with a private copy per sequence.
    The visible K/V per step is the same (268 MB); the shared prefix is read
    from HBM once per step instead of eight times."""
    import torch

    import synth
    from prefix_sliding_window_ring_b200 import PS_BF16, Cache

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    kp = dev(synth.rows(SEED, synth.TID_K, 0, HKV, 0, SP_P, D, "bf16"))
    vp = dev(synth.rows(SEED, synth.TID_V, 0, HKV, 0, SP_P, D, "bf16"))
    total = 3 + steps
    t0 = [T_START + 31 * s for s in range(B)]
    q = dev(np.stack([synth.rows(SEED, synth.TID_Q, s, HQ, t0[s], total, D, "bf16")
                      for s in range(B)], axis=1))
    kn = dev(np.stack([synth.rows(SEED, synth.TID_K, s, HKV, t0[s], total, D, "bf16")
                       for s in range(B)], axis=1))
    vn = dev(np.stack([synth.rows(SEED, synth.TID_V, s, HKV, t0[s], total, D, "bf16")
                       for s in range(B)], axis=1))
    scale = 1.0 / math.sqrt(D)
    res = {"workload": f"B={B} sequences sharing a {SP_P}-token pinned prefix, W={W}, "
                       f"t>=65536, Hq={HQ} Hkv={HKV} d={D}, bf16 (ps_decode_step)",
           "kv_bytes_per_step": B * HKV * (SP_P + W) * D * 2 * 2}
    for mode in ("private", "shared"):
        c = Cache(W, SP_P, HKV, D, PS_BF16, B)
        for s in range(B):
            c.seq_reset(s, (s * 613) % W)
            if mode == "shared" and s > 0:
                c.share_prefix(s, 0)
            else:
                c.prefill_prefix(s, kp, vp, SP_P)
            c.import_window(s, t0[s],
                            dev(synth.rows(SEED, synth.TID_K, s, HKV, t0[s] - W, W, D, "bf16")),
                            dev(synth.rows(SEED, synth.TID_V, s, HKV, t0[s] - W, W, D, "bf16")),
                            W, (s * 613) % W)
        out = torch.empty((B, HQ, D), dtype=torch.bfloat16, device="cuda")
        ws = c.decode_workspace(B, HQ)
        ids = list(range(B))
        pos = list(t0)

        def step(i, st=None):
            c.decode_step(q[i], kn[i], vn[i], ids, pos, HQ, scale, out, ws, st)
            for s in range(B):
                pos[s] += 1

        for i in range(3):
            step(i)
        torch.cuda.synchronize()
        ms = time_graph(torch, lambda i, st: step(3 + i, st), steps)
        if c.device_error():
            raise RuntimeError("device error word set by the shared-prefix decode")
        res[f"{mode}_ms_per_step"] = round(ms, 5)
        res[f"{mode}_tokens_per_s"] = round(B / (ms / 1e3), 1)
        c.close()
        torch.cuda.empty_cache()
    res["speedup"] = round(res["private_ms_per_step"] / res["shared_ms_per_step"], 3)
    return res


def paged_measure(steps: int):
    """Paged ring (block-table indirection): the decode step of the headline
    workload (B=8, Hq=16, Hkv=8, d=128, P=128, W=4096, bf16, window full) on an
    unpaged cache and on paged caches with 256- and 16-row pages.  Every cache
    is filled the same way -- the prefix, then the window appended to all eight
    sequences one page-sized piece at a time -- so a paged cache's pages are
    interleaved across sequences in the pool, as they are when sequences grow
    side by side.  The visible K/V per step is the same in every mode."""
    import torch

    import synth
    from prefix_sliding_window_ring_b200 import PS_BF16, Cache

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    total = 3 + steps
    kp = [synth.rows(SEED, synth.TID_K, s, HKV, 0, P + W + total, D, "bf16") for s in range(B)]
    vp = [synth.rows(SEED, synth.TID_V, s, HKV, 0, P + W + total, D, "bf16") for s in range(B)]
    kall = dev(np.stack(kp))  # [B][P + W + total][Hkv][d]
    vall = dev(np.stack(vp))
    q = dev(np.stack([synth.rows(SEED, synth.TID_Q, s, HQ, P + W, total, D, "bf16")
                      for s in range(B)], axis=1))
    scale = 1.0 / math.sqrt(D)
    res = {"workload": f"B={B}, Hq={HQ} Hkv={HKV} d={D}, P={P}, W={W}, window full, bf16 "
                       "(ps_decode_step); pages interleaved across sequences",
           "kv_bytes_per_step": kv_bytes_per_step()}
    ids = list(range(B))
    for page in (0, 256, 16):
        c = Cache(W, P, HKV, D, PS_BF16, B, page_rows=page, num_pages=B * W // page if page else 0)
        piece = page if page else 256
        for s in range(B):
            c.seq_reset(s, (s * 613) % W)
            c.prefill_prefix(s, kall[s, :P], vall[s, :P], P)
        for p0 in range(P, P + W, piece):
            c.append_kv(ids, kall[:, p0:p0 + piece].contiguous(), vall[:, p0:p0 + piece].contiguous(),
                        piece)
        out = torch.empty((B, HQ, D), dtype=torch.bfloat16, device="cuda")
        ws = c.decode_workspace(B, HQ)
        pos = [P + W] * B
        kn = kall[:, P + W:].transpose(0, 1).contiguous()  # [total][B][Hkv][d]
        vn = vall[:, P + W:].transpose(0, 1).contiguous()

        def step(i, st=None):
            c.decode_step(q[i], kn[i], vn[i], ids, pos, HQ, scale, out, ws, st)
            for s in range(B):
                pos[s] += 1

        for i in range(3):
            step(i)
        torch.cuda.synchronize()
        ms = time_graph(torch, lambda i, st: step(3 + i, st), steps)
        if c.device_error():
            raise RuntimeError("device error word set by the paged decode")
        key = f"page_rows_{page}" if page else "unpaged"
        res[key] = {"us_per_step": round(ms * 1e3, 2),
                    "GBps": round(kv_bytes_per_step() / (ms / 1e3) / 1e9, 1)}
        c.close()
        torch.cuda.empty_cache()
    return res


def gqa_measure(steps: int):
    """The decode call (ps_attend_decode) at B=8, Hkv=8, d=128, P=128, W=4096,
    t=65536, bf16, for GQA group sizes G = Hq / Hkv in {1, 2, 4, 8}: the same
    K/V bytes per call (138.4 MB), G query heads per kv head.  4 disjoint
    batches rotate (HBM-resident)."""
    import torch

    from prefix_sliding_window_ring_b200 import PS_BF16, Cache
    peak, _ = load_peaks()
    g = torch.Generator(device="cuda").manual_seed(SEED + 11)
    scale = 1.0 / math.sqrt(D)
    t = 65536
    res = {"note": "ps_attend_decode, B=8 Hkv=8 d=128 P=128 W=4096 t=65536 bf16, Hq = G * 8"}
    S = B * ROT
    c = Cache(W, P, HKV, D, PS_BF16, S)
    for s in range(S):
        h0 = (s * 613) % W
        c.seq_reset(s, h0)
        c.prefill_prefix(s, torch.randn((P, HKV, D), generator=g, device="cuda").to(torch.bfloat16),
                         torch.randn((P, HKV, D), generator=g, device="cuda").to(torch.bfloat16), P)
        c.import_window(s, t + 1, torch.randn((W, HKV, D), generator=g, device="cuda").to(torch.bfloat16),
                        torch.randn((W, HKV, D), generator=g, device="cuda").to(torch.bfloat16), W, h0)
    for G in (1, 2, 4, 8):
        hq = G * HKV
        q = torch.randn((B, hq, D), generator=g, device="cuda").to(torch.bfloat16)
        out = torch.empty_like(q)
        ws = c.decode_workspace(B, hq)

        def dec(i, st=None):
            r = i % ROT
            c.attend_decode(q, list(range(r * B, (r + 1) * B)), [t] * B, hq, scale, out, ws, st)

        for i in range(2 * ROT):
            dec(i)
        torch.cuda.synchronize()
        ms = time_graph(torch, dec, max(steps, 4 * ROT))
        if c.device_error():
            raise RuntimeError(f"device error word set by the decode at G={G}")
        gbs = kv_bytes_per_step() / (ms / 1e3) / 1e9
        res[f"G{G}"] = {"Hq": hq, "us_per_call": round(ms * 1e3, 2), "GBps": round(gbs, 1),
                        "frac": round(gbs / peak, 4)}
        del q, out, ws
    c.close()
    torch.cuda.empty_cache()
    return res


def t_sweep_measure(steps: int):
    """The decode call (ps_attend_decode, B=8, Hq=16, Hkv=8, d=128, bf16) at the
    positions the workload is quoted at, t in {2048, 4224, 16384, 65536} with
    P=128, W=4096: n = P + min(W, t - P + 1) visible rows (2049 at t=2048, 4224
    from t=4223 on).  Beside them the same 4224 rows as plain causal attention
    over the whole history (P=0, W=8192 >= t+1 at t=4223), the full-history
    case of the same kernel.  Inputs are seeded N(0,1) rows drawn on the device
    (only timing is taken here); 4 disjoint batches of 8 sequences rotate, so
    every call streams from HBM (at least 268 MB resident)."""
    import torch

    from prefix_sliding_window_ring_b200 import PS_BF16, Cache
    peak, _ = load_peaks()
    g = torch.Generator(device="cuda").manual_seed(SEED + 7)
    scale = 1.0 / math.sqrt(D)
    res = {"note": "ps_attend_decode, B=8 Hq=16 Hkv=8 d=128 bf16; 4 rotating batches (HBM-resident)"}
    cases = [("t2048", P, W, 2048), ("t4224", P, W, 4224), ("t16384", P, W, 16384),
             ("t65536", P, W, 65536), ("causal_P0_W8192_t4223", 0, 8192, 4223)]
    for name, Pc, Wc, t in cases:
        S = B * ROT
        c = Cache(Wc, max(Pc, 1), HKV, D, PS_BF16, S)
        nwin = min(Wc, t - Pc + 1)  # window rows held once position t is stored
        for s in range(S):
            h0 = (s * 613) % Wc
            c.seq_reset(s, h0)
            kp = torch.randn((Pc, HKV, D), generator=g, device="cuda").to(torch.bfloat16)
            vp = torch.randn((Pc, HKV, D), generator=g, device="cuda").to(torch.bfloat16)
            c.prefill_prefix(s, kp, vp, Pc)
            kw = torch.randn((nwin, HKV, D), generator=g, device="cuda").to(torch.bfloat16)
            vw = torch.randn((nwin, HKV, D), generator=g, device="cuda").to(torch.bfloat16)
            c.import_window(s, t + 1, kw, vw, nwin, h0)
            del kp, vp, kw, vw
        q = torch.randn((B, HQ, D), generator=g, device="cuda").to(torch.bfloat16)
        out = torch.empty_like(q)
        ws = c.decode_workspace(B, HQ)

        def dec(i, st=None):
            r = i % ROT
            c.attend_decode(q, list(range(r * B, (r + 1) * B)), [t] * B, HQ, scale, out, ws, st)

        for i in range(2 * ROT):
            dec(i)
        torch.cuda.synchronize()
        ms = time_graph(torch, dec, max(steps, 4 * ROT))
        if c.device_error():
            raise RuntimeError(f"device error word set by the decode at {name}")
        nvis = Pc + nwin
        gbs = B * HKV * nvis * D * 2 * 2 / (ms / 1e3) / 1e9
        res[name] = {"t": t, "P": Pc, "W": Wc, "visible_rows": nvis,
                     "us_per_call": round(ms * 1e3, 2), "GBps": round(gbs, 1),
                     "frac": round(gbs / peak, 4), "tokens_per_s": round(B / (ms / 1e3), 1)}
        c.close()
        del q, out, ws
        torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------ CPU oracle ----
def oracle_problems(seed, kscale, nseq):
    """The oracle's inputs for nseq sequences of the workload at t=T_START."""
    import oracle
    import synth
    G = HQ // HKV
    batch = oracle.Batch()
    scale = 1.0 / math.sqrt(D)
    for s in range(nseq):
        t = T_START + s
        lo = t - W + 1
        hp = np.concatenate([np.arange(0, P), np.arange(lo, t + 1)]).astype(np.int64)
        K = np.concatenate([
            synth.to_f64(synth.rows(seed, synth.TID_K, s, HKV, 0, P, D, "bf16", kscale)),
            synth.to_f64(synth.rows(seed, synth.TID_K, s, HKV, lo, t + 1 - lo, D, "bf16", kscale))])
        V = np.concatenate([
            synth.to_f64(synth.rows(seed, synth.TID_V, s, HKV, 0, P, D, "bf16")),
            synth.to_f64(synth.rows(seed, synth.TID_V, s, HKV, lo, t + 1 - lo, D, "bf16"))])
        q = synth.to_f64(synth.rows(seed, synth.TID_Q, s, HQ, t, 1, D, "bf16"))[0]
        for g in range(HKV):
            batch.add(P, W, t, scale, q[g * G:(g + 1) * G], hp, np.ascontiguousarray(K[:, g]),
                      np.ascontiguousarray(V[:, g]))
    return batch


def cpu_baseline(seed, kscale, budget_s=15.0, nthreads=None):
    """Time the oracle, as it stands, on this host's cores over a bounded sample:
    repeated decodes of one batch of B sequences of the workload."""
    import oracle
    nthreads = nthreads or oracle.host_threads()
    batch = oracle_problems(seed, kscale, B)
    reps = 0
    t0 = time.perf_counter()
    while True:
        batch.run(nthreads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 1000:
            break
    tok = reps * B
    # the same sample on one core, for a per-core figure (a short bounded run)
    reps1 = 0
    t1 = time.perf_counter()
    while True:
        batch.run(1)
        reps1 += 1
        el1 = time.perf_counter() - t1
        if el1 >= min(budget_s / 4, 5.0) or reps1 >= 250:
            break
    return {"value": round(tok / el, 2), "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": f"{reps} repetitions of one {B}-sequence decode step at t={T_START} "
                      f"(float64 masked attention, {reps * B} sequence-decodes, {el:.1f} s)",
            "one_core": {"value": round(reps1 * B / el1, 2), "unit": UNIT,
                         "sample": f"{reps1} repetitions on 1 thread, {el1:.1f} s"}}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import synth
    kscale = synth.chan_scale(SEED, HKV, D)
    cpu = cpu_baseline(SEED, kscale, budget_s=args.cpu_seconds)
    # K timed steps of the same workload, each step = one B-sequence decode by the oracle
    import oracle
    batch = oracle_problems(SEED, kscale, B)
    for _ in range(max(0, min(args.warmup, 1))):
        batch.run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        batch.run()
    el = time.perf_counter() - t0
    value = B * args.steps / el
    line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {**workload_config(), "parallelism": "host threads"},
            "cpu_baseline": {**cpu, "value": round(value, 2)},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--only", choices=["prefill", "prompt", "ragged", "shared", "paged", "t_sweep",
                                       "gqa", "chunk_small", "paged_prefill"],
                    help="run one side measurement alone and print its record (for profiling "
                         "one kernel under ncu); not a benchmark line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.only:
        import torch
        torch.cuda.set_device(local_rank)
        k = max(3, min(args.steps, 10))
        fn = {"prefill": prefill_measure, "ragged": ragged_measure,
              "shared": shared_prefix_measure, "paged": paged_measure,
              "t_sweep": lambda n: t_sweep_measure(max(n, 16)),
              "gqa": lambda n: gqa_measure(max(n, 16)),
              "chunk_small": lambda n: chunk_small_measure(max(n, 10)),
              "paged_prefill": lambda n: paged_prefill_measure(max(n, 5)),
              "prompt": lambda n: prompt_measure(n, load_bf16_peak()[0])}[args.only]
        print(json.dumps({"only": args.only, "result": fn(k)}), flush=True)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
