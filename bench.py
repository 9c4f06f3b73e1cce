#!/usr/bin/env python3
"""Benchmark of the DSA layer on B200.

Headline: DSA-layer decode tokens/s at 128K context — 4 sequences of 131072
cached tokens, 64 heads, indexer 32 x 128, top_k 2048 — one step being one
dsa_layer_forward (indexer -> top-k -> sparse attention) over the batch.  The
JSON line also carries prefill tokens/s on one 16384-token sequence, the
roofline fraction of the dominant kernel, an end-to-end number through host
buffers, and the CPU oracle timed on the host as a baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

For N > 1 launch one process per GPU with torch.distributed.run; every rank
runs an independent replica (the layer has no exchange step), timing is the
max over ranks and `value` counts the tokens of all ranks.
"""
from __future__ import annotations

import argparse
import faulthandler
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dsa_lightning_indexer_b200 import synth  # noqa: E402

METRIC = "DSA-layer decode tokens/s at 128K ctx + prefill tokens/s; % HBM / bf16 TC peak"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------ misc --

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained",
                                                     p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a background thread."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []  # (t, sm_mhz, reasons_mask)
        self.period = period_s
        self.stop_flag = threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.h = None
            prop = torch.cuda.get_device_properties(device_index)
            if all(hasattr(prop, a) for a in ("pci_domain_id", "pci_bus_id", "pci_device_id")):
                bus = "%08X:%02X:%02X.0" % (int(prop.pci_domain_id), int(prop.pci_bus_id),
                                             int(prop.pci_device_id))
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
                except Exception:  # noqa: BLE001
                    self.h = None
            if self.h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                ids = [int(x) for x in vis.split(",") if x.strip().isdigit()]
                self.h = pynvml.nvmlDeviceGetHandleByIndex(ids[device_index] if ids else
                                                           device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:  # noqa: BLE001
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, int(rs)))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self.stop_flag.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvml unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "sampled inside the timed region"
        if not inside:  # very short timed region: take the samples bracketing it
            before = [s for s in self.samples if s[0] < t0][-2:]
            after = [s for s in self.samples if s[0] > t1][:2]
            inside = before + after
            note = "timed region shorter than the sampling period; bracketing samples"
        mask = 0
        for s in inside:
            mask |= s[2]
        reasons = [n for b, n in self.REASONS.items() if mask & b and n != "gpu_idle"]
        mhz = [s[1] for s in inside]
        return {"sm_mhz": float(np.median(mhz)) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside), "note": note}


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def replica_launch_cmd(argv, n):
    """Command that runs this script as `n` ranks, one process per GPU, on
    this node (rendezvous on 127.0.0.1)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={free_port()}",
            os.path.abspath(__file__), *argv]


def dry_run(args):
    """The multi-rank plumbing without a GPU: gloo process group, barrier,
    max-over-ranks of a rank-dependent time, and the JSON line's rank and
    rate fields (launcher check)."""
    import datetime
    rank, _, world = env_rank()
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        dist.barrier()
    ms = max_over_ranks(10.0 + rank, dist)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"dry_run": True, "n_gpus": world, "gpus_flag": args.gpus,
                          "ms_per_step": ms / max(1, args.steps),
                          "value": job_rate(4, world, args.steps, ms)}), flush=True)
    return 0


def max_over_ranks(x, dist=None, device="cpu"):
    """The largest `x` over the ranks of the process group, on every rank (`x`
    itself without a group): a job's device time is its slowest replica's."""
    if not dist:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank, world, steps, ms_total):
    """Whole-job throughput: the units every rank processed over `steps`
    steps, divided by the (max-over-ranks) time of those steps."""
    return units_per_rank * world * steps / (ms_total / 1e3)


# -------------------------------------------------------- reference arm --

def run_reference(args):
    """The CPU oracle as the reference arm: each step is one query row of the
    128K decode workload, computed in full (score all 131072 keys, select,
    attend) in double precision on the host cores."""
    rank, _, world = env_rank()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    wl = synth.decode_b4_128k()
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    a = (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)

    def step(i):
        r = np.array([i % wl.Nq], np.int64)
        oracle.dsa_layer(*a, wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k, wl.scale,
                         sample=r)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    value = args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": "one query row of the 128K decode workload per step "
                                   "(all 131072 keys scored, top-2048, 64-head attention), "
                                   "rows cycled over the 4 sequences"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl, copies=2):
    return {"workload": wl.name, "batch": wl.B, "ctx": int(wl.ctx_lens.max()),
            "heads": wl.H, "index_heads": synth.HI, "index_dim": synth.DI,
            "latent_dim": synth.D, "value_dim": synth.DV, "top_k": wl.top_k,
            "global_batch": wl.B, "seq_len": int(wl.ctx_lens.max()), "parallelism": "replicas",
            "l2": f"{copies} rotating input copies; each step streams "
                  f"{indexer_bytes(wl) / 1e6:.0f} MB of indexer keys against a 126 MB L2"}


# ------------------------------------------------------------- our arm --

def decode_bytes(wl):
    """Algorithmic bytes of one layer step: indexer keys scanned, selected KV rows
    gathered, per-query inputs read and outputs written."""
    L = wl.ctx_lens.astype(np.int64)
    nsel = np.minimum(wl.top_k, L)
    kidx = int((L * synth.DI * 2).sum())
    kv = int((nsel * synth.D * 2).sum())
    per_q = wl.H * synth.D * 2 + synth.HI * synth.DI * 2 + synth.HI * 4 \
        + wl.H * synth.DV * 4 + wl.H * 4 + wl.top_k * 4
    return {"k_idx": kidx, "kv": kv, "query_io": per_q * wl.Nq,
            "total": kidx + kv + per_q * wl.Nq}


def indexer_bytes(wl):
    L = wl.ctx_lens.astype(np.int64)
    return int((L * synth.DI * 2).sum()) + wl.Nq * (synth.HI * synth.DI * 2 + synth.HI * 4)


def indexer_causal_flops(wl):
    """2 * 32 * 128 flops per (query, visible key) pair."""
    pos = wl.positions()
    return float(2 * synth.HI * synth.DI) * float((pos + 1).sum())


def attention_useful_flops(wl):
    """2 * H * (576 + 512) flops per selected key of each query row (S over
    the 576-wide rows, P.V over their first 512 dims); a row selects
    min(top_k, p + 1) keys."""
    pos = wl.positions()
    n_sel = np.minimum(wl.top_k, pos + 1).astype(np.float64)
    H = int(wl.q.shape[1])
    return float(2 * H * (synth.D + synth.DV)) * float(n_sel.sum())


def launches_per_layer(wl, sms=148):
    """Kernels one dsa_layer_forward launches: when the indexer builds score
    histograms, first the kernel that zeroes their region; the indexer (one
    launch per 64 sequences with queries); then either the fused decode tail
    (selection, attention and merge in one kernel: 6 to 12 long rows, at most
    64 heads), or the selection -- the tail kernel's selection alone for 13 to
    16 long rows, two kernels (filter and emit) for other histogram-driven
    rows, else one -- followed by the sparse attention and, when few rows
    split the selected set over CTAs, the merge of the slices."""
    nq = np.diff(wl.q_offsets)
    seqs = int((nq > 0).sum())
    max_len = int(wl.ctx_lens.max()) if wl.B else 0
    chunks = max(1, 2 * 148 // max(1, wl.Nq))  # as the library plans it
    per = -(-max_len // chunks)
    chunk = min(max(512, -(-per // 512) * 512), 8192)
    hist = (0 < wl.Nq <= 148 and max_len >= 8192 and max_len >= 4 * wl.top_k
            and -(-max_len // chunk) <= 512)
    C = 148 // max(1, wl.Nq)
    tail_fits = (0 < wl.Nq <= 16 and C >= 8 and (-(-max_len // C) + 31) // 32 <= 512)
    fused = hist and wl.H <= 64 and 6 <= wl.Nq <= 12 and tail_fits
    indexer = (seqs + 63) // 64 + (1 if hist else 0)
    if fused:
        return indexer + 1
    select_tail = hist and wl.Nq > 12 and tail_fits
    few_rows = wl.Nq * ((wl.H + 63) // 64) < sms
    selection = 1 if select_tail else (2 if hist else 1)
    return indexer + selection + 1 + (1 if few_rows and wl.top_k > 16 else 0)


def profiled_traffic(profile="profiles/indexer_score_b4_128k_traffic.json"):
    """DRAM bytes per in-layer indexer launch from the committed ncu record,
    or None once the kernel's sources differ from the ones the counters were
    taken on."""
    import hashlib
    root = os.path.dirname(os.path.abspath(__file__))
    try:
        rec = json.load(open(os.path.join(root, profile)))
        traffic = int(rec["traffic_bytes"])
        pins = dict(rec["source_sha256_prefix"])
    except (OSError, KeyError, TypeError, ValueError):
        return None
    csrc = os.path.join(root, "dsa_lightning_indexer_b200", "csrc")
    for name, prefix in pins.items():
        try:
            digest = hashlib.sha256(open(os.path.join(csrc, name), "rb").read()).hexdigest()
        except OSError:
            return None
        if not digest.startswith(prefix):
            return None
    return traffic


def run_ours(args):
    rank, local_rank, world = env_rank()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.prefill_only:  # profiling aid: the prefill object alone
        from dsa_lightning_indexer_b200 import binding as bd
        print(json.dumps({"prefill": prefill_bench(bd, dev, load_peaks(), args)}), flush=True)
        return 0
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    from dsa_lightning_indexer_b200 import binding as bd

    peaks = load_peaks()
    wl = synth.decode_b4_128k()
    copies = [bd.DeviceWorkload(wl, dev)]
    # more copies of every input so consecutive steps never find their data in L2
    for _ in range(1, max(1, args.copies)):
        c = bd.DeviceWorkload.__new__(bd.DeviceWorkload)
        c.__dict__.update(copies[0].__dict__)
        for name in ("q_idx", "w", "k_idx", "q", "kv"):
            setattr(c, name, getattr(copies[0], name).clone())
        c.ws = torch.zeros_like(copies[0].ws)
        copies.append(c)
    out, lse, idx = copies[0].new_outputs()

    def step(i):
        copies[i % len(copies)].forward(out, lse, idx)

    for i in range(max(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    for c in copies:
        bd.check_device_status(c.ws)

    # A serving loop replays the decode step as a CUDA graph (one per input copy).
    graphs = []
    if not args.no_graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            for ci in range(len(copies)):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=side):
                    step(ci)
                graphs.append(g)
        torch.cuda.current_stream(dev).wait_stream(side)
        for i in range(max(args.warmup, 3)):
            graphs[i % len(graphs)].replay()
        torch.cuda.synchronize()

    def timed_step(i):
        if graphs:
            graphs[i % len(graphs)].replay()
        else:
            step(i)

    # Timed region: every step is replayed with the L2 flushed first (a 256 MB
    # write, outside the step's events), so no step finds the previous one's
    # gathered rows, partials or scores in L2; the step's device time is the
    # sum of the per-step event intervals.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.05)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i, (a, b) in enumerate(evs):
        flush.fill_(i & 0xFF)
        a.record()
        timed_step(i)
        b.record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if dist:
        dist.barrier()
    sampler.stop()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), dist, dev)
    # For context: the same steps back to back with no flush (two rotating copies).
    torch.cuda.synchronize()
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record()
    for i in range(args.steps):
        timed_step(i)
    w1.record()
    torch.cuda.synchronize()
    ms_warm = max_over_ranks(w0.elapsed_time(w1), dist, dev) / args.steps
    for c in copies:
        bd.check_device_status(c.ws)
    del graphs, flush
    ms_step = ms / args.steps
    value = job_rate(wl.Nq, world, args.steps, ms)

    # --- per-kernel times: the same step as three C-ABI calls, events between them
    ktimes = kernel_times(bd, copies, wl, args.steps, dev) if not args.no_kernel_times else {
        "indexer_score_us": float("nan")}
    kb = indexer_bytes(wl)
    k1_s = ktimes["indexer_score_us"] * 1e-6
    achieved = kb / k1_s / 1e9
    db = decode_bytes(wl)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(config_of(wl, len(copies)),
                       launch="direct calls" if args.no_graph else "CUDA graph replay of "
                       "dsa_layer_forward",
                       l2="flushed by a 256 MB write before every timed step (outside its "
                          "CUDA events); each step also streams "
                          f"{indexer_bytes(wl) / 1e6:.0f} MB of indexer keys"),
        "ms_per_step_back_to_back": ms_warm,
        "roofline": None if args.no_kernel_times else {"bound": "hbm", "kernel": "indexer_score", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": profiled_traffic(), "peak_source": peaks["source"],
                     "algorithmic_bytes_per_launch": kb},
        "layer_roofline": {"algorithmic_bytes_per_step": db["total"],
                           "achieved_gbs": db["total"] / (ms_step * 1e-3) / 1e9,
                           "frac": db["total"] / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "kernel_times_us": ktimes,
        "gpu_launches": launches_per_layer(wl) * args.steps,
        "clocks": sampler.summary(t0, t1),
    }
    if not args.no_e2e:
        line["e2e"] = e2e_decode(bd, wl, copies[0], args.steps, max(args.warmup, 3), dev, world,
                                 dist)
    # the oracle beside the GPU numbers, on the host cores of rank 0 at N = 1
    args.with_oracle = rank == 0 and world == 1 and not args.no_cpu_baseline
    if not args.no_prefill:
        line["prefill"] = prefill_bench(bd, dev, peaks, args)
    if not args.no_other and world == 1:
        # The other decode workloads of the specification, reported beside the
        # headline (a failure here must not cost the headline line).
        other = {}
        for key, run in (("prefill_T1024_H16", lambda: tiny_prefill_bench(bd, dev, 20, 3,
                                                                          args.with_oracle)),
                         ("decode_B8_L32768",
                          lambda: decode_workload_bench(bd, synth.decode_b8_32k(), dev, peaks,
                                                        50, 3, args.with_oracle)),
                         ("ragged_B32", lambda: ragged_bench(bd, dev, peaks, 50, 3,
                                                             with_oracle=args.with_oracle)),
                         ("attention_routes_B4_L131072",
                          lambda: mask_route_bench(bd, dev, peaks, 20, 3)),
                         ("indexer_input_step", lambda: input_step_bench(bd, dev, peaks, 20, 3))):
            other[key] = _safe(run)
            torch.cuda.empty_cache()
        line["other_workloads"] = other
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def kernel_times(bd, copies, wl, steps, dev):
    """Average device time of each kernel of the step: every C-ABI call of the
    step captured alone, `reps` times (alternating input copies), in a CUDA
    graph, and the graph timed with CUDA events on the launching stream."""
    reps = 16
    c0 = copies[0]
    ld = (int(wl.ctx_lens.max()) + 3) // 4 * 4
    scores = torch.empty(wl.Nq, ld, dtype=torch.float32, device=dev)
    out, lse, idx = c0.new_outputs()

    # The histogram flag makes the two calls launch exactly the layer's kernels:
    # the indexer with its score-histogram epilogue, then the filter and emit.
    flags = bd.FLAG_SCORE_HISTOGRAM

    def k1(c):
        bd.indexer_score(c.batch, c.q_idx, c.w, c.k_idx, scores, ld, c.ws, flags=flags)

    def k2(c):
        bd.topk(c.batch, scores, ld, c.top_k, idx, c.ws, flags=flags)

    def k3(c):
        bd.sparse_attn(c.batch, c.q, c.kv, idx, c.top_k, c.scale, out, lse, c.ws)

    for c in copies:  # warm: inputs of every later call are valid
        k1(c), k2(c), k3(c)
    torch.cuda.synchronize()
    res = {}
    side = torch.cuda.Stream(dev)
    for name, fn in (("indexer_score_us", k1), ("topk_us", k2),
                     ("sparse_attn_us", k3)):
        g = torch.cuda.CUDAGraph()
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for i in range(reps):
                    fn(copies[i % len(copies)])
        torch.cuda.current_stream(dev).wait_stream(side)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        n = max(3, min(steps, 50))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        res[name] = e0.elapsed_time(e1) * 1e3 / (n * reps)
        del g
    res["launches_timed"] = n * reps
    res["method"] = "per-kernel CUDA graphs of 16 launches, CUDA events around replays"
    res["note"] = ("each C-ABI call alone, with DSA_FLAG_SCORE_HISTOGRAM: the same launches "
                   "as inside dsa_layer_forward (indexer with its histogram epilogue; "
                   "top-k filter and emit); inputs alternate between two copies")
    for c in copies:
        bd.check_device_status(c.ws)
    return res


def _packed(parts, align=256):
    """Byte offsets of `parts` (name, nbytes) packed into one buffer."""
    offs, n = {}, 0
    for name, nbytes in parts:
        offs[name] = n
        n += (nbytes + align - 1) // align * align
    return offs, n


def e2e_decode(bd, wl, dw, steps, warmup, dev, world, dist):
    """Decode steps through host buffers, as a serving loop overlaps them: each
    step's new inputs (queries, indexer queries and weights, and the new
    token's rows of both caches) arrive in one copy from pinned host memory,
    the cache rows are scattered into the resident caches, the layer runs,
    and its output, log-sum-exp and index sets leave in one copy into pinned
    host memory.  Two buffer sets alternate, and the uploads and downloads run
    on their own streams, so one step's copies overlap the neighbouring
    steps' compute (the scatter and the layer stay in order on the compute
    stream).  G steps are captured as one CUDA graph and replayed."""
    new_rows = [int(wl.kv_offsets[b] + wl.ctx_lens[b] - 1) for b in range(wl.B)]
    host_in = {"q": wl.q, "q_idx": wl.q_idx, "w": wl.w,
               "krow": wl.k_idx[new_rows], "vrow": wl.kv[new_rows]}
    offs, n_in = _packed([(k, v.nbytes) for k, v in host_in.items()])
    Nq, H, top_k = wl.Nq, wl.H, wl.top_k
    oo, n_out = _packed([("out", Nq * H * 512 * 4), ("lse", Nq * H * 4), ("idx", Nq * top_k * 4)])

    def dview(buf, o, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        return buf[o:o + nbytes].view(dtype).view(*shape)

    sets = []
    for _ in range(2):
        h_in = torch.empty(n_in, dtype=torch.uint8).pin_memory()
        hv = h_in.numpy()
        for k, v in host_in.items():
            hv[offs[k]:offs[k] + v.nbytes] = np.ascontiguousarray(v).view(np.uint8).ravel()
        d_in = torch.empty(n_in, dtype=torch.uint8, device=dev)
        d_out = torch.empty(n_out, dtype=torch.uint8, device=dev)
        sets.append({
            "h_in": h_in, "d_in": d_in, "d_out": d_out,
            "h_out": torch.empty(n_out, dtype=torch.uint8).pin_memory(),
            "q": dview(d_in, offs["q"], wl.q.shape, torch.bfloat16),
            "q_idx": dview(d_in, offs["q_idx"], wl.q_idx.shape, torch.bfloat16),
            "w": dview(d_in, offs["w"], wl.w.shape, torch.float32),
            "krow": dview(d_in, offs["krow"], host_in["krow"].shape, torch.int16),
            "vrow": dview(d_in, offs["vrow"], host_in["vrow"].shape, torch.int16),
            "out": dview(d_out, oo["out"], (Nq, H, 512), torch.float32),
            "lse": dview(d_out, oo["lse"], (Nq, H), torch.float32),
            "idx": dview(d_out, oo["idx"], (Nq, top_k), torch.int32),
        })
    rows = torch.tensor(new_rows, dtype=torch.long, device=dev)
    k16, v16 = dw.k_idx.view(torch.int16), dw.kv.view(torch.int16)
    s_comp, s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("up", "comp", "down")}
    G = max(g for g in range(1, 9) if steps % g == 0)  # steps per captured graph

    def enqueue(i, first):
        b = i & 1
        st = sets[b]
        with torch.cuda.stream(s_up):
            if not first:
                s_up.wait_event(ev["comp"][b])   # the layer that read this buffer is done
            st["d_in"].copy_(st["h_in"], non_blocking=True)
            ev["up"][b].record(s_up)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev["up"][b])
            if not first:
                s_comp.wait_event(ev["down"][b])  # this output buffer has been read out
            k16.index_copy_(0, rows, st["krow"])
            v16.index_copy_(0, rows, st["vrow"])
            bd.layer_forward(dw.batch, st["q"], st["q_idx"], st["w"], dw.k_idx, dw.kv, top_k,
                             wl.scale, st["out"], st["lse"], st["idx"], dw.ws)
            ev["comp"][b].record(s_comp)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev["comp"][b])
            st["h_out"].copy_(st["d_out"], non_blocking=True)
            ev["down"][b].record(s_down)

    cur = torch.cuda.current_stream(dev)

    def capture():
        g = torch.cuda.CUDAGraph()
        for s_ in (s_comp, s_up, s_down):
            s_.wait_stream(cur)
        with torch.cuda.graph(g, stream=s_comp):
            s_up.wait_stream(s_comp)
            s_down.wait_stream(s_comp)
            for i in range(G):
                enqueue(i, first=i < 2)
            s_comp.wait_stream(s_up)
            s_comp.wait_stream(s_down)
        cur.wait_stream(s_comp)
        return g

    for i in range(2):  # eager warm-up (lazy initialisation before capture)
        enqueue(i, first=True)
    torch.cuda.synchronize()
    g = capture()
    for _ in range(max(1, warmup // G + 1)):
        g.replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps // G):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    bd.check_device_status(dw.ws)
    # The replayed steps really moved the results: compare with a plain call.
    ref_out, ref_lse, ref_idx = dw.forward()
    torch.cuda.synchronize()
    for st in sets:
        hb = st["h_out"].numpy()
        got_idx = hb[oo["idx"]:oo["idx"] + Nq * top_k * 4].view(np.int32).reshape(Nq, top_k)
        got_out = hb[oo["out"]:oo["out"] + Nq * H * 512 * 4].view(np.float32).reshape(Nq, H, 512)
        if not (np.array_equal(got_idx, ref_idx.cpu().numpy())
                and np.allclose(got_out, ref_out.cpu().numpy(), rtol=0.0, atol=1e-5)):
            raise RuntimeError("e2e: the results read back differ from a direct layer call")
    del g
    return {"value": job_rate(wl.Nq, world, steps, ms), "unit": UNIT,
            "h2d_bytes_per_step": int(n_in), "d2h_bytes_per_step": int(n_out),
            "ms_per_step": ms / steps, "steps_per_graph": G,
            "method": "two buffer sets; per step one packed H2D copy (upload stream), cache-row "
                      "scatter and dsa_layer_forward (compute stream), one packed D2H copy "
                      "(download stream); G steps per CUDA graph, replayed"}


def prefill_bench(bd, dev, peaks, args):
    """One causal prefill (64 heads, top_k 2048, planted indexer keys): the
    specified 16384 tokens, or --prefill-tokens for a smaller profiling case."""
    if args.prefill_tokens == 16384:
        wl = synth.prefill_16k()
    else:
        wl = synth.prefill(args.prefill_tokens, 64, 2048, seed=2, planted=True)
    dw = bd.DeviceWorkload(wl, dev)
    out, lse, idx = dw.new_outputs()
    ld = (int(wl.ctx_lens.max()) + 3) // 4 * 4
    scores = torch.empty(wl.Nq, ld, dtype=torch.float32, device=dev)
    n = max(1, min(args.prefill_steps, 10))
    for _ in range(2):
        dw.forward(out, lse, idx)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        dw.forward(out, lse, idx)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    k1 = []
    k2 = []
    k3 = []
    for _ in range(n):
        ev[0].record()
        bd.indexer_score(dw.batch, dw.q_idx, dw.w, dw.k_idx, scores, ld, dw.ws)
        ev[1].record()
        bd.topk(dw.batch, scores, ld, dw.top_k, idx, dw.ws)
        ev[2].record()
        bd.sparse_attn(dw.batch, dw.q, dw.kv, idx, dw.top_k, dw.scale, out, lse, dw.ws)
        ev[3].record()
        torch.cuda.synchronize()
        k1.append(ev[0].elapsed_time(ev[1]))
        k2.append(ev[1].elapsed_time(ev[2]))
        k3.append(ev[2].elapsed_time(ev[3]))
    bd.check_device_status(dw.ws)
    del dw, out, lse, idx, scores
    fl = indexer_causal_flops(wl)
    k1s = float(np.mean(k1)) * 1e-3
    tf = fl / k1s / 1e12
    afl = attention_useful_flops(wl)
    atf = afl / (float(np.mean(k3)) * 1e-3) / 1e12
    extra = {}
    if getattr(args, "with_oracle", False):
        extra["cpu_baseline"] = _safe(lambda: prefill_oracle(wl))
    return {**{"workload": wl.name, "tokens_per_s": wl.Nq / (ms * 1e-3), "ms_per_step": ms,
            "steps": n, "indexer_ms": k1s * 1e3, "topk_ms": float(np.mean(k2)),
            "sparse_attn_ms": float(np.mean(k3)),
            "indexer_roofline": {"bound": "tensor", "achieved": tf,
                                 "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                 "frac": tf / peaks["bf16_tflops"], "causal_flops": fl},
            "attention_roofline": {"bound": "tensor", "achieved": atf,
                                   "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                   "frac": atf / peaks["bf16_tflops"], "useful_flops": afl,
                                   "note": "S and P.V over the selected keys only"}},
            **extra}


def _graph_of(fn, dev):
    """`fn` captured once as a CUDA graph on a side stream, after one eager call."""
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        fn()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fn()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    return g


def _time_flushed(g, steps, warmup, dev):
    """Mean device time (ms) of one replay of `g`.  Before each timed replay a
    256 MB write flushes the L2; CUDA events bracket the replay alone."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        g.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i, (a, b) in enumerate(evs):
        flush.fill_(i & 0xFF)
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def decode_workload_bench(bd, wl, dev, peaks, steps, warmup, with_oracle=False):
    """One decode workload's layer step (a CUDA graph of dsa_layer_forward),
    inputs resident, L2 flushed before every timed step; with the oracle's
    time for the same step on the host cores beside it if asked."""
    dw = bd.DeviceWorkload(wl, dev)
    out, lse, idx = dw.new_outputs()
    g = _graph_of(lambda: dw.forward(out, lse, idx), dev)
    ms = _time_flushed(g, steps, warmup, dev)
    bd.check_device_status(dw.ws)
    del g
    del dw, out, lse, idx
    db = decode_bytes(wl)
    gbs = db["total"] / (ms * 1e-3) / 1e9
    res = {"workload": wl.name, "tokens_per_s": wl.Nq / (ms * 1e-3), "ms_per_step": ms,
           "steps": steps, "l2": "flushed by a 256 MB write before each timed step",
           "layer_roofline": {"bound": "hbm", "algorithmic_bytes_per_step": db["total"],
                              "achieved_gbs": gbs, "peak": peaks["hbm_gbs"],
                              "frac": gbs / peaks["hbm_gbs"]}}
    if with_oracle:
        res["cpu_baseline"] = _safe(lambda: oracle_full(wl))
    return res


def tiny_prefill_bench(bd, dev, steps, warmup, with_oracle=False):
    """The 1024-token, 16-head prefill at top_k 256 and 2048 (a parity case;
    timed for completeness), with the oracle on all host cores (and, at
    top_k 256, on one)."""
    res = {}
    for k in (256, 2048):
        wl = synth.tiny_prefill(k)
        dw = bd.DeviceWorkload(wl, dev)
        out, lse, idx = dw.new_outputs()
        g = _graph_of(lambda: dw.forward(out, lse, idx), dev)
        ms = _time_flushed(g, steps, warmup, dev)
        bd.check_device_status(dw.ws)
        del g, dw, out, lse, idx
        r = {"workload": wl.name, "tokens_per_s": wl.Nq / (ms * 1e-3), "ms_per_step": ms,
             "steps": steps, "l2": "flushed by a 256 MB write before each timed step"}
        if with_oracle:
            r["cpu_baseline"] = _safe(lambda: oracle_full(wl))
            if k == 256:  # and once single-threaded
                r["cpu_baseline_1_thread"] = _safe(lambda: oracle_full(wl, threads=1))
        res[f"top_k_{k}"] = r
    return res


def glue_step(out, proj, q):
    """The stacked ragged workload's glue on the device, in fp32: the next
    layer's query from this layer's output -- mean over heads, RMS-normalised,
    rounded to bf16, times the fixed bf16 projection, rounded to bf16."""
    m = out.mean(dim=1)
    m = m * torch.rsqrt((m * m).mean(dim=1, keepdim=True) + 1e-6)
    q.copy_((m.to(torch.bfloat16) @ proj).view(q.shape))


def ragged_bench(bd, dev, peaks, steps, warmup, layers=24, with_oracle=False):
    """The ragged serving batch (32 sequences, log-uniform contexts in
    [1024, 131072]): one layer's step, and a step of `layers` stacked layers,
    each with its own seeded caches and indexer inputs, with the glue between
    them (the last layer's output feeds the first layer's query of the next
    step)."""
    wl0 = synth.ragged_layer(0)
    res = decode_workload_bench(bd, wl0, dev, peaks, steps, warmup, with_oracle)
    t0 = time.perf_counter()
    dws, layer_bytes = [], 0
    for layer in range(layers):
        wl = wl0 if layer == 0 else synth.ragged_layer(layer)
        dw = bd.DeviceWorkload(wl, dev)
        dw.wl = None  # the host arrays are not needed once the inputs are on the device
        layer_bytes += decode_bytes(wl)["total"]
        if layer > 0:
            del dw.ws  # one workspace serves every layer (same batch, calls in order)
        dws.append(dw)
        del wl
    draw_s = time.perf_counter() - t0
    ws = dws[0].ws
    out, lse, idx = dws[0].new_outputs()
    proj = bd.bf16_tensor(synth.glue_projection(4), dev)

    def stack():
        for layer, dw in enumerate(dws):
            bd.layer_forward(dw.batch, dw.q, dw.q_idx, dw.w, dw.k_idx, dw.kv, dw.top_k,
                             dw.scale, out, lse, idx, ws)
            glue_step(out, proj, dws[(layer + 1) % layers].q)

    g = _graph_of(stack, dev)
    n = max(3, steps // 10)
    ms = _time_flushed(g, n, min(warmup, 3), dev)
    bd.check_device_status(ws)
    del g, dws, ws, out, lse, idx
    gbs = layer_bytes / (ms * 1e-3) / 1e9
    res["stack"] = {
        "layers": layers, "ms_per_step": ms, "steps": n,
        "tokens_per_s": wl0.Nq / (ms * 1e-3),
        "ms_per_layer_with_glue": ms / layers,
        "inputs": f"{layers} layers, each with its own seeded caches, indexer inputs and "
                  f"weights (drawn in {draw_s:.0f} s); the main query chains through the glue",
        "glue": "head mean, RMS norm, bf16, x [512, 64*576] bf16 projection (torch ops, fp32)",
        "layer_roofline": {"bound": "hbm", "algorithmic_bytes_per_step": layer_bytes,
                           "achieved_gbs": gbs, "peak": peaks["hbm_gbs"],
                           "frac": gbs / peaks["hbm_gbs"],
                           "note": "layers' algorithmic bytes only; glue time included"}}
    return res


def mask_route_bench(bd, dev, peaks, steps, warmup):
    """The two ways to run step 3 on the 128K decode workload, each on the
    layer's own index sets, L2 flushed before every timed call: the gather of
    the selected latent rows (this library's route) and the mask over the
    whole cache (the route the pages describe for llama.cpp)."""
    wl = synth.decode_b4_128k()
    dw = bd.DeviceWorkload(wl, dev)
    ws = bd.alloc_workspace(dw.batch, wl.H, wl.top_k, dev, flags=bd.FLAG_MASKED_ROUTE)
    out, lse, idx = dw.new_outputs()
    dw.forward(out, lse, idx)
    o2, l2 = torch.empty_like(out), torch.empty_like(lse)
    res = {"workload": wl.name}
    L = wl.ctx_lens.astype(np.int64)
    per_q = wl.H * synth.D * 2 + wl.H * synth.DV * 4 + wl.H * 4 + wl.top_k * 4
    routes = {
        "gather": (lambda: bd.sparse_attn(dw.batch, dw.q, dw.kv, idx, wl.top_k, wl.scale, o2, l2,
                                          ws),
                   int((np.minimum(wl.top_k, L) * synth.D * 2).sum()) + per_q * wl.Nq),
        "mask_whole_cache": (lambda: bd.masked_attn(dw.batch, dw.q, dw.kv, idx, wl.top_k,
                                                    wl.scale, o2, l2, ws),
                             int((L * synth.D * 2).sum()) + per_q * wl.Nq),
    }
    kidx = int((L * synth.DI * 2).sum()) + wl.Nq * (synth.HI * synth.DI * 2 + synth.HI * 4)
    for name, (fn, nbytes) in routes.items():
        g = _graph_of(fn, dev)
        ms = _time_flushed(g, steps, warmup, dev)
        bd.check_device_status(ws)
        del g
        res[name] = {"attention_ms": ms, "attention_bytes_per_call": nbytes,
                     "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                     "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "layer_bytes_per_token_mb": (kidx + nbytes) / wl.Nq / 1e6}
    # both routes compute the same attention
    bd.masked_attn(dw.batch, dw.q, dw.kv, idx, wl.top_k, wl.scale, o2, l2, ws)
    bd.sparse_attn(dw.batch, dw.q, dw.kv, idx, wl.top_k, wl.scale, out, lse, ws)
    torch.cuda.synchronize()
    res["max_abs_diff_between_routes"] = float((o2 - out).abs().max().item())
    res["mask_over_gather_time"] = res["mask_whole_cache"]["attention_ms"] / res["gather"][
        "attention_ms"]
    del dw, ws, out, lse, idx, o2, l2
    return res


D_MODEL, D_Q = 7168, 1536  # assumed widths of the hidden state and the query latent


def input_step_bench(bd, dev, peaks, steps, warmup):
    """The indexer's input step (q_b, k and head-weight projections, k appended
    to the key cache) on the decode batch's 4 new tokens (weight streaming:
    HBM-bound) and on the 16384 tokens of the prefill (tensor-bound), at the
    assumed widths (hidden 7168, query latent 1536), L2 flushed before every
    timed call."""
    g = torch.Generator(device=dev)
    g.manual_seed(7)

    def bf(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device=dev) * std).to(torch.bfloat16)
    w_q_b = bf(4096, D_Q, std=D_Q ** -0.5)
    w_k = bf(128, D_MODEL, std=D_MODEL ** -0.5)
    w_proj = bf(32, D_MODEL, std=D_MODEL ** -0.5)
    weight_bytes = 2 * (4096 * D_Q + 128 * D_MODEL + 32 * D_MODEL)
    res = {"widths": {"d_model": D_MODEL, "d_q": D_Q, "note": "assumed; the pages give none"}}
    for name, lens, nq in (("decode_B4_L131072", [131072] * 4, [1] * 4),
                           ("prefill_T16384", [16384], [16384])):
        T = sum(nq)
        kv_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        b = bd.Batch(np.concatenate([[0], np.cumsum(nq)]).astype(np.int32), kv_off,
                     np.array(lens, np.int32), dev)
        x, c_q = bf(T, D_MODEL), bf(T, D_Q)
        k_cache = torch.zeros(int(kv_off[-1]), 128, dtype=torch.bfloat16, device=dev)
        q_idx = torch.empty(T, 32, 128, dtype=torch.bfloat16, device=dev)
        w = torch.empty(T, 32, device=dev)
        ws = bd.indexer_project_workspace(b, D_MODEL, D_Q, dev)
        fn = (lambda: bd.indexer_project(b, x, c_q, w_q_b, w_k, w_proj, q_idx, k_cache, w, ws))
        gr = _graph_of(fn, dev)
        ms = _time_flushed(gr, steps, warmup, dev)
        bd.check_device_status(ws)
        del gr
        flops = 2.0 * T * (4096 * D_Q + 160 * D_MODEL)
        nbytes = weight_bytes + 2 * T * (D_MODEL + D_Q) + T * (4096 * 2 + 128 * 2 + 32 * 4)
        r = {"tokens": T, "ms": ms, "tokens_per_s": T / (ms * 1e-3), "bytes": nbytes,
             "flops": flops, "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
             "achieved_tflops": flops / (ms * 1e-3) / 1e12}
        if T <= 64:
            r["roofline"] = {"bound": "hbm", "frac": r["achieved_gbs"] / peaks["hbm_gbs"],
                             "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        else:
            r["roofline"] = {"bound": "tensor", "frac": r["achieved_tflops"] / peaks["bf16_tflops"],
                             "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
        res[name] = r
        del x, c_q, k_cache, q_idx, w, ws, b
    return res


def _safe(fn):
    """fn(), or a record of its failure: an optional measurement must not cost
    the JSON line."""
    try:
        return fn()
    except Exception as e:  # noqa: BLE001
        return {"error": repr(e)}


def oracle_seconds(wl, rows=None, threads=None):
    """Wall time of the oracle, as it stands, for the whole layer on `rows`
    (every query row when None), OpenMP over `threads` host cores (all of
    them when None); and the thread count."""
    import oracle
    oracle.build()
    threads = threads or len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    a = (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)
    t0 = time.perf_counter()
    oracle.dsa_layer(*a, wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k, wl.scale, sample=rows)
    return time.perf_counter() - t0, threads


def oracle_full(wl, threads=None):
    """The oracle on every query row of `wl`, as a cpu_baseline object."""
    dt, threads = oracle_seconds(wl, threads=threads)
    return {"value": wl.Nq / dt, "unit": UNIT, "cores": min(threads, wl.Nq), "kind": "oracle",
            "sample": f"every query row ({wl.Nq}), OpenMP over rows, {dt:.1f} s"}


def prefill_sample_rows(n_rows, total=512, seed=2):
    """Seeded query rows of a prefill for the oracle: every t < 64, every t in
    [2040, 2056] (around top_k), the rest drawn uniformly without repetition."""
    fixed = np.array([t for t in list(range(64)) + list(range(2040, 2057)) if t < n_rows])
    rest = np.setdiff1d(np.arange(n_rows), fixed)
    g = np.random.Generator(np.random.PCG64(seed))
    pick = g.choice(rest, size=max(0, min(rest.size, total - fixed.size)), replace=False)
    return np.sort(np.concatenate([fixed, pick])).astype(np.int64)


def prefill_oracle(wl, total=512):
    """The oracle on a seeded sample of a prefill's query rows, with the full
    run's time extrapolated by each row's work (indexer flops over its causal
    keys plus attention flops over its selected rows)."""
    rows = prefill_sample_rows(wl.Nq, total)
    dt, threads = oracle_seconds(wl, rows)
    pos = wl.positions()
    work = (2.0 * synth.HI * synth.DI * (pos + 1)
            + 2.0 * wl.H * (synth.D + synth.DV) * np.minimum(wl.top_k, pos + 1))
    full_s = dt * float(work.sum()) / float(work[rows].sum())
    return {"value": wl.Nq / full_s, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows.size} seeded query rows (all t < 64, t in [2040, 2056], the rest "
                      f"uniform) in {dt:.1f} s; value is EXTRAPOLATED to all {wl.Nq} rows "
                      f"by per-row work",
            "per_row_ms": dt / rows.size * 1e3, "extrapolated_full_s": full_s}


def cpu_baseline(wl):
    """The oracle, as it stands, on the host cores: all 4 query rows of one step."""
    import oracle
    oracle.build()
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    a = (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)
    t0 = time.perf_counter()
    oracle.dsa_layer(*a, wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k, wl.scale)
    dt = time.perf_counter() - t0
    return {"value": wl.Nq / dt, "unit": UNIT, "cores": min(threads, wl.Nq), "kind": "oracle",
            "sample": f"one full step of the workload ({wl.Nq} query rows, OpenMP over rows, "
                      f"{dt:.1f} s)"}


def profile_layer(spec, calls):
    """Runs dsa_layer_forward on one synthetic workload `calls` times, each
    after an L2 flush, checks the device status and exits (no timing: a
    driver for ncu, whose own launch list and counters are the output)."""
    from dsa_lightning_indexer_b200 import binding as bd
    kind, *dims = spec.split(",")
    if kind == "project":  # the indexer's input step on T new tokens (one per sequence)
        T = int(dims[0])
        dev = torch.device("cuda")
        g = torch.Generator(device=dev)
        g.manual_seed(7)

        def bf(*shape, std=1.0):
            return (torch.randn(*shape, generator=g, device=dev) * std).to(torch.bfloat16)
        lens = [131072] * T
        kv_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        b = bd.Batch(np.arange(T + 1, dtype=np.int32), kv_off, np.array(lens, np.int32), dev)
        args = (b, bf(T, D_MODEL), bf(T, D_Q), bf(4096, D_Q, std=D_Q ** -0.5),
                bf(128, D_MODEL, std=D_MODEL ** -0.5), bf(32, D_MODEL, std=D_MODEL ** -0.5),
                torch.empty(T, 32, 128, dtype=torch.bfloat16, device=dev),
                torch.zeros(int(kv_off[-1]), 128, dtype=torch.bfloat16, device=dev),
                torch.empty(T, 32, device=dev))
        ws = bd.indexer_project_workspace(b, D_MODEL, D_Q, dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # 2x the L2
        for i in range(calls):
            flush.fill_(i & 0xFF)
            bd.indexer_project(*args, ws)
        torch.cuda.synchronize()
        bd.check_device_status(ws)
        print(f"profile-layer input step, {T} tokens: {calls} calls ok", flush=True)
        return 0
    if kind == "decode":
        wl = synth.decode(int(dims[0]), int(dims[1]), 64, 2048, seed=3)
    elif kind == "prefill":
        wl = synth.prefill(int(dims[0]), 64, 2048, seed=2, planted=True)
    else:
        raise SystemExit(f"--profile-layer: unknown workload {spec!r}")
    dw = bd.DeviceWorkload(wl)
    out, lse, idx = dw.new_outputs()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # 2x the L2
    for i in range(calls):
        flush.fill_(i & 0xFF)
        dw.forward(out, lse, idx)
    torch.cuda.synchronize()
    bd.check_device_status(dw.ws)
    print(f"profile-layer {wl.name}: {calls} calls ok", flush=True)
    return 0


def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--prefill-steps", type=int, default=3)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the prefill measurement (profiling aid)")
    ap.add_argument("--prefill-tokens", type=int, default=16384)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kernel-times", action="store_true")
    ap.add_argument("--no-other", action="store_true",
                    help="skip the 32K decode and ragged-batch objects")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch each step directly instead of replaying a CUDA graph")
    ap.add_argument("--copies", type=int, default=2,
                    help="rotating copies of the decode inputs (L2 defeat)")
    ap.add_argument("--dry-run", action="store_true",
                    help="check the multi-rank launch path without a GPU (gloo)")
    ap.add_argument("--profile-layer", default=None, metavar="SPEC",
                    help="profiling aid: 'decode,B,L', 'prefill,T' or 'project,T' -- run "
                         "the layer (or the indexer's input step) --profile-calls times "
                         "(L2 flushed before each) and exit")
    ap.add_argument("--profile-calls", type=int, default=3)
    args = ap.parse_args()
    if args.profile_layer:
        return profile_layer(args.profile_layer, args.profile_calls)
    _, _, world = env_rank()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # One process per GPU: run this script again as --gpus ranks.
        return subprocess.call(replica_launch_cmd(sys.argv[1:], args.gpus))
    if "WORLD_SIZE" in os.environ and world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one rank per GPU",
              file=sys.stderr)
        return 2
    if args.dry_run:
        return dry_run(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
